// NVFP4 quantisation for the NVFP4 layer (page 1 of the MoK pages,
// "MoE layer as the bottleneck", names NVFP4 training kernels as earlier work;
// the format is NVIDIA's published one): E2M1 codes, one E4M3 scale per 16
// values along a GEMM's contraction dimension and one fp32 scale per tensor,
// gs = 2688 / amax(tensor), so that the tensor's largest magnitude maps to the
// largest value the two levels can hold (6 x 448).  Per block (nv_quant16 in
// ptx.cuh): s = e4m3((amax_block / 6) gs), codes e2m1(v gs / s); the value of a
// code is q s / gs, and a GEMM over two such operands multiplies its fp32
// accumulator by 1 / (gs_A gs_B) in the epilogue.
//
// Every tensor needs its amax before any of its blocks can be quantised, so
// each operand takes two passes: an amax reduction (max is order-free, so the
// atomicMax result is the same every run), then the quantisation.  For H the
// first pass is the gate/up GEMM's own epilogue, which writes H in fp32; for dA
// and dB (one tensor, the dgrad of gate/up's K = 2I operand) it is the dgrad of
// W_down's epilogue.
#include <cfloat>

#include "moe_internal.cuh"
#include "ptx.cuh"

namespace moe {

namespace {

__device__ __forceinline__ void unpack8_bf16(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 t = unpack_bf16(w[j]);
    f[2 * j] = t.x;
    f[2 * j + 1] = t.y;
  }
}

// |x| max over the block, one atomicMax per block (fp32 bits of a non-negative value order as
// unsigned integers)
__global__ void __launch_bounds__(256) k_nv_amax(const uint4* __restrict__ x, int64_t n8,
                                                 unsigned* __restrict__ amax) {
  __shared__ float part[8];
  float m = 0.f;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * 256) {
    float f[8];
    unpack8_bf16(__ldg(x + i), f);
#pragma unroll
    for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(f[j]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = part[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) b = fmaxf(b, part[w]);
    if (b > 0.f) atomicMax(amax, __float_as_uint(b));
  }
}

__global__ void k_nv_scale(const unsigned* __restrict__ amax, float* __restrict__ gs, int n) {
  const int i = threadIdx.x;
  if (i >= n) return;
  const float a = __uint_as_float(amax[i]);
  float g = a > 0.f ? __fdiv_rn(2688.0f, a) : 1.0f;
  if (g > FLT_MAX) g = FLT_MAX;  // amax below 2688 / FLT_MAX
  gs[i] = g;
}

// One warp per padded row in [*lo, *hi); lane i takes the row's 16-value blocks i, i + 32, ...
// (32 bytes of bf16 in, 8 bytes of codes out, contiguous across the warp).  Row R takes token
// row_asg[R] / k; live pad rows get zero codes and scale 0; dead pad rows are skipped (the GEMM
// reads them but no epilogue stores their rows).  With dst the bf16 row is stored there too
// (the bf16 weight gradients' operand; live pad rows zero).
__global__ void __launch_bounds__(256) k_nv_gather_x(const __nv_bfloat16* __restrict__ src,
                                                     const int* __restrict__ row_asg, const int* __restrict__ lo,
                                                     const int* __restrict__ hi, int k, int d,
                                                     const float* __restrict__ gsp, uint8_t* __restrict__ q,
                                                     uint8_t* __restrict__ qs, __nv_bfloat16* __restrict__ dst) {
  const int r0 = __ldg(lo), r1 = __ldg(hi);
  const float gs = __ldg(gsp);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = d / 16;
  for (int64_t R = r0 + static_cast<int64_t>(blockIdx.x) * 8 + warp; R < r1;
       R += static_cast<int64_t>(gridDim.x) * 8) {
    const int a = __ldg(row_asg + R);
    if (a == ROW_DEAD) continue;
    const uint4* in = a >= 0 ? reinterpret_cast<const uint4*>(src + static_cast<size_t>(a / k) * d) : nullptr;
    uint2* qd = reinterpret_cast<uint2*>(q + R * (d / 2));
    uint4* o = dst ? reinterpret_cast<uint4*>(dst + R * d) : nullptr;
    for (int c = lane; c < nb; c += 32) {
      float v[16];
      const uint4 u0 = in ? __ldg(in + 2 * c) : make_uint4(0, 0, 0, 0);
      const uint4 u1 = in ? __ldg(in + 2 * c + 1) : make_uint4(0, 0, 0, 0);
      unpack8_bf16(u0, v);
      unpack8_bf16(u1, v + 8);
      if (o) {
        o[2 * c] = u0;
        o[2 * c + 1] = u1;
      }
      uint32_t w[2];
      const uint8_t sb = nv_quant16(v, gs, w);
      qd[c] = make_uint2(w[0], w[1]);
      qs[nv_sf_index(static_cast<int>(R), 16 * c, d)] = sb;
    }
  }
}

// H (fp32 [RP, I], written by the gate/up GEMM for every live row) quantised along I; same
// walk as k_nv_gather_x with 64 bytes of fp32 in per block.  With dst (dA, dB in the backward)
// the rows are also stored in bf16 (round to nearest even), the weight gradients' operand.
__global__ void __launch_bounds__(256) k_nv_quant_h(const float* __restrict__ h, const int* __restrict__ row_asg,
                                                    const int* __restrict__ lo, const int* __restrict__ hi, int I,
                                                    const float* __restrict__ gsp, uint8_t* __restrict__ q,
                                                    uint8_t* __restrict__ qs, __nv_bfloat16* __restrict__ dst) {
  const int r0 = __ldg(lo), r1 = __ldg(hi);
  const float gs = __ldg(gsp);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = I / 16;
  for (int64_t R = r0 + static_cast<int64_t>(blockIdx.x) * 8 + warp; R < r1;
       R += static_cast<int64_t>(gridDim.x) * 8) {
    if (__ldg(row_asg + R) == ROW_DEAD) continue;
    const float4* in = reinterpret_cast<const float4*>(h + R * I);
    uint2* qd = reinterpret_cast<uint2*>(q + R * (I / 2));
    uint4* o = dst ? reinterpret_cast<uint4*>(dst + R * I) : nullptr;
    for (int c = lane; c < nb; c += 32) {
      float v[16];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 f = __ldg(in + 4 * c + j);
        v[4 * j] = f.x;
        v[4 * j + 1] = f.y;
        v[4 * j + 2] = f.z;
        v[4 * j + 3] = f.w;
      }
      if (o) {
        o[2 * c] = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                              pack_bf16(v[6], v[7]));
        o[2 * c + 1] = make_uint4(pack_bf16(v[8], v[9]), pack_bf16(v[10], v[11]), pack_bf16(v[12], v[13]),
                                  pack_bf16(v[14], v[15]));
      }
      uint32_t w[2];
      const uint8_t sb = nv_quant16(v, gs, w);
      qd[c] = make_uint2(w[0], w[1]);
      qs[nv_sf_index(static_cast<int>(R), 16 * c, I)] = sb;
    }
  }
}

// Rows of a row-major bf16 [R, K] quantised along K (no transpose: the backward's weight layouts
// W_down [El*I, d], W_gate / W_up [El*d, I]); one warp per row, lanes over its 16-value blocks.
__global__ void __launch_bounds__(256) k_nv_quant_rows(const __nv_bfloat16* __restrict__ src, int64_t R, int K,
                                                       const float* __restrict__ gsp, uint8_t* __restrict__ q,
                                                       uint8_t* __restrict__ qs) {
  const float gs = __ldg(gsp);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = K / 16;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + warp; r < R; r += static_cast<int64_t>(gridDim.x) * 8) {
    const uint4* in = reinterpret_cast<const uint4*>(src + r * K);
    uint2* qd = reinterpret_cast<uint2*>(q + r * (K / 2));
    for (int c = lane; c < nb; c += 32) {
      float v[16];
      unpack8_bf16(__ldg(in + 2 * c), v);
      unpack8_bf16(__ldg(in + 2 * c + 1), v + 8);
      uint32_t w[2];
      const uint8_t sb = nv_quant16(v, gs, w);
      qd[c] = make_uint2(w[0], w[1]);
      qs[nv_sf_index(static_cast<int>(r), 16 * c, K)] = sb;
    }
  }
}

// One block = 128 output rows x 128 K of a K-major NVFP4 weight [R_out, K], 128 threads.  The
// source tile (128 rows k of W [El][K][N], 128 output columns n) is staged in shared memory as
// bf16 as it is read (a warp loads 4 source rows x 128 bytes per step), then thread r quantises
// output row r: eight 16-value blocks from its column of the tile, 64 bytes of codes and eight
// scale bytes out.
//   paired = 0: output row el * N + n
//   paired = 1: gate/up, output rows per expert in blocks of 128 = 64 gate rows then 64 up rows
//               (columns j * 64 .. j * 64 + 63 of block j), gate under gs[0], up under gs[1]
constexpr int kNvPitch = 136;  // bf16 per staged row: 272 bytes, 16-byte aligned, rows 4 banks apart
__global__ void __launch_bounds__(128) k_nv_quant_weight(const __nv_bfloat16* __restrict__ src0,
                                                         const __nv_bfloat16* __restrict__ src1, int paired, int K,
                                                         int N, const float* __restrict__ gsp,
                                                         uint8_t* __restrict__ q, uint8_t* __restrict__ qs) {
  extern __shared__ __align__(16) uint8_t nv_tile_raw[];
  __nv_bfloat16* tile = reinterpret_cast<__nv_bfloat16*>(nv_tile_raw);
  const int k0 = blockIdx.x * 128;
  const int o0 = blockIdx.y * 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint4 u[16];
  int kk[16], nc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int g = 4 * i + warp;  // step g: source rows k0 + 4 (g / 2) .. + 3, output rows (g % 2) 64 .. + 63
    kk[i] = (g >> 1) * 4 + (lane >> 3);
    nc[i] = ((g & 1) * 8 + (lane & 7)) * 8;
    const int o = o0 + nc[i];
    const __nv_bfloat16* src = src0;
    size_t off;
    if (!paired) {
      const int el = o / N, n = o - el * N;
      off = (static_cast<size_t>(el) * K + k0 + kk[i]) * N + n;
    } else {
      const int el = o / (2 * N), w = o - el * 2 * N;
      const int j = w >> 7, hsel = (w >> 6) & 1, n = j * 64 + (w & 63);
      if (hsel) src = src1;
      off = (static_cast<size_t>(el) * K + k0 + kk[i]) * N + n;
    }
    u[i] = __ldg(reinterpret_cast<const uint4*>(src + off));
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) *reinterpret_cast<uint4*>(tile + kk[i] * kNvPitch + nc[i]) = u[i];
  __syncthreads();
  const int r = threadIdx.x;
  const int o = o0 + r;
  const float gs = __ldg(gsp + (paired && ((o % (2 * N)) >> 6) & 1 ? 1 : 0));
  uint32_t w[16];
  uint8_t sb[8];
#pragma unroll
  for (int b = 0; b < 8; ++b) {
    float v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __bfloat162float(tile[(b * 16 + i) * kNvPitch + r]);
    uint32_t qq[2];
    sb[b] = nv_quant16(v, gs, qq);
    w[2 * b] = qq[0];
    w[2 * b + 1] = qq[1];
  }
  uint4* d = reinterpret_cast<uint4*>(q + static_cast<size_t>(o) * (K / 2) + k0 / 2);
#pragma unroll
  for (int j = 0; j < 4; ++j) d[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
#pragma unroll
  for (int b = 0; b < 8; ++b) qs[nv_sf_index(o, k0 + 16 * b, K)] = sb[b];
}

int nv_grid_rows(int64_t rows) {
  const int64_t g = (rows + 7) / 8;
  return static_cast<int>(g < 1 ? 1 : (g > 148 * 8 ? 148 * 8 : g));
}

}  // namespace

cudaError_t launch_nv_amax(const __nv_bfloat16* x, int64_t n, unsigned* amax, cudaStream_t st) {
  const int64_t n8 = n / 8;
  int64_t g = (n8 + 255) / 256;
  if (g > 148 * 8) g = 148 * 8;
  if (g < 1) g = 1;
  k_nv_amax<<<static_cast<int>(g), 256, 0, st>>>(reinterpret_cast<const uint4*>(x), n8, amax);
  return cudaGetLastError();
}

cudaError_t launch_nv_scale(const unsigned* amax, float* gs, int n, cudaStream_t st) {
  k_nv_scale<<<1, 32, 0, st>>>(amax, gs, n);
  return cudaGetLastError();
}

cudaError_t launch_nv_gather_x(const Layout& L, const Ctx& c, const __nv_bfloat16* X, const float* gs, uint8_t* q,
                               uint8_t* qs, __nv_bfloat16* dst, cudaStream_t st) {
  k_nv_gather_x<<<nv_grid_rows(L.RP), 256, 0, st>>>(X, c.row_asg, c.poff, c.poff + L.El, L.k, L.d, gs, q, qs, dst);
  return cudaGetLastError();
}

cudaError_t launch_nv_quant_rows(const __nv_bfloat16* src, int64_t R, int K, const float* gs, uint8_t* q, uint8_t* qs,
                                 cudaStream_t st) {
  k_nv_quant_rows<<<nv_grid_rows(R), 256, 0, st>>>(src, R, K, gs, q, qs);
  return cudaGetLastError();
}

cudaError_t launch_nv_quant_h(const Layout& L, const Ctx& c, const float* h, const float* gs, uint8_t* q, uint8_t* qs,
                              __nv_bfloat16* dst, cudaStream_t st) {
  k_nv_quant_h<<<nv_grid_rows(L.RP), 256, 0, st>>>(h, c.row_asg, c.poff, c.poff + L.El, L.I, gs, q, qs, dst);
  return cudaGetLastError();
}

cudaError_t launch_nv_quant_weight(bool paired, const __nv_bfloat16* src0, const __nv_bfloat16* src1, int El, int K,
                                   int N, const float* gs, uint8_t* q, uint8_t* qs, cudaStream_t st) {
  const int smem = 128 * kNvPitch * 2;
  static bool configured[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(k_nv_quant_weight, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const int64_t R_out = static_cast<int64_t>(El) * N * (paired ? 2 : 1);
  k_nv_quant_weight<<<dim3(K / 128, static_cast<unsigned>(R_out / 128)), 128, smem, st>>>(src0, src1, paired ? 1 : 0,
                                                                                          K, N, gs, q, qs);
  return cudaGetLastError();
}

}  // namespace moe
