// MXFP8 quantisation: prepared weights (once per optimiser step) and the
// dispatched activations (fused into the gather that builds X_perm / dY_perm).
// Every 32-value block along a GEMM's contraction dimension gets one E8M0 scale
// (floor(log2 amax) - 8, the OCP MX rule) and E4M3 codes rounded to nearest
// even with saturation; scales are laid out in the 512-byte chunks the
// block-scaled MMA copies into tensor memory (see sf_index in ptx.cuh).
#include "moe_internal.cuh"
#include "ptx.cuh"

namespace moe {

// One block = 128 output rows x 128 K of a K-major fp8 weight [R_out, K], 128 threads.
//   mode 0: source [R_out, K] row-major (K contiguous)
//   mode 1: source [El][K][N] (N contiguous), output row el*N + n
//   mode 2: paired gate/up, source gate/up [El][K][N]; output rows per expert come in
//           blocks of 128 = 64 gate rows then 64 up rows (columns j*64 .. j*64+63)
// Each thread issues all 16 of its 16-byte source loads before it uses any of them.
// Mode 0 needs no transpose: thread (warp w, lane) owns the 32-value block lane % 4 of rows
// 32 i + 8 w + lane / 4 (i = 0..3), so the four lanes of a row read its 256 source bytes and
// write its 128 code bytes contiguously.  Modes 1 and 2 stage the tile in shared memory as it
// is read (bf16, one row per source row k, 128 output rows wide): a warp loads and stores 4
// source rows x 128 bytes, and thread r then quantises output row r reading its column.
constexpr int kQuantPitch = 136;  // bf16 elements per staged row: 272 bytes, 16-byte aligned, rows 4 banks apart

__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 t = unpack_bf16(w[j]);
    f[2 * j] = t.x;
    f[2 * j + 1] = t.y;
  }
}

__global__ void __launch_bounds__(128) k_quant_weight(const __nv_bfloat16* __restrict__ src0,
                                                      const __nv_bfloat16* __restrict__ src1, int mode, int K, int N,
                                                      uint8_t* __restrict__ q, uint8_t* __restrict__ qs) {
  extern __shared__ __align__(16) uint8_t tile_raw[];  // modes 1, 2: [128 k][kQuantPitch] bf16
  __nv_bfloat16* tile = reinterpret_cast<__nv_bfloat16*>(tile_raw);
  const int k0 = blockIdx.x * 128;
  const int o0 = blockIdx.y * 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint4 u[16];
  if (mode == 0) {
    const int blk = lane & 3;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = 32 * i + 8 * warp + (lane >> 2);
      const uint4* s4 = reinterpret_cast<const uint4*>(src0 + static_cast<size_t>(o0 + r) * K + k0 + blk * 32);
#pragma unroll
      for (int j = 0; j < 4; ++j) u[4 * i + j] = __ldg(s4 + j);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int o = o0 + 32 * i + 8 * warp + (lane >> 2);
      float v[32];
#pragma unroll
      for (int j = 0; j < 4; ++j) unpack8(u[4 * i + j], v + 8 * j);
      uint32_t w[8];
      const uint8_t sb = mx_quant32(v, w);
      uint4* d = reinterpret_cast<uint4*>(q + static_cast<size_t>(o) * K + k0 + blk * 32);
      d[0] = make_uint4(w[0], w[1], w[2], w[3]);
      d[1] = make_uint4(w[4], w[5], w[6], w[7]);
      qs[sf_index(o, k0 + blk * 32, K)] = sb;
    }
    return;
  }
  // modes 1, 2: load step g = 4 i + warp covers source rows k0 + 4 (g / 2) .. + 3 and the
  // 64 output rows (g % 2) * 64 .. + 63, eight per lane
  int kk[16], nc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int g = 4 * i + warp;
    kk[i] = (g >> 1) * 4 + (lane >> 3);
    nc[i] = ((g & 1) * 8 + (lane & 7)) * 8;
    const int o = o0 + nc[i];
    const __nv_bfloat16* src;
    size_t off;
    if (mode == 1) {
      const int el = o / N, n = o - el * N;
      src = src0;
      off = (static_cast<size_t>(el) * K + k0 + kk[i]) * N + n;
    } else {
      const int el = o / (2 * N), w = o - el * 2 * N;
      const int j = w >> 7, h = (w >> 6) & 1, n = j * 64 + (w & 63);
      src = h ? src1 : src0;
      off = (static_cast<size_t>(el) * K + k0 + kk[i]) * N + n;
    }
    u[i] = __ldg(reinterpret_cast<const uint4*>(src + off));
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) *reinterpret_cast<uint4*>(tile + kk[i] * kQuantPitch + nc[i]) = u[i];
  __syncthreads();
  const int r = threadIdx.x;
  const int o = o0 + r;
#pragma unroll 1
  for (int b = 0; b < 4; ++b) {
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __bfloat162float(tile[(b * 32 + i) * kQuantPitch + r]);
    uint32_t w[8];
    const uint8_t sb = mx_quant32(v, w);
    uint4* d = reinterpret_cast<uint4*>(q + static_cast<size_t>(o) * K + k0 + b * 32);
    d[0] = make_uint4(w[0], w[1], w[2], w[3]);
    d[1] = make_uint4(w[4], w[5], w[6], w[7]);
    qs[sf_index(o, k0 + b * 32, K)] = sb;
  }
}

// Dispatch / reverse-combine in MXFP8 mode: rows [lo, hi) of the padded layout get the bf16 row
// (kept for the weight gradients) and its fp8 codes + scales along d; dead pad rows are skipped.
__global__ void __launch_bounds__(256) k_gather_rows_mx(const __nv_bfloat16* __restrict__ src,
                                                        const int* __restrict__ row_asg, const int* __restrict__ lo,
                                                        const int* __restrict__ hi, int k, int d,
                                                        __nv_bfloat16* __restrict__ dst, uint8_t* __restrict__ q,
                                                        uint8_t* __restrict__ qs) {
  // One warp per padded row.  Lane i takes the row's 16-byte chunks i, i + 32, ... (8 values
  // each), four chunks in flight; the four lanes 4m .. 4m+3 hold one 32-value block and share
  // its amax through two xor shuffles.  d is a multiple of 256, so every lane runs the same
  // number of chunks and the shuffles see the whole warp.
  const int r0 = __ldg(lo), r1 = __ldg(hi);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nv = d / 8;
  for (int64_t R = r0 + blockIdx.x * 8 + warp; R < r1; R += gridDim.x * 8) {
    const int a = __ldg(row_asg + R);
    if (a == ROW_DEAD) continue;  // never read; a live pad row gets zero codes and scale 0
    const uint4* in = a >= 0 ? reinterpret_cast<const uint4*>(src + static_cast<size_t>(a / k) * d) : nullptr;
    uint4* o = reinterpret_cast<uint4*>(dst + R * d);
    uint2* qd = reinterpret_cast<uint2*>(q + R * d);
    for (int c0 = lane; c0 < nv; c0 += 128) {
      uint4 u[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = c0 + 32 * j;
        u[j] = (in != nullptr && c < nv) ? __ldg(in + c) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = c0 + 32 * j;
        if (c >= nv) break;  // the same for every lane of the warp
        o[c] = u[j];
        const uint32_t w4[4] = {u[j].x, u[j].y, u[j].z, u[j].w};
        float v[8];
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = unpack_bf16(w4[i]);
          v[2 * i] = f.x;
          v[2 * i + 1] = f.y;
          amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        // the block rule of mx_quant32: exponent floor(log2 amax) - 8, byte clamped to [0, 254]
        int byte = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFF) - 8;
        byte = byte < 0 ? 0 : (byte > 254 ? 254 : byte);
        const float inv = __uint_as_float(static_cast<uint32_t>(254 - byte) << 23);
        uint32_t w[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint16_t p0, p1;
          asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(p0) : "f"(v[4 * h] * inv), "f"(v[4 * h + 1] * inv));
          asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(p1) : "f"(v[4 * h + 2] * inv), "f"(v[4 * h + 3] * inv));
          w[h] = amax == 0.f ? 0u : (static_cast<uint32_t>(p0) | (static_cast<uint32_t>(p1) << 16));
        }
        qd[c] = make_uint2(w[0], w[1]);
        if ((lane & 3) == 0) qs[sf_index(static_cast<int>(R), c * 8, d)] = static_cast<uint8_t>(byte);
      }
    }
  }
}

cudaError_t launch_quant_weight(int mode, const __nv_bfloat16* src0, const __nv_bfloat16* src1, int64_t R_out, int K,
                                int N, uint8_t* q, uint8_t* qs, cudaStream_t st) {
  const int smem = 128 * kQuantPitch * 2;
  static bool configured[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(k_quant_weight, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  // mode 0 quantises from registers: without the transpose tile more blocks fit on an SM
  k_quant_weight<<<dim3(K / 128, static_cast<unsigned>(R_out / 128)), 128, mode == 0 ? 0 : smem, st>>>(
      src0, src1, mode, K, N, q, qs);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows_mx(const Layout& L, const Ctx& c, const __nv_bfloat16* src, __nv_bfloat16* dst,
                                  uint8_t* q, uint8_t* qs, cudaStream_t st) {
  const int64_t g = (L.RP + 7) / 8;
  const int grid = static_cast<int>(g < 148 * 8 ? (g > 0 ? g : 1) : 148 * 8);
  k_gather_rows_mx<<<grid, 256, 0, st>>>(src, c.row_asg, c.poff, c.poff + L.El, L.k, L.d, dst, q, qs);
  return cudaGetLastError();
}

}  // namespace moe
