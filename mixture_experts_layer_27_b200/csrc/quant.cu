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
// With a ring position (*shift), the bf16 row goes to row R + *shift, and so do the codes when
// shift_codes is set (a ring of codes beside the bf16 ring); otherwise the codes stay at row R.
__global__ void __launch_bounds__(256) k_gather_rows_mx(const __nv_bfloat16* __restrict__ src,
                                                        const int* __restrict__ row_asg, const int* __restrict__ lo,
                                                        const int* __restrict__ hi, const int* __restrict__ shift,
                                                        int shift_codes, int k, int d, __nv_bfloat16* __restrict__ dst,
                                                        uint8_t* __restrict__ q, uint8_t* __restrict__ qs) {
  // One warp per padded row.  Lane i takes the row's 16-byte chunks i, i + 32, ... (8 values
  // each), four chunks in flight; the four lanes 4m .. 4m+3 hold one 32-value block and share
  // its amax through two xor shuffles.  d is a multiple of 256, so every lane runs the same
  // number of chunks and the shuffles see the whole warp.
  const int r0 = __ldg(lo), r1 = __ldg(hi);
  const int64_t sh = shift ? __ldg(shift) : 0;
  const int64_t shq = shift_codes ? sh : 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nv = d / 8;
  for (int64_t R = r0 + blockIdx.x * 8 + warp; R < r1; R += gridDim.x * 8) {
    const int a = __ldg(row_asg + R);
    if (a == ROW_DEAD) continue;  // never read; a live pad row gets zero codes and scale 0
    const uint4* in = a >= 0 ? reinterpret_cast<const uint4*>(src + static_cast<size_t>(a / k) * d) : nullptr;
    uint4* o = reinterpret_cast<uint4*>(dst + (R + sh) * d);
    uint2* qd = reinterpret_cast<uint2*>(q + (R + shq) * d);
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
        if ((lane & 3) == 0) qs[sf_index(static_cast<int>(R + shq), c * 8, d)] = static_cast<uint8_t>(byte);
      }
    }
  }
}

// Dispatch / reverse-combine with MXFP8 weight gradients: rows [lo, hi) of the padded layout
// gathered from src (row R takes token row_asg[R] / k; pad rows are zero) and quantised twice,
// with no bf16 copy kept: along d (q_d, the dgrad and gate/up GEMMs' K) in the row-major layout
// of k_gather_rows_mx, and along the rows in blocks of 32 (q_r, the weight-gradient GEMMs' K) in
// the 128-row-tile-major layout (rowq_index, rowq_sf_index).  Every expert segment starts on a
// multiple of 128 and is its real rows rounded up to 128, so a tile lies in one expert and starts
// with a real row.
// Work items are (128-row tile, 64-column group) pairs, column groups fastest, dealt round-robin
// to a grid of resident CTAs (so CTAs running together share a tile's rows and every CTA gets the
// same number of items, give or take one).  A CTA walks its items through a ring of GQ_STAGES
// shared-memory stages: each
// thread copies four 16-byte pieces of a tile with cp.async (zero-filled for pad rows), so the
// copies of the next GQ_STAGES - 1 tiles are in flight (the row assignments they need are loaded
// one tile earlier still) while one tile is quantised: thread t takes the 32-value d-block t % 2
// of row t / 2 (dead pad rows are skipped: nothing reads them), and thread (column t % 64, block
// t / 64) the column's 32 rows (a block that starts past the expert's real rows is skipped: the
// GEMM never reads it).
constexpr int kQRowsPitch = 72;  // bf16 per staged row: 144 bytes (16-byte aligned; rows 4 banks apart)
constexpr int GQ_STAGES = 4;
constexpr size_t GQ_STAGE_BYTES = 128 * kQRowsPitch * 2 + 128 * 4;  // rows, then their row_asg
constexpr size_t GQ_SMEM = GQ_STAGES * GQ_STAGE_BYTES;

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool fill) {
  // src-size 0 writes 16 zero bytes and reads nothing
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(fill ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void gq_load_asg(const int* __restrict__ row_asg, int64_t r0, bool valid, int t,
                                            int (&a)[4]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) a[j] = valid ? __ldg(row_asg + r0 + ((t + 256 * j) >> 3)) : ROW_DEAD;
}
// Copies of one tile into a stage (rows of tokens a / k; zeros for pad rows) and its row flags.
__device__ __forceinline__ void gq_issue(const __nv_bfloat16* __restrict__ src, const int (&a)[4], int k, int d,
                                         int c0, int t, uint8_t* stage) {
  __nv_bfloat16* tile = reinterpret_cast<__nv_bfloat16*>(stage);
  int* flag = reinterpret_cast<int*>(stage + 128 * kQRowsPitch * 2);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int i = t + 256 * j;
    const bool real = a[j] >= 0;
    const __nv_bfloat16* g = src + (real ? static_cast<size_t>(a[j] / k) * d : 0) + c0 + (i & 7) * 8;
    cp_async16(tile + (i >> 3) * kQRowsPitch + (i & 7) * 8, g, real);
    if ((i & 7) == 0) flag[i >> 3] = a[j];
  }
}

__global__ void __launch_bounds__(256, 3) k_gather_quant2(const __nv_bfloat16* __restrict__ src,
                                                          const int* __restrict__ row_asg, const int* __restrict__ lo,
                                                          const int* __restrict__ hi, const int* __restrict__ dshift,
                                                          int k, int d, uint8_t* __restrict__ qd,
                                                          uint8_t* __restrict__ qds, uint8_t* __restrict__ qr,
                                                          uint8_t* __restrict__ qrs) {
  extern __shared__ __align__(16) uint8_t gq_smem[];
  const int64_t r_lo = __ldg(lo);
  const int64_t dsh = dshift ? __ldg(dshift) : 0;  // the codes along d at a ring position
  const int ng = d / 64;                              // column groups
  const int64_t items = (__ldg(hi) - r_lo) / 128 * ng;  // (tile, column group) pairs
  const int t = threadIdx.x;
  auto row0 = [&](int64_t it) { return r_lo + (it / ng) * 128; };
  auto col0 = [&](int64_t it) { return static_cast<int>(it % ng) * 64; };
  int a[4];
  // prologue: items 0 .. GQ_STAGES - 2 of this CTA in flight, the row assignments of the next one loaded
#pragma unroll
  for (int s = 0; s < GQ_STAGES - 1; ++s) {
    const int64_t it = blockIdx.x + static_cast<int64_t>(s) * gridDim.x;
    gq_load_asg(row_asg, row0(it), it < items, t, a);
    if (it < items) gq_issue(src, a, k, d, col0(it), t, gq_smem + s * GQ_STAGE_BYTES);
    cp_async_commit();
  }
  {
    const int64_t it = blockIdx.x + static_cast<int64_t>(GQ_STAGES - 1) * gridDim.x;
    gq_load_asg(row_asg, row0(it), it < items, t, a);
  }
  int n = 0;
  for (int64_t it = blockIdx.x; it < items; it += gridDim.x, ++n) {
    const int64_t r0 = row0(it);
    const int c0 = col0(it);
    cp_async_wait<GQ_STAGES - 2>();  // this thread's copies of item n have landed
    __syncthreads();                 // everyone's; and item n - 1's stage is no longer read
    {
      const int64_t in = it + static_cast<int64_t>(GQ_STAGES - 1) * gridDim.x;  // into the stage item n - 1 used
      if (in < items) gq_issue(src, a, k, d, col0(in), t, gq_smem + ((n + GQ_STAGES - 1) % GQ_STAGES) * GQ_STAGE_BYTES);
      cp_async_commit();
      const int64_t in2 = in + gridDim.x;
      gq_load_asg(row_asg, row0(in2), in2 < items, t, a);
    }
    const uint8_t* stage = gq_smem + (n % GQ_STAGES) * GQ_STAGE_BYTES;
    const __nv_bfloat16* tile = reinterpret_cast<const __nv_bfloat16*>(stage);
    const int* flag = reinterpret_cast<const int*>(stage + 128 * kQRowsPitch * 2);
    {  // along d: block t % 2 (32 columns) of row t / 2
      const int rr = t >> 1, blk = t & 1;
      if (flag[rr] != ROW_DEAD) {
        float v[32];
        const uint4* s4 = reinterpret_cast<const uint4*>(tile + rr * kQRowsPitch + blk * 32);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const uint4 w4 = s4[q4];
          const uint32_t ww[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float2 f = unpack_bf16(ww[h]);
            v[8 * q4 + 2 * h] = f.x;
            v[8 * q4 + 2 * h + 1] = f.y;
          }
        }
        uint32_t w[8];
        const uint8_t sb = mx_quant32(v, w);
        const int64_t R = r0 + rr + dsh;
        uint4* dst = reinterpret_cast<uint4*>(qd + R * d + c0 + blk * 32);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
        qds[sf_index(static_cast<int>(R), c0 + blk * 32, d)] = sb;
      }
    }
    {  // along the rows: rows 32 b .. 32 b + 31 of column c
      const int c = t & 63, b = t >> 6;
      if (flag[b * 32] >= 0) {
        float v[32];
#pragma unroll
        for (int r = 0; r < 32; ++r) v[r] = __bfloat162float(tile[(b * 32 + r) * kQRowsPitch + c]);
        uint32_t w[8];
        const uint8_t sb = mx_quant32(v, w);
        uint4* dst = reinterpret_cast<uint4*>(qr + rowq_index(c0 + c, r0 + b * 32, d));
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
        qrs[rowq_sf_index(c0 + c, r0 + b * 32, d)] = sb;
      }
    }
  }
  cp_async_wait<0>();  // no copy outlives the CTA's shared memory
}

cudaError_t launch_gather_quant2_range(const Layout& L, const Ctx& c, const __nv_bfloat16* src, const int* lo,
                                       const int* hi, const int* dshift, uint8_t* qd, uint8_t* qds, uint8_t* qr,
                                       uint8_t* qrs, cudaStream_t st) {
  static bool configured[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    const cudaError_t e =
        cudaFuncSetAttribute(k_gather_quant2, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(GQ_SMEM));
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  // The padded-row capacity RP is a worst case (every token's k assignments local): the routed
  // rows are often far fewer, so the grid is one wave of resident CTAs (three of 256 threads fit
  // an SM) that deals the items among themselves, instead of one CTA per possible item.
  int sms = 148;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) sms = 148;
  const int64_t max_items = L.RP / 128 * (L.d / 64);
  int64_t grid = static_cast<int64_t>(sms) * 3;
  if (grid > max_items) grid = max_items;
  if (grid < 1) grid = 1;
  k_gather_quant2<<<static_cast<unsigned>(grid), 256, GQ_SMEM, st>>>(src, c.row_asg, lo, hi, dshift, L.k, L.d, qd,
                                                                      qds, qr, qrs);
  return cudaGetLastError();
}

cudaError_t launch_gather_quant2(const Layout& L, const Ctx& c, const __nv_bfloat16* src, uint8_t* qd, uint8_t* qds,
                                 uint8_t* qr, uint8_t* qrs, cudaStream_t st) {
  if (L.M > 0)  // all rows of the stream
    return launch_gather_quant2_range(L, c, src, c.tab.seg_poff, c.tab.seg_poff + L.M * L.El, nullptr, qd, qds, qr,
                                      qrs, st);
  return launch_gather_quant2_range(L, c, src, c.poff, c.poff + L.El, nullptr, qd, qds, qr, qrs, st);
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

cudaError_t launch_gather_range_mx(const Layout& L, const Ctx& c, const __nv_bfloat16* src, const int* lo,
                                   const int* hi, const int* shift, bool shift_codes, int64_t max_rows,
                                   __nv_bfloat16* dst, uint8_t* q, uint8_t* qs, cudaStream_t st) {
  const int64_t g = (max_rows + 7) / 8;
  const int grid = static_cast<int>(g < 148 * 8 ? (g > 0 ? g : 1) : 148 * 8);
  k_gather_rows_mx<<<grid, 256, 0, st>>>(src, c.row_asg, lo, hi, shift, shift_codes ? 1 : 0, L.k, L.d, dst, q, qs);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows_mx(const Layout& L, const Ctx& c, const __nv_bfloat16* src, __nv_bfloat16* dst,
                                  uint8_t* q, uint8_t* qs, cudaStream_t st) {
  if (L.M > 0)  // all rows of the stream
    return launch_gather_range_mx(L, c, src, c.tab.seg_poff, c.tab.seg_poff + L.M * L.El, nullptr, false, L.RP, dst,
                                  q, qs, st);
  return launch_gather_range_mx(L, c, src, c.poff, c.poff + L.El, nullptr, false, L.RP, dst, q, qs, st);
}

}  // namespace moe
