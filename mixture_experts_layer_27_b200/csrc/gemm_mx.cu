// MXFP8 expert-grouped GEMMs (page 1 of the MoK pages, closing paragraph of
// "Three design decisions that matter": BF16 and MXFP8 precision modes).
//
// Same persistent warp-specialised structure as the bf16 engine (gemm.cu), with
// tcgen05.mma kind::mxf8f6f4.block_scale: E4M3 operands, one E8M0 scale per 32
// values along K.  Every stage carries a 128-byte-deep K slice of a 128-row A
// tile and a 256-row B tile, with their 512-byte scale chunks (one for A, two
// for B); the MMA thread copies the chunks into a per-stage TMEM slot
// (tcgen05.cp) and issues four K = 32 MMAs whose sf_id selects the K block.
// Output tiles are 128 x 256 (gate/up, down, dgrad of gate/up): 32 KB of fp8
// weights per stage keeps as many weight bytes in flight per SM as the bf16
// engine; the fp32 accumulator takes 256 TMEM columns and the scale slots sit
// above it, so there is one accumulator (the producer keeps loading while the
// epilogue drains it).  The dgrad of W_down, whose epilogue reads A and B and
// writes five outputs, uses 128 x 128 tiles with two accumulators instead, so
// its epilogue overlaps the next tile's MMAs.
#include "moe_internal.cuh"
#include "ptx.cuh"

namespace moe {

struct MxTile {
  int el, m0, n0, nt, nk;
};

template <int KIND>
__device__ __forceinline__ int mx_ntiles_n(const MxParams& p) {
  if (KIND == MX_GATEUP) return p.I / (mx_bn(KIND) / 2);  // per tile: [64 gate | 64 up] column pairs
  if (KIND == MX_DGRAD_DOWN) return p.I / mx_bn(KIND);
  return p.d / mx_bn(KIND);  // MX_DOWN, MX_DGRAD_GATEUP
}
template <int KIND>
__device__ __forceinline__ int mx_kblocks(const MxParams& p) {
  if (KIND == MX_GATEUP || KIND == MX_DGRAD_DOWN) return p.d / 128;
  if (KIND == MX_DOWN) return p.I / 128;
  return 2 * p.I / 128;
}

__device__ __forceinline__ int mx_segment_of_row(const int* poff, int nseg, int R) {
  int lo = 0, hi = nseg - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(poff + mid) <= R) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int KIND>
__device__ __forceinline__ int mx_num_tiles(const MxParams& p) {
  return ((__ldg(p.poff + p.nseg) - __ldg(p.poff)) / 128) * mx_ntiles_n<KIND>(p);
}

template <int KIND>
__device__ __forceinline__ MxTile mx_decode(const MxParams& p, int t) {
  const int NT = mx_ntiles_n<KIND>(p);
  const int base = __ldg(p.poff);
  const int seg = mx_segment_of_row(p.poff, p.nseg, base + (t / NT) * 128);
  const int p0 = __ldg(p.poff + seg), p1 = __ldg(p.poff + seg + 1);
  const int mte = (p1 - p0) / 128;
  const int local = t - NT * ((p0 - base) / 128);
  const int nt = local / mte, mi = local - nt * mte;
  MxTile tl;
  tl.el = seg % p.El;
  tl.m0 = p0 + mi * 128;
  tl.nt = nt;
  tl.n0 = nt * (KIND == MX_GATEUP ? mx_bn(KIND) / 2 : mx_bn(KIND));  // MX_GATEUP: first column of H / A / B
  tl.nk = mx_kblocks<KIND>(p);
  return tl;
}

// TMA + bulk loads of K block kb (128 elements) of tile tl into one stage.
template <int KIND>
__device__ __forceinline__ void mx_load(const MxParams& p, const MxTile& tl, int kb, uint8_t* st, uint64_t* bar,
                                        uint64_t pol_act, uint64_t pol_w) {
  uint8_t* sA = st;
  constexpr int BN = mx_bn(KIND);
  uint8_t* sB = st + MX_A_BYTES;
  uint8_t* sSF = sB + BN * 128;  // the A chunk, then a B chunk per 128 rows of the B tile
  const CUtensorMap* ma = &p.ta0;
  const CUtensorMap* mb = &p.tb0;
  const uint8_t* sfa = p.sfa0;
  const uint8_t* sfb = p.sfb0;
  int kl = kb, brow, KA, KB;
  if constexpr (KIND == MX_GATEUP) {
    brow = tl.el * 2 * p.I + tl.nt * BN;  // blocks of paired [64 gate | 64 up] rows of the prepared weight
    KA = KB = p.d;
  } else if constexpr (KIND == MX_DOWN) {
    brow = tl.el * p.d + tl.n0;
    KA = KB = p.I;
  } else if constexpr (KIND == MX_DGRAD_DOWN) {
    brow = tl.el * p.I + tl.n0;
    KA = KB = p.d;
  } else {
    const int half = p.I / 128;
    if (kb >= half) {  // second half of K: dB with W_up
      kl = kb - half;
      ma = &p.ta1;
      mb = &p.tb1;
      sfa = p.sfa1;
      sfb = p.sfb1;
    }
    brow = tl.el * p.d + tl.n0;
    KA = KB = p.I;
  }
  tma_load_2d(sA, ma, bar, kl * 128, tl.m0, pol_act);
  tma_load_2d(sB, mb, bar, kl * 128, brow, pol_w);
  bulk_load(sSF, sfa + (static_cast<size_t>(tl.m0 >> 7) * (KA >> 7) + kl) * 512, 512, bar);
  bulk_load(sSF + 512, sfb + (static_cast<size_t>(brow >> 7) * (KB >> 7) + kl) * 512, 512, bar);
  if constexpr (BN == 256)
    bulk_load(sSF + 1024, sfb + (static_cast<size_t>((brow >> 7) + 1) * (KB >> 7) + kl) * 512, 512, bar);
}

__device__ __forceinline__ float mx_sigmoid(float a) { return 1.0f / (1.0f + expf(-a)); }
// silu(a) = a / (1 + e^-a) with the fast exponential and reciprocal intrinsics: its result only
// feeds H, which is rounded to E4M3 (3 mantissa bits) for the down GEMM, and the intrinsics'
// errors are a few ulp of fp32.
__device__ __forceinline__ float mx_silu_fast(float a) { return a * __frcp_rn(1.0f + __expf(-a)); }

__device__ __forceinline__ void mx_store_bf16_32(__nv_bfloat16* dst, const float (&v)[32]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    d4[q] = make_uint4(pack_bf16(v[8 * q], v[8 * q + 1]), pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                       pack_bf16(v[8 * q + 4], v[8 * q + 5]), pack_bf16(v[8 * q + 6], v[8 * q + 7]));
}
__device__ __forceinline__ void mx_load_bf16_32(const __nv_bfloat16* src, float (&v)[32]) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 u = s4[q];
    float2 f;
    f = unpack_bf16(u.x); v[8 * q + 0] = f.x; v[8 * q + 1] = f.y;
    f = unpack_bf16(u.y); v[8 * q + 2] = f.x; v[8 * q + 3] = f.y;
    f = unpack_bf16(u.z); v[8 * q + 4] = f.x; v[8 * q + 5] = f.y;
    f = unpack_bf16(u.w); v[8 * q + 6] = f.x; v[8 * q + 7] = f.y;
  }
}
// quantise a 32-value block and store its 32 codes and scale byte (row R, column c0 of a [*, K] operand)
__device__ __forceinline__ void mx_store_q32(uint8_t* q, uint8_t* qs, int R, int c0, int K, const float (&v)[32]) {
  uint32_t w[8];
  const uint8_t sb = mx_quant32(v, w);
  uint4* d = reinterpret_cast<uint4*>(q + static_cast<size_t>(R) * K + c0);
  d[0] = make_uint4(w[0], w[1], w[2], w[3]);
  d[1] = make_uint4(w[4], w[5], w[6], w[7]);
  qs[sf_index(R, c0, K)] = sb;
}

// Rows past a segment's live pad rows (row_asg == ROW_DEAD) store nothing: no later kernel
// reads them.
// [cbeg, cend): this warp's share of the accumulator's 32-column chunks (all of them, or half
// when two warps share a TMEM lane quarter).
template <int KIND>
__device__ __forceinline__ void mx_epilogue(const MxParams& p, const MxTile& tl, int row, uint32_t taddr, int cbeg,
                                            int cend) {
  const int R = tl.m0 + row;
  const size_t Rz = static_cast<size_t>(R);
  const bool live = __ldg(p.row_asg + R) != ROW_DEAD;
  constexpr int BN = mx_bn(KIND);
  if constexpr (KIND == MX_GATEUP) {
#pragma unroll 1
    for (int c = cbeg; c < cend; ++c) {  // 32 H columns each; accumulator: [64 gate | 64 up] per 128
      const int j = c >> 1, c32 = (c & 1) * 32;
      float a[32], b[32], h[32];
      tmem_ld32(taddr + j * 128 + c32, a);       // gate
      tmem_ld32(taddr + j * 128 + 64 + c32, b);  // up
#pragma unroll
      for (int i = 0; i < 32; ++i) h[i] = mx_silu_fast(a[i]) * b[i];
      const int col = tl.n0 + j * 64 + c32;
      if (live) {
        mx_store_bf16_32(p.out0 + Rz * p.I + col, a);
        mx_store_bf16_32(p.out1 + Rz * p.I + col, b);
        mx_store_q32(p.q0, p.qs0, R, col, p.I, h);  // H, the down GEMM's A operand (K = I)
      }
    }
  } else if constexpr (KIND == MX_DOWN) {
    const float g = p.row_gate[R];
#pragma unroll 1
    for (int c = cbeg; c < cend; ++c) {
      float o[32];
      tmem_ld32(taddr + c * 32, o);
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] *= g;
      if (live) mx_store_bf16_32(p.out0 + Rz * p.d + tl.n0 + c * 32, o);
    }
  } else if constexpr (KIND == MX_DGRAD_DOWN) {
    const float g = p.row_gate[R];
    float dg = 0.f;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      float dh[32], a[32], b[32];
      tmem_ld32(taddr + c * 32, dh);
      const int col = tl.n0 + c * 32;
      if (live) {
        mx_load_bf16_32(p.in0 + Rz * p.I + col, a);
        mx_load_bf16_32(p.in1 + Rz * p.I + col, b);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) a[i] = b[i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float s = mx_sigmoid(a[i]);
        const float sl = a[i] * s;
        const float hh = sl * b[i];
        dg = fmaf(dh[i], hh, dg);
        const float dhg = g * dh[i];
        a[i] = dhg * b[i] * (s * (1.0f + a[i] * (1.0f - s)));  // dA
        b[i] = dhg * sl;                                       // dB
        dh[i] = g * hh;                                        // Hg
      }
      if (live) {
        mx_store_bf16_32(p.out0 + Rz * p.I + col, a);
        mx_store_bf16_32(p.out1 + Rz * p.I + col, b);
        mx_store_bf16_32(p.out2 + Rz * p.I + col, dh);
        mx_store_q32(p.q0, p.qs0, R, col, p.I, a);  // dA, dB: the gate/up dgrad's A operands (K = I)
        mx_store_q32(p.q1, p.qs1, R, col, p.I, b);
      }
    }
    if (live) p.outf[Rz * (p.I / BN) + tl.nt] = dg;
  } else {
#pragma unroll 1
    for (int c = cbeg; c < cend; ++c) {
      float v[32];
      tmem_ld32(taddr + c * 32, v);
      if (live) mx_store_bf16_32(p.out0 + Rz * p.d + tl.n0 + c * 32, v);
    }
  }
}

__device__ __forceinline__ void mx_wait_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > MOE_SPIN_CYCLES) return;
  }
}

template <int KIND>
__global__ void __launch_bounds__(mx_threads(KIND), 1) k_moe_gemm_mx(const __grid_constant__ MxParams p) {
  constexpr int BN = mx_bn(KIND), ACCS = mx_accs(KIND), STAGES = mx_stages(KIND), EPI = mx_epi_warps(KIND);
  constexpr size_t SB = mx_stage_bytes(KIND);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * SB);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;  // per accumulator
  uint64_t* tempty = tfull + ACCS;
  uint64_t* drain = tempty + ACCS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < ACCS; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], EPI);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&p.ta0);
    prefetch_tmap(&p.ta1);
    prefetch_tmap(&p.tb0);
    prefetch_tmap(&p.tb1);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const int ntiles = mx_num_tiles<KIND>(p);

  if (warp == 0) {
    if (lane == 0) {  // TMA producer
      const uint64_t pol_act = policy_evict_last();
      const uint64_t pol_w = policy_evict_first();
      int stage = 0;
      uint32_t phase = 0;
      int last_parity[MX_MAX_STAGES];
      for (int s = 0; s < STAGES; ++s) last_parity[s] = -1;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        const MxTile tl = mx_decode<KIND>(p, t);
        for (int kb = 0; kb < tl.nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, p.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>(mx_stage_tx(KIND)));
          mx_load<KIND>(p, tl, kb, smem + stage * SB, &full[stage], pol_act, pol_w);
          last_parity[stage] = static_cast<int>(phase);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok)
        for (int s = 0; s < STAGES; ++s)
          if (last_parity[s] >= 0) mx_wait_drain(&full[s], static_cast<uint32_t>(last_parity[s]));
    }
  } else if (warp == 1) {
    if (lane == 0) {  // MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++it) {
        const MxTile tl = mx_decode<KIND>(p, t);
        const int acc = it % ACCS;
        const uint32_t accp = (it / ACCS) & 1;
        if (!mbar_wait(&tempty[acc], accp ^ 1, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dtm = tbase + acc * BN;  // accumulators in columns [0, 256)
        for (int kb = 0; kb < tl.nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * SB);
          const uint32_t b0 = a0 + static_cast<uint32_t>(MX_A_BYTES);
          const uint32_t sf0 = b0 + static_cast<uint32_t>(BN * 128);
          // scale slot of this stage: 16 columns from column 256 on; A in the first 4,
          // B (rows 0..127, then 128..255) in the columns from 8 on
          const uint32_t sfa_t = tbase + 256 + stage * 16, sfb_t = sfa_t + 8;
          tc_cp_sf(sfa_t, sf0);
          tc_cp_sf(sfb_t, sf0 + 512);
          if constexpr (BN == 256) tc_cp_sf(sfb_t + 4, sf0 + 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_mxf8(dtm, sdesc_sw128(a0 + kk * 32, 16, 1024), sdesc_sw128(b0 + kk * 32, 16, 1024),
                      idesc_mxf8(128, BN, static_cast<uint32_t>(kk)), sfa_t, sfb_t, (kb | kk) != 0 ? 1u : 0u);
          umma_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
      }
      umma_commit(drain);
      mx_wait_drain(drain, 0);
    }
  } else {  // epilogue warps 2 .. 2 + EPI - 1
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    constexpr int NCH = KIND == MX_GATEUP ? BN / 64 : BN / 32;  // 32-column chunks of the epilogue
    const int half = EPI == 8 ? (warp - 2) >> 2 : 0;
    const int cbeg = half * (NCH * 4 / EPI), cend = cbeg + NCH * 4 / EPI;
    int it = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++it) {
      const MxTile tl = mx_decode<KIND>(p, t);
      const int acc = it % ACCS;
      const uint32_t accp = (it / ACCS) & 1;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&tfull[acc], accp, p.status) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      __syncwarp();
      tc_fence_after();
      mx_epilogue<KIND>(p, tl, row, tbase + (static_cast<uint32_t>(quarter * 32) << 16) + acc * BN, cbeg, cend);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

template <int KIND>
static cudaError_t mx_launch_kind(const MxParams& p, int grid, cudaStream_t st) {
  static bool configured[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(k_moe_gemm_mx<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(mx_smem_bytes(KIND)));
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  k_moe_gemm_mx<KIND><<<grid, mx_threads(KIND), mx_smem_bytes(KIND), st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_gemm_mx(MxKind kind, const MxParams& p, int grid, cudaStream_t st) {
  switch (kind) {
    case MX_GATEUP: return mx_launch_kind<MX_GATEUP>(p, grid, st);
    case MX_DOWN: return mx_launch_kind<MX_DOWN>(p, grid, st);
    case MX_DGRAD_DOWN: return mx_launch_kind<MX_DGRAD_DOWN>(p, grid, st);
    case MX_DGRAD_GATEUP: return mx_launch_kind<MX_DGRAD_GATEUP>(p, grid, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace moe
