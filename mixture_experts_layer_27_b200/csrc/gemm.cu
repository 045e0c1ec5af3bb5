// Expert-grouped GEMMs of the MoE layer on sm_100a tensor cores.
//
// One persistent, warp-specialised kernel template serves the six GEMMs of
// the forward and backward ("expert-grouped GEMM", page 1 of the MoK pages,
// "Three design decisions that matter", bullet 2) and the router GEMM:
//
//   warp 0      one thread issues TMA tile loads into a 3-4 stage smem ring
//   warp 1      allocates 512 TMEM columns; one thread issues tcgen05.mma
//   warps 2..5  epilogue: tcgen05.ld from TMEM, fused math, global stores
//               (the wgrad GEMMs stage their tiles in smem for TMA stores)
//
// The output tile is 128 x 256 (fp32 in TMEM), K advances 64 at a time
// (one 128-byte swizzle atom of bf16).  Two accumulators let the epilogue of
// tile i overlap the MMAs of tile i+1.  Every output element is produced by
// one CTA with one fixed K order, so results are bit-reproducible (no
// atomics; the router GEMM's fixed K splits are summed in split order by the
// top-k kernel).  Expert tiles are listed on the device from the padded
// expert offsets, so the host never needs the routing result.
#include <cstdio>

#include "moe_internal.cuh"
#include "ptx.cuh"

namespace moe {

template <int KIND>
struct Traits;
template <> struct Traits<G_GATEUP>       { static constexpr bool A_MN = false, B_MN = true; };
template <> struct Traits<G_DOWN>         { static constexpr bool A_MN = false, B_MN = true; };
template <> struct Traits<G_DGRAD_DOWN>   { static constexpr bool A_MN = false, B_MN = false; };
template <> struct Traits<G_DGRAD_GATEUP> { static constexpr bool A_MN = false, B_MN = false; };
template <> struct Traits<G_WGRAD_GATEUP> { static constexpr bool A_MN = true, B_MN = true; };
template <> struct Traits<G_WGRAD_DOWN>   { static constexpr bool A_MN = true, B_MN = true; };
template <> struct Traits<G_ROUTER>       { static constexpr bool A_MN = false, B_MN = false; };
template <> struct Traits<G_ROUTER_WGRAD> { static constexpr bool A_MN = true, B_MN = true; };

// The wgrad GEMMs have short K loops (one expert's rows) and write a full
// 128 x 256 output tile per tile: they trade a smem stage for a staging
// buffer that feeds TMA stores.
template <int KIND>
constexpr bool is_wgrad() { return KIND == G_WGRAD_GATEUP || KIND == G_WGRAD_DOWN; }
template <int KIND>
constexpr int stages_of() { return is_wgrad<KIND>() ? 3 : GEMM_STAGES; }
// With SCHED, the tiles a CTA works on are decoded once, by a scheduler warp, into a ring of
// SCHED_DEPTH entries that the producer, the MMA issuer and the epilogue warps read in order
// (the ring is deeper than the producer runs ahead of the epilogue, so it never throttles it).
// That takes the decode's global-load latency off the epilogue's path, which is the critical
// one in a weight-gradient GEMM whose tiles have one or two K blocks (64 tokens per expert:
// the kernel is bound by its gradient stores).  Where tiles have many K blocks the MMA issuer
// and the producer are critical, and there every role decodes its own tiles (measured 2-10%
// faster than the ring for the long-K weight gradients and the other kinds).
constexpr int SCHED_DEPTH = 8;
constexpr size_t SCHED_TAIL_BYTES = 1024;  // barriers, TMEM slot and the tile ring
template <int KIND>
constexpr size_t smem_bytes() {
  return stages_of<KIND>() * GEMM_STAGE_BYTES + (is_wgrad<KIND>() ? GEMM_STAGE_OUT_BYTES : 0) + 1024 +
         SCHED_TAIL_BYTES;
}

struct Tile {
  int t;    // tile index; -1 marks the end of this CTA's tiles
  int m;    // macrobatch (wgrad: first macrobatch of the chunk)
  int shift;  // row shift of the X_perm operand (ring position) / wgrad: last macrobatch + 1
  int el;   // local expert
  int m0;   // first output row (padded token row, or weight row for wgrad)
  int n0;   // first output column
  int nt;   // n-tile index
  int kb0;  // first 64-wide K block (wgrad: first padded row / 64)
  int nk;   // number of K blocks
  int u;    // unit kind of the fused forward (FusedUnit); unused elsewhere
};

template <int KIND>
__device__ __forceinline__ int ntiles_n(const GemmParams& p) {
  if (KIND == G_GATEUP) return p.I / 128;  // 128 gate + 128 up columns per tile
  if (KIND == G_DOWN || KIND == G_DGRAD_GATEUP || KIND == G_WGRAD_DOWN) return p.d / 256;
  if (KIND == G_DGRAD_DOWN) return p.I / 256;
  return 2 * p.I / 256;  // G_WGRAD_GATEUP: gate n-tiles then up n-tiles
}
template <int KIND>
__device__ __forceinline__ int mtiles_w(const GemmParams& p) {
  return KIND == G_WGRAD_GATEUP ? p.d / 128 : p.I / 128;
}

// Segment s with poff[s] <= R < poff[s+1] (the largest s with poff[s] <= R; empty
// segments before a non-empty one are skipped because they share its start).
__device__ __forceinline__ int segment_of_row(const int* poff, int nseg, int R) {
  int lo = 0, hi = nseg - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(poff + mid) <= R) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int KIND>
__device__ __forceinline__ int num_tiles(const GemmParams& p) {
  if (KIND == G_ROUTER) return ((p.T + 127) / 128) * ((p.E + 255) / 256) * p.splits;
  if (KIND == G_ROUTER_WGRAD) return (p.d / 128) * ((p.E + 255) / 256);
  if (KIND <= G_DGRAD_GATEUP) return ((__ldg(p.poff + p.nseg) - __ldg(p.poff)) / 128) * ntiles_n<KIND>(p);
  if (p.chunk && __ldg(p.chunk + 2) == 0) return 0;  // chunk not used by this routing
  return p.El * mtiles_w<KIND>(p) * ntiles_n<KIND>(p);
}

// Real rows of segment (macrobatch m, local expert el): a prefix of the segment, pad rows after.
__device__ __forceinline__ int seg_rows(const GemmParams& p, int m, int el) {
  const int tot = __ldg(p.cnt + el);
  if (!p.cum) return tot;
  const int nm = p.nseg / p.El;
  return (m + 1 < nm ? __ldg(p.cum + (m + 1) * p.El + el) : tot) - __ldg(p.cum + m * p.El + el);
}
// K blocks (64 rows) of a segment in a weight-gradient GEMM: its real rows rounded up to 64, so
// the 128-row padding adds no K work.  In the last block the MMAs skip the K16 steps past the
// real rows; the pad rows of the last step they issue (up to the next multiple of 16) are the
// segment's "live" pad rows, which every producer writes as zeros.
__device__ __forceinline__ int wgrad_kblocks(const GemmParams& p, int m, int el) { return (seg_rows(p, m, el) + 63) / 64; }

// 64-token K blocks of one dl term in the router weight gradient: all T tokens, or the
// listed ones (their number is on the device)
__device__ __forceinline__ int router_wgrad_kblocks(const GemmParams& p) {
  return ((p.act_n ? __ldg(p.act_n) : p.T) + 63) / 64;
}

template <int KIND>
__device__ __forceinline__ Tile decode(const GemmParams& p, int t) {
  Tile tl;
  tl.t = t;
  if constexpr (KIND == G_ROUTER) {
    // tile = (m-tile, n-tile, K split); the splits of one output tile are adjacent
    const int S = p.splits, NTr = (p.E + 255) / 256, KB = p.d / 64;
    const int sp = t % S, rest = t / S;
    const int nt = rest % NTr, mt = rest / NTr;
    tl.el = sp;  // the split index rides in the expert slot
    tl.m0 = mt * 128;
    tl.nt = nt;
    tl.n0 = nt * p.router_bn;
    tl.kb0 = sp * KB / S;
    tl.nk = (sp + 1) * KB / S - tl.kb0;
    return tl;
  }
  if constexpr (KIND == G_ROUTER_WGRAD) {
    // tile = (128 rows of d, 256 experts); K = all tokens in 64-row blocks
    const int NTe = (p.E + 255) / 256;
    const int mt = t / NTe, nt = t - mt * NTe;
    tl.m = 0;
    tl.shift = 0;
    tl.el = 0;
    tl.m0 = mt * 128;
    tl.nt = nt;
    tl.n0 = nt * 256;
    tl.kb0 = 0;
    tl.nk = 2 * router_wgrad_kblocks(p);  // the hi terms of dl, then the lo terms
    return tl;
  }
  const int NT = ntiles_n<KIND>(p);
  if constexpr (KIND <= G_DGRAD_GATEUP) {
    // Tiles of segment s are [NT*(poff[s]-poff[0])/128, NT*(poff[s+1]-poff[0])/128),
    // n-tile major so that the m-tiles of a hot expert sharing one weight tile run back to back.
    const int base = __ldg(p.poff);
    const int seg = segment_of_row(p.poff, p.nseg, base + (t / NT) * 128);
    const int p0 = __ldg(p.poff + seg), p1 = __ldg(p.poff + seg + 1);
    const int mte = (p1 - p0) / 128;
    const int local = t - NT * ((p0 - base) / 128);
    const int nt = local / mte, mi = local - nt * mte;
    const int el = seg % p.El;
    tl.m = seg / p.El;
    tl.shift = p.ring_shift ? __ldg(p.ring_shift + tl.m) : 0;
    tl.el = el;
    tl.m0 = p0 + mi * 128;
    tl.nt = nt;
    tl.n0 = nt * (KIND == G_GATEUP ? 128 : 256);
    tl.kb0 = 0;
    tl.nk = (KIND == G_GATEUP || KIND == G_DGRAD_DOWN) ? p.d / 64 : (KIND == G_DOWN ? p.I / 64 : 2 * p.I / 64);
  } else {
    // contraction over the expert's rows in every macrobatch of the chunk, in order
    const int tpe = mtiles_w<KIND>(p) * NT;
    const int el = t / tpe, local = t - el * tpe;
    const int mt = local / NT, nt = local - mt * NT;
    const int m_lo = p.chunk ? __ldg(p.chunk) : 0;
    const int m_hi = p.chunk ? __ldg(p.chunk + 1) : p.nseg / p.El;
    int nk = 0;
    for (int m = m_lo; m < m_hi; ++m) nk += wgrad_kblocks(p, m, el);
    tl.m = m_lo;
    tl.shift = m_hi;
    tl.el = el;
    tl.m0 = mt * 128;
    tl.nt = nt;
    tl.n0 = nt * 256;
    tl.kb0 = 0;
    tl.nk = nk;
  }
  return tl;
}

// Issue the TMA loads of K block kb of tile tl into one stage.
template <int KIND>
__device__ __forceinline__ void load_stage(const GemmParams& p, const Tile& tl, int kb, uint8_t* sA, uint8_t* sB,
                                           uint64_t* bar, uint64_t pol_act, uint64_t pol_w) {
  const int k0 = kb * 64;
  if constexpr (KIND == G_GATEUP) {
    tma_load_2d(sA, &p.ta0, bar, k0, tl.m0 + tl.shift, pol_act);  // X_perm [rows, d] (K-major), maybe a ring
    const int krow = tl.el * p.d + k0;                 // W_gate / W_up as [El*d, I] (N contiguous)
    tma_load_2d(sB, &p.tb0, bar, tl.n0, krow, pol_w);
    tma_load_2d(sB + 8192, &p.tb0, bar, tl.n0 + 64, krow, pol_w);
    tma_load_2d(sB + 16384, &p.tb1, bar, tl.n0, krow, pol_w);
    tma_load_2d(sB + 24576, &p.tb1, bar, tl.n0 + 64, krow, pol_w);
  } else if constexpr (KIND == G_DOWN) {
    tma_load_2d(sA, &p.ta0, bar, k0, tl.m0, pol_act);  // H [rows, I]
    const int krow = tl.el * p.I + k0;                 // W_down as [El*I, d]
#pragma unroll
    for (int j = 0; j < 4; ++j) tma_load_2d(sB + j * 8192, &p.tb0, bar, tl.n0 + 64 * j, krow, pol_w);
  } else if constexpr (KIND == G_DGRAD_DOWN) {
    tma_load_2d(sA, &p.ta0, bar, k0, tl.m0, pol_act);                  // dY_perm [rows, d]
    tma_load_2d(sB, &p.tb0, bar, k0, tl.el * p.I + tl.n0, pol_w);      // W_down rows = n (I), cols = k (d)
  } else if constexpr (KIND == G_DGRAD_GATEUP) {
    if (k0 < p.I) {
      tma_load_2d(sA, &p.ta0, bar, k0, tl.m0, pol_act);                // dA [rows, I]
      tma_load_2d(sB, &p.tb0, bar, k0, tl.el * p.d + tl.n0, pol_w);    // W_gate rows = n (d), cols = k (I)
    } else {
      tma_load_2d(sA, &p.ta1, bar, k0 - p.I, tl.m0, pol_act);          // dB
      tma_load_2d(sB, &p.tb1, bar, k0 - p.I, tl.el * p.d + tl.n0, pol_w);  // W_up
    }
  } else if constexpr (KIND == G_ROUTER) {
    const int kx = (tl.kb0 + kb) * 64;
    tma_load_2d(sA, &p.ta0, bar, kx, tl.m0, pol_act);  // X [T, d], rows >= T read as zero
    tma_load_2d(sB, &p.tb0, bar, kx, tl.n0, pol_act);  // W_r^T [E, d], rows >= E read as zero
  } else if constexpr (KIND == G_ROUTER_WGRAD) {
    // X [T, d] (or the listed tokens' rows) and DL [2 * Tpad, E64] (hi rows from 0, lo rows
    // from Tpad) with the contraction over tokens: both MN-major (d and E contiguous); the
    // first `half` K blocks take the hi rows, the rest the lo rows, each paired with the same
    // X block; tokens >= T read as zero, experts >= E64 too
    const int half = router_wgrad_kblocks(p);
    const bool lo = kb >= half;
    const int kx = (lo ? kb - half : kb) * 64;
    const int krow = lo ? (p.T + 63) / 64 * 64 + kx : kx;
    tma_load_2d(sA, &p.ta0, bar, tl.m0, kx, pol_act);
    tma_load_2d(sA + 8192, &p.ta0, bar, tl.m0 + 64, kx, pol_act);
#pragma unroll
    for (int j = 0; j < 4; ++j) tma_load_2d(sB + j * 8192, &p.tb0, bar, tl.n0 + 64 * j, krow, pol_act);
  }
}

// wgrad: the 64-row K block starting at padded row `row`; X_perm rows live at row + xshift
// (a ring position in the streamed backward).  Contraction over rows, so both operands
// are MN-major: M = d (or I) and N = I (or d) are the contiguous dimensions.
template <int KIND>
__device__ __forceinline__ void load_wgrad(const GemmParams& p, const Tile& tl, int row, int xshift, uint8_t* sA,
                                           uint8_t* sB, uint64_t* bar, uint64_t pol) {
  if constexpr (KIND == G_WGRAD_GATEUP) {
    tma_load_2d(sA, &p.ta0, bar, tl.m0, row + xshift, pol);            // X_perm
    tma_load_2d(sA + 8192, &p.ta0, bar, tl.m0 + 64, row + xshift, pol);
    const int NTg = p.I / 256;
    const CUtensorMap* mb = tl.nt < NTg ? &p.tb0 : &p.tb1;             // dA for gate, dB for up
    const int nb = (tl.nt < NTg ? tl.nt : tl.nt - NTg) * 256;
#pragma unroll
    for (int j = 0; j < 4; ++j) tma_load_2d(sB + j * 8192, mb, bar, nb + 64 * j, row, pol);
  } else {
    tma_load_2d(sA, &p.ta0, bar, tl.m0, row, pol);                     // Hg, M = I
    tma_load_2d(sA + 8192, &p.ta0, bar, tl.m0 + 64, row, pol);
#pragma unroll
    for (int j = 0; j < 4; ++j) tma_load_2d(sB + j * 8192, &p.tb0, bar, tl.n0 + 64 * j, row, pol);  // dY_perm
  }
}

__device__ __forceinline__ float sigmoidf_(float a) { return 1.0f / (1.0f + expf(-a)); }

__device__ __forceinline__ void store_row32(__nv_bfloat16* dst, const float (&v)[32]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 u;
    u.x = pack_bf16(v[8 * q + 0], v[8 * q + 1]);
    u.y = pack_bf16(v[8 * q + 2], v[8 * q + 3]);
    u.z = pack_bf16(v[8 * q + 4], v[8 * q + 5]);
    u.w = pack_bf16(v[8 * q + 6], v[8 * q + 7]);
    d4[q] = u;
  }
}
__device__ __forceinline__ void load_row32(const __nv_bfloat16* src, float (&v)[32]) {
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

// Epilogue for one output row (this thread's TMEM lane) of tile tl.  Rows past a segment's
// live pad rows (row_asg == ROW_DEAD) store nothing: no later kernel reads them, so their
// operand rows may hold anything.  Live pad rows come from zero operand rows and store zeros.
template <int KIND>
__device__ __forceinline__ void epilogue_row(const GemmParams& p, const Tile& tl, int row, uint32_t taddr) {
  if constexpr (KIND == G_GATEUP) {
    const size_t R = static_cast<size_t>(tl.m0 + row);
    const bool live = __ldg(p.row_asg + R) != ROW_DEAD;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      float a[32], b[32], h[32];
      tmem_ld32(taddr + c * 32, a);        // gate columns
      tmem_ld32(taddr + 128 + c * 32, b);  // up columns
#pragma unroll
      for (int i = 0; i < 32; ++i) h[i] = a[i] * sigmoidf_(a[i]) * b[i];  // SwiGLU
      if (live) {
        const size_t off = R * p.I + tl.n0 + c * 32;
        store_row32(p.out0 + off, a);
        store_row32(p.out1 + off, b);
        store_row32(p.out2 + off, h);
      }
    }
  } else if constexpr (KIND == G_DOWN) {
    const size_t R = static_cast<size_t>(tl.m0 + row);
    const bool live = __ldg(p.row_asg + R) != ROW_DEAD;
    const float g = p.row_gate[R];  // combine weight
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      float o[32];
      tmem_ld32(taddr + c * 32, o);
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] *= g;
      if (live) store_row32(p.out0 + R * p.d + tl.n0 + c * 32, o);
    }
  } else if constexpr (KIND == G_DGRAD_DOWN) {
    // dH' = dY W_down^T arrives in TMEM.  With H = silu(A) B rebuilt from the saved A, B:
    //   dg partial = sum_i dH'_i H_i          (router-gate gradient, "SonicMoE-style")
    //   dH = g dH',  dA = dH B silu'(A),  dB = dH silu(A),  Hg = g H (wgrad operand)
    const size_t R = static_cast<size_t>(tl.m0 + row);
    const bool live = __ldg(p.row_asg + R) != ROW_DEAD;
    const float g = p.row_gate[R];
    float dg = 0.f;
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      float dh[32], a[32], b[32];
      tmem_ld32(taddr + c * 32, dh);
      const size_t off = R * p.I + tl.n0 + c * 32;
      if (live) {
        load_row32(p.in0 + off, a);
        load_row32(p.in1 + off, b);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) a[i] = b[i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float s = sigmoidf_(a[i]);
        const float sl = a[i] * s;
        const float hh = sl * b[i];
        dg = fmaf(dh[i], hh, dg);
        const float dhg = g * dh[i];
        const float da = dhg * b[i] * (s * (1.0f + a[i] * (1.0f - s)));
        const float db = dhg * sl;
        a[i] = da;
        b[i] = db;
        dh[i] = g * hh;
      }
      if (live) {
        store_row32(p.out0 + off, a);   // dA
        store_row32(p.out1 + off, b);   // dB
        store_row32(p.out2 + off, dh);  // Hg
      }
    }
    if (live) p.outf[R * (p.I / 256) + tl.nt] = dg;
  } else if constexpr (KIND == G_DGRAD_GATEUP) {
    const size_t R = static_cast<size_t>(tl.m0 + row);
    const bool live = __ldg(p.row_asg + R) != ROW_DEAD;
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      float v[32];
      tmem_ld32(taddr + c * 32, v);
      if (live) store_row32(p.out0 + R * p.d + tl.n0 + c * 32, v);
    }
  } else if constexpr (KIND == G_ROUTER_WGRAD) {
    // dW_r row (of d) tl.m0 + row, fp32; columns >= E are dropped; no listed token: zero
    float* dst = p.outf + static_cast<size_t>(tl.m0 + row) * p.E;
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      float v[32];
      if (tl.nk > 0) {
        tmem_ld32(taddr + c * 32, v);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      }
      const int e0 = tl.n0 + c * 32;
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (e0 + i < p.E) dst[e0 + i] = v[i];
    }
  } else if constexpr (KIND == G_ROUTER) {
    // fp32 partial logits of K split tl.el; rows >= T and columns >= E are dropped
    const int t = tl.m0 + row;
    float* dst = p.outf + (static_cast<size_t>(tl.el) * p.T + t) * p.E;
#pragma unroll 1
    for (int c = 0; c < p.router_bn / 32 + (p.router_bn % 32 != 0); ++c) {
      float v[32];
      tmem_ld32(taddr + c * 32, v);  // every lane loads (warp-collective), then masks
      const int e0 = tl.n0 + c * 32;
      if (t < p.T) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (c * 32 + i < p.router_bn && e0 + i < p.E) dst[e0 + i] = v[i];  // this tile's columns only
      }
    }
  }
}

// wgrad epilogue: the warp's 32 x 256 slice of the output tile.  Mode (from the chunk
// descriptor of a ring-streamed backward; 0 otherwise):
//   0  dW (the whole contraction was in this launch): bf16, or fp32 when p.wout32
//   1  fp32 partial into the accumulator (first of several chunks)
//   2  fp32: accumulator + this chunk's partial, back into the accumulator
// All go through a 128B-swizzled staging buffer and out by TMA stores.
// Chunks run in a fixed order, so the sum is reproducible.
__device__ __forceinline__ void stage_chunk16(uint8_t* box, int lane, int chunk, uint4 u) {
  *reinterpret_cast<uint4*>(box + lane * 128 + ((chunk ^ (lane & 7)) << 4)) = u;
}

template <int KIND>
__device__ __forceinline__ void epilogue_wgrad(const GemmParams& p, const Tile& tl, int quarter, int lane,
                                               uint32_t taddr, uint8_t* stage_out) {
  int x0, y0, yacc = 0, up = 0;
  if constexpr (KIND == G_WGRAD_GATEUP) {
    const int NTg = p.I / 256;
    up = tl.nt < NTg ? 0 : 1;  // dW_gate or dW_up as [El*d, I]
    x0 = (tl.nt - up * NTg) * 256;
    y0 = tl.el * p.d + tl.m0 + quarter * 32;
    yacc = (up * p.El + tl.el) * p.d + tl.m0 + quarter * 32;  // accumulator as [2*El*d, I] fp32
  } else {
    x0 = tl.n0;  // dW_down as [El*I, d]
    y0 = tl.el * p.I + tl.m0 + quarter * 32;
  }
  const int mode = (KIND == G_WGRAD_GATEUP && p.chunk) ? __ldg(p.chunk + 3) : 0;
  // The warp's 16 KB staging slice holds four boxes.  Each box is staged, stored and committed
  // as its own bulk group, and a box slot is refilled once the store issued from it one tile
  // (bf16) or half a tile (fp32) earlier has been read: all but the 3 newest groups.  So the
  // TMA engine drains box b while the warp converts box b+1.  (Stores of two or four adjacent
  // boxes at once, through a 3-D map, measured slower: fewer stores, less overlap.)
  if (mode == 0 && !p.wout32) {
    // TMEM loads pipelined one box ahead: box b+1's load is in flight while box b is converted
    uint32_t r[2][64];
    const bool any = tl.nk > 0;  // an expert without tokens has a zero gradient
    if (any) {
      tmem_ld64_issue(taddr, r[0]);
      tmem_ld64_wait(r[0]);
    } else {
#pragma unroll
      for (int i = 0; i < 64; ++i) r[0][i] = r[1][i] = 0u;
    }
#pragma unroll
    for (int b = 0; b < 4; ++b) {  // 64 bf16 columns per box
      if (any && b < 3) tmem_ld64_issue(taddr + (b + 1) * 64, r[(b + 1) & 1]);
      const uint32_t (&w)[64] = r[b & 1];
      if (lane == 0) bulk_wait_read<3>();
      __syncwarp();
      uint8_t* box = stage_out + b * 4096;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        uint4 u;
        u.x = pack_bf16(__uint_as_float(w[8 * q + 0]), __uint_as_float(w[8 * q + 1]));
        u.y = pack_bf16(__uint_as_float(w[8 * q + 2]), __uint_as_float(w[8 * q + 3]));
        u.z = pack_bf16(__uint_as_float(w[8 * q + 4]), __uint_as_float(w[8 * q + 5]));
        u.w = pack_bf16(__uint_as_float(w[8 * q + 6]), __uint_as_float(w[8 * q + 7]));
        stage_chunk16(box, lane, q, u);
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(up ? &p.to1 : &p.to0, box, x0 + b * 64, y0);
        bulk_commit();
      }
      if (any && b < 3) tmem_ld64_wait(r[(b + 1) & 1]);
    }
    return;
  }
  // fp32: eight 32 x 32 boxes, into the accumulator (modes 1, 2) or the output (mode 0)
  const CUtensorMap* tm = mode == 0 ? (up ? &p.to1 : &p.to0) : &p.tacc;
  const int ys = mode == 0 ? y0 : yacc;
  const float* prev = mode == 2 ? p.acc32 + static_cast<size_t>(yacc + lane) * p.I + x0 : nullptr;
#pragma unroll 1
  for (int j = 0; j < 8; ++j) {
    const int col = j * 32;
    float v[32];
    if (tl.nk > 0) {
      tmem_ld32(taddr + col, v);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = 0.f;
    }
    if (mode == 2) {
      const float4* pv = reinterpret_cast<const float4*>(prev + col);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 o = pv[q];
        v[4 * q + 0] = o.x + v[4 * q + 0];
        v[4 * q + 1] = o.y + v[4 * q + 1];
        v[4 * q + 2] = o.z + v[4 * q + 2];
        v[4 * q + 3] = o.w + v[4 * q + 3];
      }
    }
    if (lane == 0) bulk_wait_read<3>();
    __syncwarp();
    uint8_t* box = stage_out + (j & 3) * 4096;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      uint4 u;
      u.x = __float_as_uint(v[4 * q + 0]);
      u.y = __float_as_uint(v[4 * q + 1]);
      u.z = __float_as_uint(v[4 * q + 2]);
      u.w = __float_as_uint(v[4 * q + 3]);
      stage_chunk16(box, lane, q, u);
    }
    fence_proxy_async();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tm, box, x0 + col, ys);
      bulk_commit();
    }
  }
}

// Wait bounded by time only (used while draining after an error).
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > MOE_SPIN_CYCLES) return;
  }
}

// The next tile of this CTA from the scheduler's ring (the producer and the MMA issuer: one
// thread each).  Returns false on a device error; the tile with t = -1 ends the loop.
__device__ __forceinline__ bool next_tile(const Tile* ring, uint64_t* sfull, uint64_t* sempty, int j, Tile& tl,
                                          int* status) {
  const int slot = j % SCHED_DEPTH;
  if (!mbar_wait(&sfull[slot], (j / SCHED_DEPTH) & 1, status)) return false;
  tl = ring[slot];
  mbar_arrive(&sempty[slot]);
  return true;
}
// The j-th tile of this CTA: from the scheduler's ring, or decoded here for kinds without it.
template <int KIND, bool SCHED>
__device__ __forceinline__ bool role_tile(const GemmParams& p, const Tile* ring, uint64_t* sfull, uint64_t* sempty,
                                          int j, int ntiles, Tile& tl) {
  if constexpr (SCHED) {
    return next_tile(ring, sfull, sempty, j, tl, p.status);
  } else {
    const int t = blockIdx.x + j * gridDim.x;
    if (t < ntiles) tl = decode<KIND>(p, t);
    else tl.t = -1;
    return true;
  }
}

template <int KIND, bool SCHED>
__global__ void __launch_bounds__(SCHED ? GEMM_THREADS_SCHED : GEMM_THREADS, 1)
    k_moe_gemm(const __grid_constant__ GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int STAGES = stages_of<KIND>();
  uint8_t* stage_out = smem + STAGES * GEMM_STAGE_BYTES;  // wgrad only: 4 x 16 KB
  uint64_t* full = reinterpret_cast<uint64_t*>(stage_out + (is_wgrad<KIND>() ? GEMM_STAGE_OUT_BYTES : 0));
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* sfull = drain + 1;  // scheduler ring: entry written / entry read by every role
  uint64_t* sempty = sfull + SCHED_DEPTH;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sempty + SCHED_DEPTH);
  Tile* ring = reinterpret_cast<Tile*>(sempty + SCHED_DEPTH + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    for (int s = 0; s < SCHED_DEPTH; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], 6);  // producer, MMA issuer, four epilogue warps
    }
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
  constexpr uint32_t IDESC = idesc_bf16(GEMM_BM, GEMM_BN, Traits<KIND>::A_MN, Traits<KIND>::B_MN);
  const int ntiles = SCHED ? 0 : num_tiles<KIND>(p);

  if (warp == 6) {
    if (SCHED && lane == 0) {
      // ---------------- scheduler: this CTA's tiles, decoded ahead of the roles ----------------
      const int nt_all = num_tiles<KIND>(p);
      for (int t = blockIdx.x, j = 0;; t += gridDim.x, ++j) {
        const int slot = j % SCHED_DEPTH;
        if (!mbar_wait(&sempty[slot], ((j / SCHED_DEPTH) & 1) ^ 1, p.status)) break;
        if (t < nt_all) {
          ring[slot] = decode<KIND>(p, t);
        } else {
          ring[slot].t = -1;
        }
        mbar_arrive(&sfull[slot]);
        if (t >= nt_all) break;
      }
    }
  } else if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      const uint64_t pol_act = policy_evict_last();
      const uint64_t pol_w = policy_evict_first();
      int stage = 0;
      uint32_t phase = 0;
      int last_parity[STAGES];
      for (int s = 0; s < STAGES; ++s) last_parity[s] = -1;
      bool ok = true;
      for (int j = 0; ok; ++j) {
        Tile tl;
        if (!role_tile<KIND, SCHED>(p, ring, sfull, sempty, j, ntiles, tl)) { ok = false; break; }
        if (tl.t < 0) break;
        if constexpr (is_wgrad<KIND>()) {
          // K runs over the expert's rows in each macrobatch of the chunk, in order
          for (int m = tl.m; m < tl.shift && ok; ++m) {
            const int sg = m * p.El + tl.el;
            const int r0 = __ldg(p.poff + sg), r1 = r0 + 64 * wgrad_kblocks(p, m, tl.el);
            const int xs = (KIND == G_WGRAD_GATEUP && p.ring_shift) ? __ldg(p.ring_shift + m) : 0;
            for (int row = r0; row < r1; row += 64) {
              if (!mbar_wait(&empty[stage], phase ^ 1, p.status)) { ok = false; break; }
              uint8_t* sA = smem + stage * GEMM_STAGE_BYTES;
              mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>(GEMM_STAGE_BYTES));
              load_wgrad<KIND>(p, tl, row, xs, sA, sA + GEMM_A_BYTES, &full[stage], pol_act);
              last_parity[stage] = static_cast<int>(phase);
              if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
          }
        } else {
          for (int kb = 0; kb < tl.nk; ++kb) {
            if (!mbar_wait(&empty[stage], phase ^ 1, p.status)) { ok = false; break; }
            uint8_t* sA = smem + stage * GEMM_STAGE_BYTES;
            uint8_t* sB = sA + GEMM_A_BYTES;
            mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>(GEMM_STAGE_BYTES));
            load_stage<KIND>(p, tl, kb, sA, sB, &full[stage], pol_act, pol_w);
            last_parity[stage] = static_cast<int>(phase);
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
          }
        }
      }
      if (!ok) {  // let copies already in flight land before the CTA's smem goes away
        for (int s = 0; s < STAGES; ++s)
          if (last_parity[s] >= 0) mbar_wait_drain(&full[s], static_cast<uint32_t>(last_parity[s]));
      }
    }
  } else if (warp == 1 && is_wgrad<KIND>()) {
    if (lane == 0) {
      // ---------------- MMA issuer, weight gradients: walks the segments of the tile's expert so
      // that a segment's last block issues only the K16 steps that hold real rows ----------------
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int it = 0; ok; ++it) {
        Tile tl;
        if (!role_tile<KIND, SCHED>(p, ring, sfull, sempty, it, ntiles, tl)) { ok = false; break; }
        if (tl.t < 0) break;
        const int acc = it & 1;
        const uint32_t accp = (it >> 1) & 1;
        if (!mbar_wait(&tempty[acc], accp ^ 1, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dtm = tbase + acc * GEMM_BN;
        int kb = 0;
        for (int m = tl.m; m < tl.shift && ok; ++m) {
          const int rows = seg_rows(p, m, tl.el);
          for (int r = 0; r < rows; r += 64, ++kb) {
            if (!mbar_wait(&full[stage], phase, p.status)) { ok = false; break; }
            tc_fence_after();
            const uint32_t a0 = smem_u32(smem + stage * GEMM_STAGE_BYTES);
            const uint32_t b0 = a0 + static_cast<uint32_t>(GEMM_A_BYTES);
            const int valid = rows - r < 64 ? rows - r : 64;
            for (int kk = 0; kk * 16 < valid; ++kk)
              umma_bf16(dtm, sdesc_sw128(a0 + kk * 2048, 8192, 1024), sdesc_sw128(b0 + kk * 2048, 8192, 1024), IDESC,
                        (kb | kk) != 0 ? 1u : 0u);
            umma_commit(&empty[stage]);  // frees the stage once these MMAs have read it
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
          }
        }
        if (!ok) break;
        if (kb > 0) umma_commit(&tfull[acc]);
        else mbar_arrive(&tfull[acc]);
      }
      umma_commit(drain);  // all MMAs issued by this thread are complete once this lands
      mbar_wait_drain(drain, 0);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int it = 0; ok; ++it) {
        Tile tl;
        if (!role_tile<KIND, SCHED>(p, ring, sfull, sempty, it, ntiles, tl)) { ok = false; break; }
        if (tl.t < 0) break;
        const int acc = it & 1;
        const uint32_t accp = (it >> 1) & 1;
        if (!mbar_wait(&tempty[acc], accp ^ 1, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dtm = tbase + acc * GEMM_BN;
        for (int kb = 0; kb < tl.nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * GEMM_STAGE_BYTES);
          const uint32_t b0 = a0 + static_cast<uint32_t>(GEMM_A_BYTES);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // 4 x K16 per 64-wide block
            const uint64_t ad = Traits<KIND>::A_MN ? sdesc_sw128(a0 + kk * 2048, 8192, 1024)
                                                   : sdesc_sw128(a0 + kk * 32, 16, 1024);
            const uint64_t bd = Traits<KIND>::B_MN ? sdesc_sw128(b0 + kk * 2048, 8192, 1024)
                                                   : sdesc_sw128(b0 + kk * 32, 16, 1024);
            umma_bf16(dtm, ad, bd, KIND == G_ROUTER ? idesc_bf16(GEMM_BM, p.router_bn, false, false) : IDESC,
                      (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[stage]);  // frees the stage once these MMAs have read it
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if (tl.nk > 0) umma_commit(&tfull[acc]);
        else mbar_arrive(&tfull[acc]);
      }
      umma_commit(drain);  // all MMAs issued by this thread are complete once this lands
      mbar_wait_drain(drain, 0);
    }
  } else if (warp >= 2 && warp <= 5) {
    // ---------------- epilogue warps 2..5 ----------------
    const int quarter = warp & 3;  // TMEM lanes this warp may access: 32*quarter ..
    const int row = quarter * 32 + lane;
    for (int it = 0;; ++it) {
      int ok = 1;
      Tile tl;
      if constexpr (SCHED) {
        const int slot = it % SCHED_DEPTH;
        if (lane == 0) ok = mbar_wait(&sfull[slot], (it / SCHED_DEPTH) & 1, p.status) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        __syncwarp();  // lane 0's acquire of the entry, then every lane reads it
        tl = ring[slot];
        __syncwarp();  // every lane has read the entry before lane 0 releases it
        if (lane == 0) mbar_arrive(&sempty[slot]);
      } else {
        const int t = blockIdx.x + it * gridDim.x;
        if (t >= ntiles) break;
        tl = decode<KIND>(p, t);
      }
      if (tl.t < 0) break;
      const int acc = it & 1;
      const uint32_t accp = (it >> 1) & 1;
      if (lane == 0) ok = mbar_wait(&tfull[acc], accp, p.status) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      __syncwarp();
      tc_fence_after();
      const uint32_t taddr = tbase + (static_cast<uint32_t>(quarter * 32) << 16) + acc * GEMM_BN;
      if constexpr (is_wgrad<KIND>())
        epilogue_wgrad<KIND>(p, tl, quarter, lane, taddr, stage_out + (warp - 2) * (GEMM_STAGE_OUT_BYTES / 4));
      else
        epilogue_row<KIND>(p, tl, row, taddr);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
    if constexpr (is_wgrad<KIND>()) {
      if (lane == 0) bulk_wait0();  // stores complete before the CTA (and its smem) goes away
      __syncwarp();
    }
  }
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

template <int KIND, bool SCHED>
static cudaError_t configure_kind() {
  static bool configured[64] = {};  // the attribute is set once per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(k_moe_gemm<KIND, SCHED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem_bytes<KIND>()));
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  return cudaSuccess;
}

template <int KIND, bool SCHED = false>
static cudaError_t launch_kind(const GemmParams& p, int grid, cudaStream_t st) {
  const cudaError_t e = configure_kind<KIND, SCHED>();
  if (e != cudaSuccess) return e;
  k_moe_gemm<KIND, SCHED><<<grid, SCHED ? GEMM_THREADS_SCHED : GEMM_THREADS, smem_bytes<KIND>(), st>>>(p);
  return cudaGetLastError();
}

template <int KIND>
static cudaError_t preload_kind() {
  cudaFuncAttributes a;
  const cudaError_t e = cudaFuncGetAttributes(&a, k_moe_gemm<KIND, false>);  // loads the kernel's module
  return e != cudaSuccess ? e : configure_kind<KIND, false>();
}

cudaError_t preload_gemm(GemmKind kind) {
  switch (kind) {
    case G_GATEUP: return preload_kind<G_GATEUP>();
    case G_DOWN: return preload_kind<G_DOWN>();
    case G_DGRAD_DOWN: return preload_kind<G_DGRAD_DOWN>();
    case G_DGRAD_GATEUP: return preload_kind<G_DGRAD_GATEUP>();
    case G_WGRAD_GATEUP: return preload_kind<G_WGRAD_GATEUP>();
    case G_WGRAD_DOWN: return preload_kind<G_WGRAD_DOWN>();
    case G_ROUTER: return preload_kind<G_ROUTER>();
    case G_ROUTER_WGRAD: return preload_kind<G_ROUTER_WGRAD>();
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_gemm(GemmKind kind, const GemmParams& p, int grid, cudaStream_t st, bool sched) {
  switch (kind) {
    case G_GATEUP: return launch_kind<G_GATEUP>(p, grid, st);
    case G_DOWN: return launch_kind<G_DOWN>(p, grid, st);
    case G_DGRAD_DOWN: return launch_kind<G_DGRAD_DOWN>(p, grid, st);
    case G_DGRAD_GATEUP: return launch_kind<G_DGRAD_GATEUP>(p, grid, st);
    case G_WGRAD_GATEUP:
      return sched ? launch_kind<G_WGRAD_GATEUP, true>(p, grid, st) : launch_kind<G_WGRAD_GATEUP>(p, grid, st);
    case G_WGRAD_DOWN:
      return sched ? launch_kind<G_WGRAD_DOWN, true>(p, grid, st) : launch_kind<G_WGRAD_DOWN>(p, grid, st);
    case G_ROUTER: return launch_kind<G_ROUTER>(p, grid, st);
    case G_ROUTER_WGRAD: return launch_kind<G_ROUTER_WGRAD>(p, grid, st);
  }
  return cudaErrorInvalidValue;
}

// ===========================================================================
// Two dependent grouped GEMMs in one persistent launch
// ===========================================================================
// The forward's gate/up and down GEMMs, or the backward's dgrad of W_down and dgrad of
// gate/up: the second GEMM of the pair reads, for its 128 rows, what every tile of the first
// GEMM wrote for those rows (H; or dA and dB).  Work units, in ticket order: every tile of the
// first GEMM, then every tile of the second.  A CTA takes a ticket
// when it starts and one for each further unit it claims.  While the grid still has CTAs that
// have not started, a claim is the cancellation of one of them through Cluster Launch Control
// (its work moves to the running CTA); once the hardware reports none left, claims come from
// the ticket counter alone, until the tickets run past the last unit.  So the work spreads
// over the CTAs that actually run, whatever the grid size, and second-GEMM tiles fill the SMs
// that the last round of first-GEMM tiles leaves idle.  A second-GEMM tile waits (bounded)
// until every first-GEMM tile of its 128 rows has stored its rows.  Tickets are handed out in
// one global order and a second-GEMM tile only waits for first-GEMM tiles, which have lower
// tickets and are held by running (or finished) CTAs, so the waits end.  Every wait gives up
// once the status word is set.
//
// A unit computes exactly what the separate GEMM launches compute (the same decode, loads and
// epilogue functions), so the results are the same bits.
//
// Measured and kept out: dispatch and combine as units of this kernel, run by its four
// epilogue warps.  With one CTA per SM those warps keep too few loads in flight for a copy:
// traced per unit, the combine ran 12x and the dispatch 2x slower than their own kernels, and
// gate/up tiles stalled behind the dispatch.
enum PairUnit { FU_FIRST = 1, FU_SECOND = 2 };

// ctl: [0] ticket counter, [1, 1 + cap) first-GEMM epilogue warps done per m-tile.
struct PairCounts {
  int mt, n1, n2;
  __device__ int total() const { return n1 + n2; }
};
template <int K1, int K2>
__device__ __forceinline__ PairCounts pair_counts(const GemmPairParams& P) {
  PairCounts c;
  c.mt = (__ldg(P.p1.poff + P.p1.nseg) - __ldg(P.p1.poff)) / 128;
  c.n1 = c.mt * ntiles_n<K1>(P.p1);
  c.n2 = c.mt * ntiles_n<K2>(P.p2);
  return c;
}
template <int K1, int K2>
__device__ __forceinline__ Tile pair_decode(const GemmPairParams& P, const PairCounts& c, int t) {
  Tile tl;
  if (t < c.n1) {
    tl = decode<K1>(P.p1, t);
    tl.u = FU_FIRST;
    return tl;
  }
  t -= c.n1;
  if (t < c.n2) {
    tl = decode<K2>(P.p2, t);
    tl.u = FU_SECOND;
    return tl;
  }
  tl.t = -1;
  return tl;
}

// Bounded wait (one thread) until *p >= target, written by other CTAs with release order.
__device__ __noinline__ bool wait_count(const int* p, int target, int* status) {
  if (ld_acquire_gpu(p) >= target) return true;
  const long long t0 = clock64();
  for (uint32_t n = 1;; ++n) {
    __nanosleep(64);
    if (ld_acquire_gpu(p) >= target) return true;
    if ((n & 31u) == 0) {
      if (status_set(status)) return false;
      if (clock64() - t0 > MOE_SPIN_CYCLES) {
        raise_status(status, MOE_ERR_DEVICE_TIMEOUT);
        return false;
      }
    }
  }
}
// One warp's global stores, then one count: the stores are visible to a CTA that has acquired
// the count (and, after its proxy fence, to that CTA's TMA loads).
__device__ __forceinline__ void warp_release_count(int* p, int lane) {
  __syncwarp();
  if (lane == 0) {
    fence_proxy_async_global();
    __threadfence();
    atomicAdd(p, 1);
  }
}

constexpr size_t FUSED_TAIL_BYTES = 1024;
constexpr size_t fused_smem_bytes() { return GEMM_STAGES * GEMM_STAGE_BYTES + 1024 + FUSED_TAIL_BYTES; }

template <int K1, int K2>
__global__ void __launch_bounds__(GEMM_THREADS_SCHED, 1) k_moe_gemm_pair(const __grid_constant__ GemmPairParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int STAGES = GEMM_STAGES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * GEMM_STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* sfull = drain + 1;
  uint64_t* sempty = sfull + SCHED_DEPTH;
  uint64_t* staken = sempty + SCHED_DEPTH;  // the producer has read ring entry j
  uint64_t* clc_bar = staken + SCHED_DEPTH;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(clc_bar + 1);
  uint4* clc_resp = reinterpret_cast<uint4*>((reinterpret_cast<uintptr_t>(clc_bar + 2) + 15) & ~uintptr_t(15));
  Tile* ring = reinterpret_cast<Tile*>(clc_resp + 1);
  int* status = P.p1.status;
  int* hcnt = P.ctl + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init(drain, 1);
    for (int s = 0; s < SCHED_DEPTH; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], 6);  // producer, MMA issuer, four epilogue warps
      mbar_init(&staken[s], 1);
    }
    mbar_init(clc_bar, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&P.p1.ta0);
    prefetch_tmap(&P.p1.ta1);
    prefetch_tmap(&P.p1.tb0);
    prefetch_tmap(&P.p1.tb1);
    prefetch_tmap(&P.p2.ta0);
    prefetch_tmap(&P.p2.ta1);
    prefetch_tmap(&P.p2.tb0);
    prefetch_tmap(&P.p2.tb1);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  static_assert(Traits<K1>::A_MN == Traits<K2>::A_MN && Traits<K1>::B_MN == Traits<K2>::B_MN && !Traits<K1>::A_MN,
                "one instruction descriptor serves both GEMMs of the pair");
  constexpr bool B_MN = Traits<K1>::B_MN;
  constexpr uint32_t IDESC = idesc_bf16(GEMM_BM, GEMM_BN, false, B_MN);

  if (warp == 6) {
    if (lane == 0) {
      // ---------------- scheduler: tickets in, decoded units into the ring ----------------
      const PairCounts cnt = pair_counts<K1, K2>(P);
      const int total = cnt.total();
      uint32_t clc_phase = 0;
      bool may_cancel = true;  // false after an answer that cancelled nothing
      const int skip = P.skip_first ? cnt.n1 : 0;
      int ticket = status_set(status) ? total : skip + atomicAdd(P.ctl, 1);
      for (int j = 0;; ++j) {
        const int slot = j % SCHED_DEPTH;
        // claim the next unit while this one is queued: cancel a CTA that has not started
        bool asked = false;
        if (ticket < total && may_cancel) {
          fence_proxy_async();  // the last answer was read (generic proxy) before the next is written
          mbar_arrive_expect_tx(clc_bar, 16);
          clc_try_cancel(clc_resp, clc_bar);
          asked = true;
        }
        // stay at most two units ahead of the producer, so that unclaimed work stays with CTAs
        // that reach it first (the tail stays balanced)
        bool ok = true;
        if (j >= 2) ok = mbar_wait(&staken[(j - 2) % SCHED_DEPTH], ((j - 2) / SCHED_DEPTH) & 1, status);
        if (ok) ok = mbar_wait(&sempty[slot], ((j / SCHED_DEPTH) & 1) ^ 1, status);
        if (ok) {
          if (ticket < total && !status_set(status)) ring[slot] = pair_decode<K1, K2>(P, cnt, ticket);
          else ring[slot].t = -1;
          mbar_arrive(&sfull[slot]);
        }
        const bool last = !ok || ring[slot].t < 0;
        if (asked) {
          // the answer lands in this CTA's shared memory: wait for it (bounded by time only,
          // also after an error) before the CTA can end
          mbar_wait_drain(clc_bar, clc_phase);
          if (!mbar_try_wait(clc_bar, clc_phase)) {
            raise_status(status, MOE_ERR_DEVICE_TIMEOUT);
            break;
          }
          clc_phase ^= 1;
          if (!clc_cancelled(clc_resp)) may_cancel = false;  // no CTA left to take over
        }
        if (last) break;
        ticket = skip + atomicAdd(P.ctl, 1);
      }
      // Out of units: cancel the CTAs that have not started yet, so that they never launch
      // only to find no work.  This overlaps with the last units of this CTA's roles.
      while (may_cancel && !status_set(status)) {
        fence_proxy_async();
        mbar_arrive_expect_tx(clc_bar, 16);
        clc_try_cancel(clc_resp, clc_bar);
        mbar_wait_drain(clc_bar, clc_phase);
        if (!mbar_try_wait(clc_bar, clc_phase)) {
          raise_status(status, MOE_ERR_DEVICE_TIMEOUT);
          break;
        }
        clc_phase ^= 1;
        may_cancel = clc_cancelled(clc_resp);
      }
    }
  } else if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      const uint64_t pol_act = policy_evict_last();
      const uint64_t pol_w = policy_evict_first();
      const int n1_n = ntiles_n<K1>(P.p1);
      const int poff0 = __ldg(P.p1.poff);
      int stage = 0;
      uint32_t phase = 0;
      int last_parity[STAGES];
      for (int s = 0; s < STAGES; ++s) last_parity[s] = -1;
      bool ok = true;
      for (int j = 0; ok; ++j) {
        Tile tl;
        const int slot = j % SCHED_DEPTH;
        if (!mbar_wait(&sfull[slot], (j / SCHED_DEPTH) & 1, status)) break;
        tl = ring[slot];
        mbar_arrive(&sempty[slot]);
        mbar_arrive(&staken[slot]);
        if (tl.t < 0) break;
        if (tl.u == FU_SECOND) {
          // every first-GEMM tile of these 128 rows has stored its rows
          if (!wait_count(hcnt + ((tl.m0 - poff0) >> 7), 4 * n1_n, status)) { ok = false; break; }
          fence_proxy_async_global();
        }
        for (int kb = 0; kb < tl.nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, status)) { ok = false; break; }
          uint8_t* sA = smem + stage * GEMM_STAGE_BYTES;
          uint8_t* sB = sA + GEMM_A_BYTES;
          mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>(GEMM_STAGE_BYTES));
          if (tl.u == FU_FIRST) load_stage<K1>(P.p1, tl, kb, sA, sB, &full[stage], pol_act, pol_w);
          else load_stage<K2>(P.p2, tl, kb, sA, sB, &full[stage], pol_act, pol_w);
          last_parity[stage] = static_cast<int>(phase);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        for (int s = 0; s < STAGES; ++s)
          if (last_parity[s] >= 0) mbar_wait_drain(&full[s], static_cast<uint32_t>(last_parity[s]));
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer: GEMM units only ----------------
      int stage = 0;
      uint32_t phase = 0;
      int g = 0;  // GEMM units so far: picks the accumulator
      bool ok = true;
      for (int j = 0; ok; ++j) {
        Tile tl;
        if (!next_tile(ring, sfull, sempty, j, tl, status)) break;
        if (tl.t < 0) break;
        const int acc = g & 1;
        const uint32_t accp = (g >> 1) & 1;
        ++g;
        if (!mbar_wait(&tempty[acc], accp ^ 1, status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dtm = tbase + acc * GEMM_BN;
        for (int kb = 0; kb < tl.nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * GEMM_STAGE_BYTES);
          const uint32_t b0 = a0 + static_cast<uint32_t>(GEMM_A_BYTES);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(dtm, sdesc_sw128(a0 + kk * 32, 16, 1024),
                      B_MN ? sdesc_sw128(b0 + kk * 2048, 8192, 1024) : sdesc_sw128(b0 + kk * 32, 16, 1024), IDESC,
                      (kb | kk) != 0 ? 1u : 0u);
          umma_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if (tl.nk > 0) umma_commit(&tfull[acc]);
        else mbar_arrive(&tfull[acc]);
      }
      umma_commit(drain);
      mbar_wait_drain(drain, 0);
    }
  } else if (warp >= 2 && warp <= 5) {
    // ---------------- epilogue warps ----------------
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int poff0 = __ldg(P.p1.poff);
    int g = 0;
    for (int it = 0;; ++it) {
      int ok = 1;
      Tile tl;
      const int slot = it % SCHED_DEPTH;
      if (lane == 0) ok = mbar_wait(&sfull[slot], (it / SCHED_DEPTH) & 1, status) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      __syncwarp();
      tl = ring[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&sempty[slot]);
      if (tl.t < 0) break;
      const int acc = g & 1;
      const uint32_t accp = (g >> 1) & 1;
      ++g;
      if (lane == 0) ok = mbar_wait(&tfull[acc], accp, status) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      __syncwarp();
      tc_fence_after();
      const uint32_t taddr = tbase + (static_cast<uint32_t>(quarter * 32) << 16) + acc * GEMM_BN;
      if (tl.u == FU_FIRST) epilogue_row<K1>(P.p1, tl, row, taddr);
      else epilogue_row<K2>(P.p2, tl, row, taddr);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (tl.u == FU_FIRST) warp_release_count(hcnt + ((tl.m0 - poff0) >> 7), lane);
    }
  }
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

template <int K1, int K2>
static cudaError_t launch_pair(const GemmPairParams& p, int64_t grid, cudaStream_t st) {
  static bool configured[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(k_moe_gemm_pair<K1, K2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(fused_smem_bytes()));
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  if (grid < 1 || grid > 0x7fffffff) return cudaErrorInvalidValue;
  k_moe_gemm_pair<K1, K2><<<static_cast<unsigned>(grid), GEMM_THREADS_SCHED, fused_smem_bytes(), st>>>(p);
  return cudaGetLastError();
}

int64_t gemm_pair_units(GemmPair pair, int64_t RP, int d, int I) {
  const int64_t mt = RP / 128;
  return pair == PAIR_FWD ? mt * (I / 128 + d / 256) : mt * (I / 256 + d / 256);
}

cudaError_t launch_gemm_pair(GemmPair pair, const GemmPairParams& p, int64_t grid, cudaStream_t st) {
  switch (pair) {
    case PAIR_FWD: return launch_pair<G_GATEUP, G_DOWN>(p, grid, st);
    case PAIR_DGRAD: return launch_pair<G_DGRAD_DOWN, G_DGRAD_GATEUP>(p, grid, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace moe
