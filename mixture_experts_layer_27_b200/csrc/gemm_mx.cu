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
//
// The weight-gradient GEMMs contract over an expert's rows: their operands are
// quantised along the rows by their producers (the dispatch, the reverse-combine
// and the dgrad of W_down) and stored K-major in 128-row tiles (rowq_index), so a
// 128-row K stage of either operand is one TMA box; a tile is 128 weight rows x 256
// weight columns of one expert, K the real rows of each of the expert's segments in
// 128-row stages (the last stage of a segment issues only the K = 32 steps that hold
// real rows).  Their epilogue moves the accumulator to registers, releases it at
// once, and writes the gradient through shared memory with TMA box stores.
#include "moe_internal.cuh"
#include "ptx.cuh"

namespace moe {

struct MxTile {
  int el, m0, n0, nt, nk;
};

// Weight-gradient kinds: segment m (of nseg / El) of local expert el: its first padded row and its
// real rows (one segment per expert, or one per macrobatch of a ring-streamed layer).
__device__ __forceinline__ void mx_wseg(const MxParams& p, int m, int el, int& r0, int& rows) {
  const int sg = m * p.El + el;
  r0 = __ldg(p.poff + sg);
  if (!p.cum) {
    rows = __ldg(p.cnt + el);
  } else {
    const int nm = p.nseg / p.El;
    rows = (m + 1 < nm ? __ldg(p.cum + sg + p.El) : __ldg(p.cnt + el)) - __ldg(p.cum + sg);
  }
}

template <int KIND>
__device__ __forceinline__ int mx_ntiles_n(const MxParams& p) {
  if (KIND == MX_GATEUP || KIND == NV_GATEUP) return p.I / (mx_bn(KIND) / 2);  // per tile: [64 gate | 64 up] column pairs
  if (KIND == MX_DGRAD_DOWN || KIND == NV_DGRAD_DOWN) return p.I / mx_bn(KIND);
  if (KIND == MX_WGRAD_GATEUP) return 2 * p.I / 256;  // gate n-tiles, then up n-tiles
  return p.d / mx_bn(KIND);  // MX_DOWN, MX_DGRAD_GATEUP, MX_WGRAD_DOWN
}
// weight-gradient kinds: 128-row tiles of the gradient (rows of d for gate/up, of I for down)
template <int KIND>
__device__ __forceinline__ int mx_mtiles_w(const MxParams& p) {
  return KIND == MX_WGRAD_GATEUP ? p.d / 128 : p.I / 128;
}
template <int KIND>
__device__ __forceinline__ int mx_kblocks(const MxParams& p) {
  if (KIND == NV_GATEUP || KIND == NV_DGRAD_DOWN) return p.d / 256;  // 128-byte K stages of 256 E2M1 codes
  if (KIND == NV_DOWN) return p.I / 256;
  if (KIND == NV_DGRAD_GATEUP) return 2 * p.I / 256;
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
  if constexpr (mx_is_wgrad(KIND)) return p.El * mx_mtiles_w<KIND>(p) * mx_ntiles_n<KIND>(p);
  return ((__ldg(p.poff + p.nseg) - __ldg(p.poff)) / 128) * mx_ntiles_n<KIND>(p);
}

template <int KIND>
__device__ __forceinline__ MxTile mx_decode(const MxParams& p, int t) {
  const int NT = mx_ntiles_n<KIND>(p);
  if constexpr (mx_is_wgrad(KIND)) {
    // per expert, m-tile major and n-tile minor: CTAs that run at the same time write adjacent
    // column blocks of the same gradient rows
    const int tpe = mx_mtiles_w<KIND>(p) * NT;
    const int el = t / tpe, local = t - el * tpe;
    const int mt = local / NT;
    MxTile tl;
    tl.el = el;
    tl.m0 = mt * 128;
    tl.nt = local - mt * NT;
    tl.n0 = tl.nt * 256;
    tl.nk = 0;  // 128-row K blocks over the expert's segments
    for (int m = 0, nm = p.nseg / p.El; m < nm; ++m) {
      int r0, rows;
      mx_wseg(p, m, el, r0, rows);
      tl.nk += (rows + 127) / 128;
    }
    return tl;
  }
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
  tl.n0 = nt * (KIND == MX_GATEUP || KIND == NV_GATEUP ? mx_bn(KIND) / 2 : mx_bn(KIND));  // gate/up: first H column
  tl.nk = mx_kblocks<KIND>(p);
  return tl;
}

// TMA + bulk loads of K block kb (128 elements) of tile tl into one stage; the weight-gradient
// kinds take the block's first padded row (krow) instead.
template <int KIND>
__device__ __forceinline__ void mx_load(const MxParams& p, const MxTile& tl, int kb, int krow, uint8_t* st,
                                        uint64_t* bar, uint64_t pol_act, uint64_t pol_w) {
  uint8_t* sA = st;
  constexpr int BN = mx_bn(KIND);
  uint8_t* sB = st + MX_A_BYTES;
  uint8_t* sSF = sB + BN * 128;  // the A chunk, then a B chunk per 128 rows of the B tile
  const CUtensorMap* ma = &p.ta0;
  const CUtensorMap* mb = &p.tb0;
  const uint8_t* sfa = p.sfa0;
  const uint8_t* sfb = p.sfb0;
  if constexpr (mx_is_nv(KIND)) {
    // NVFP4: 128 bytes of K = 256 codes; per 128 rows the stage's four 64-deep scale chunks are
    // contiguous (2 KB): A's, then those of B's 128-row halves
    int brow, K, kl = kb;
    if constexpr (KIND == NV_GATEUP) {
      brow = tl.el * 2 * p.I + tl.nt * BN;
      K = p.d;
    } else if constexpr (KIND == NV_DOWN) {
      brow = tl.el * p.d + tl.n0;
      K = p.I;
    } else if constexpr (KIND == NV_DGRAD_DOWN) {
      brow = tl.el * p.I + tl.n0;
      K = p.d;
    } else {  // NV_DGRAD_GATEUP: K = 2I, the dA / W_gate half, then the dB / W_up half
      const int half = p.I / 256;
      if (kb >= half) {
        kl = kb - half;
        ma = &p.ta1;
        mb = &p.tb1;
        sfa = p.sfa1;
        sfb = p.sfb1;
      }
      brow = tl.el * p.d + tl.n0;
      K = p.I;
    }
    const int arow = tl.m0;
    tma_load_2d(sA, ma, bar, kl * 128, arow, pol_act);
    tma_load_2d(sB, mb, bar, kl * 128, brow, pol_w);
    bulk_load(sSF, sfa + (static_cast<size_t>(arow >> 7) * (K >> 6) + 4 * kl) * 512, 2048, bar);
    bulk_load(sSF + 2048, sfb + (static_cast<size_t>(brow >> 7) * (K >> 6) + 4 * kl) * 512, 2048, bar);
    if constexpr (BN == 256)
      bulk_load(sSF + 4096, sfb + (static_cast<size_t>((brow >> 7) + 1) * (K >> 6) + 4 * kl) * 512, 2048, bar);
    (void)krow;
    return;
  }
  if constexpr (mx_is_wgrad(KIND)) {
    // the K block = row tile kt = krow / 128 of both operands (rowq layout): A = lines
    // kt CA + m0 .., B = lines kt CB + nb .. of 128 codes, and the tile's scale chunks
    const size_t kt = static_cast<size_t>(krow >> 7);
    (void)kb;
    const int CA = KIND == MX_WGRAD_GATEUP ? p.d : p.I, CB = KIND == MX_WGRAD_GATEUP ? p.I : p.d;
    int nb = tl.n0;
    if constexpr (KIND == MX_WGRAD_GATEUP) {
      const int NTg = p.I / 256;
      if (tl.nt >= NTg) {  // dW_up: Xq with dBq
        nb = (tl.nt - NTg) * 256;
        mb = &p.tb1;
        sfb = p.sfb1;
      }
    }
    tma_load_2d(sA, ma, bar, 0, static_cast<int>(kt * CA) + tl.m0, pol_act);
    tma_load_2d(sB, mb, bar, 0, static_cast<int>(kt * CB) + nb, pol_act);
    bulk_load(sSF, sfa + (kt * (CA >> 7) + (tl.m0 >> 7)) * 512, 512, bar);
    bulk_load(sSF + 512, sfb + (kt * (CB >> 7) + (nb >> 7)) * 512, 512, bar);
    bulk_load(sSF + 1024, sfb + (kt * (CB >> 7) + (nb >> 7) + 1) * 512, 512, bar);
    (void)pol_w;
    return;
  }
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
  const int arow = tl.m0 + (p.ring_shift ? __ldg(p.ring_shift) : 0);  // the A operand's row (ring position)
  tma_load_2d(sA, ma, bar, kl * 128, arow, pol_act);
  tma_load_2d(sB, mb, bar, kl * 128, brow, pol_w);
  bulk_load(sSF, sfa + (static_cast<size_t>(arow >> 7) * (KA >> 7) + kl) * 512, 512, bar);
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

// The warp's 32 rows (one 32-row block of one expert: tiles start on multiples of 128) x 32
// columns quantised along the rows for the MXFP8 weight gradients: the fp32 values go through
// the warp's shared-memory slice (32 x 33 words: row writes and column reads both hit 32
// distinct banks), lane i reads column col + i's 32 values, quantises them as one block
// (mx_quant32) and stores their 32 codes in the K-major, 128-row-tile-major operand q
// (rowq_index; C = I columns) and the scale byte.  v holds 0 for pad rows.
constexpr int MX_TPITCH = 33;
__device__ __forceinline__ void mx_store_rows_q32(uint8_t* q, uint8_t* qs, int R0, int col, int C,
                                                  const float (&v)[32], int lane, float* scratch) {
#pragma unroll
  for (int i = 0; i < 32; ++i) scratch[lane * MX_TPITCH + i] = v[i];
  __syncwarp();
  float c[32];
#pragma unroll
  for (int r = 0; r < 32; ++r) c[r] = scratch[r * MX_TPITCH + lane];
  __syncwarp();  // every lane has read the block before the next one is written
  uint32_t w[8];
  const uint8_t sb = mx_quant32(c, w);
  uint4* d = reinterpret_cast<uint4*>(q + rowq_index(col + lane, R0, C));
  d[0] = make_uint4(w[0], w[1], w[2], w[3]);
  d[1] = make_uint4(w[4], w[5], w[6], w[7]);
  qs[rowq_sf_index(col + lane, R0, C)] = sb;
}

// Rows past a segment's live pad rows (row_asg == ROW_DEAD) store nothing: no later kernel
// reads them.
// [cbeg, cend): this warp's share of the accumulator's 32-column chunks (all of them, or half
// when two warps share a TMEM lane quarter).
template <int KIND>
__device__ __forceinline__ void mx_epilogue(const MxParams& p, const MxTile& tl, int row, uint32_t taddr, int cbeg,
                                            int cend, float* scratch) {
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
  } else if constexpr (KIND == NV_GATEUP) {
    // A = acc / (gs_X gs_gate), B = acc / (gs_X gs_up); H = silu(A) B in fp32 for the second pass
    // (its amax sets H's global scale), the warp's largest |H| into *amax
    const float ag = __frcp_rn(__fmul_rn(__ldg(p.gsa), __ldg(p.gsb)));
    const float au = __frcp_rn(__fmul_rn(__ldg(p.gsa), __ldg(p.gsb + 1)));
    float hmax = 0.f;
#pragma unroll 1
    for (int c = cbeg; c < cend; ++c) {
      const int j = c >> 1, c32 = (c & 1) * 32;
      float a[32], b[32];
      tmem_ld32(taddr + j * 128 + c32, a);       // gate
      tmem_ld32(taddr + j * 128 + 64 + c32, b);  // up
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        a[i] *= ag;
        b[i] *= au;
      }
      if (live && p.out0) {  // A, B saved (bf16) for the backward
        mx_store_bf16_32(p.out0 + Rz * p.I + tl.n0 + j * 64 + c32, a);
        mx_store_bf16_32(p.out1 + Rz * p.I + tl.n0 + j * 64 + c32, b);
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        a[i] = a[i] / (1.0f + expf(-a[i])) * b[i];
        hmax = fmaxf(hmax, fabsf(a[i]));
      }
      if (live) {
        float4* dst = reinterpret_cast<float4*>(p.hout + Rz * p.I + tl.n0 + j * 64 + c32);
#pragma unroll
        for (int q = 0; q < 8; ++q) dst[q] = make_float4(a[4 * q], a[4 * q + 1], a[4 * q + 2], a[4 * q + 3]);
      }
    }
    if (!live) hmax = 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) hmax = fmaxf(hmax, __shfl_xor_sync(0xffffffffu, hmax, o));
    if ((row & 31) == 0 && hmax > 0.f) atomicMax(p.amax, __float_as_uint(hmax));
  } else if constexpr (KIND == NV_DOWN) {
    const float al = __frcp_rn(__fmul_rn(__ldg(p.gsa), __ldg(p.gsb)));
    const float g = p.row_gate[R];
#pragma unroll 1
    for (int c = cbeg; c < cend; ++c) {
      float o[32];
      tmem_ld32(taddr + c * 32, o);
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] = o[i] * al * g;
      if (live) mx_store_bf16_32(p.out0 + Rz * p.d + tl.n0 + c * 32, o);
    }
  } else if constexpr (KIND == NV_DGRAD_DOWN) {
    // dH' = acc / (gs_dY gs_down); the SwiGLU backward from the saved bf16 A, B as in
    // MX_DGRAD_DOWN; bf16 Hg for the bf16 weight gradient of W_down, fp32 dA, dB for their NVFP4
    // quantisation (which also writes their bf16 copies; out0 / out1 NULL) and the largest
    // |dA|, |dB| of the warp's live rows into *amax
    const float al = __frcp_rn(__fmul_rn(__ldg(p.gsa), __ldg(p.gsb)));
    const float g = p.row_gate[R];
    float dg = 0.f, amx = 0.f;
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
        const float d1 = dh[i] * al;
        const float s = mx_sigmoid(a[i]);
        const float sl = a[i] * s;
        const float hh = sl * b[i];
        dg = fmaf(d1, hh, dg);
        const float dhg = g * d1;
        a[i] = dhg * b[i] * (s * (1.0f + a[i] * (1.0f - s)));  // dA
        b[i] = dhg * sl;                                       // dB
        dh[i] = g * hh;                                        // Hg
        amx = fmaxf(amx, fmaxf(fabsf(a[i]), fabsf(b[i])));
      }
      if (live) {
        if (p.out0) {
          mx_store_bf16_32(p.out0 + Rz * p.I + col, a);
          mx_store_bf16_32(p.out1 + Rz * p.I + col, b);
        }
        mx_store_bf16_32(p.out2 + Rz * p.I + col, dh);
        float4* fa = reinterpret_cast<float4*>(p.hout + Rz * p.I + col);
        float4* fb = reinterpret_cast<float4*>(p.hout2 + Rz * p.I + col);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          fa[q] = make_float4(a[4 * q], a[4 * q + 1], a[4 * q + 2], a[4 * q + 3]);
          fb[q] = make_float4(b[4 * q], b[4 * q + 1], b[4 * q + 2], b[4 * q + 3]);
        }
      }
    }
    if (live) p.outf[Rz * (p.I / BN) + tl.nt] = dg;
    if (!live) amx = 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amx = fmaxf(amx, __shfl_xor_sync(0xffffffffu, amx, o));
    if ((row & 31) == 0 && amx > 0.f) atomicMax(p.amax, __float_as_uint(amx));
  } else if constexpr (KIND == NV_DGRAD_GATEUP) {
    const float al = __frcp_rn(__fmul_rn(__ldg(p.gsa), __ldg(p.gsb)));
#pragma unroll 1
    for (int c = cbeg; c < cend; ++c) {
      float v[32];
      tmem_ld32(taddr + c * 32, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] *= al;
      if (live) mx_store_bf16_32(p.out0 + Rz * p.d + tl.n0 + c * 32, v);
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
        if (p.out0) {  // bf16 operands of the bf16 weight gradients
          mx_store_bf16_32(p.out0 + Rz * p.I + col, a);
          mx_store_bf16_32(p.out1 + Rz * p.I + col, b);
          mx_store_bf16_32(p.out2 + Rz * p.I + col, dh);
        }
        mx_store_q32(p.q0, p.qs0, R, col, p.I, a);  // dA, dB: the gate/up dgrad's A operands (K = I)
        mx_store_q32(p.q1, p.qs1, R, col, p.I, b);
      }
      const int R0 = tl.m0 + (row & ~31);
      // MXFP8 weight gradients: dA, dB, Hg along the rows (warp-collective); a 32-row block that
      // starts past the expert's real rows is never read by the GEMM
      if (p.tq[0] && __ldg(p.row_asg + R0) >= 0) {
        const bool real = __ldg(p.row_asg + R) >= 0;
        const int lane = row & 31;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          if (!real) a[i] = b[i] = dh[i] = 0.f;
        }
        mx_store_rows_q32(p.tq[0], p.tqs[0], R0, col, p.I, a, lane, scratch);
        mx_store_rows_q32(p.tq[1], p.tqs[1], R0, col, p.I, b, lane, scratch);
        mx_store_rows_q32(p.tq[2], p.tqs[2], R0, col, p.I, dh, lane, scratch);
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

// Weight-gradient epilogue of one warp: its 32 gradient rows (TMEM lane quarter) x 128 columns
// (half of the 256-wide tile).  The accumulator slice goes to registers first and the warp
// releases it (acc_empty) before any store, so the next tile's MMAs run while the gradient is
// written: bf16 as two 64 x 32 boxes, or fp32 (wout32) as four 32 x 32 boxes, each staged in
// one of the warp's two 4 KB slots (128-byte swizzle, as the output maps expect) and written by
// a TMA store; a slot is refilled once the store issued from it has read it.  An expert without
// rows has a zero gradient.
__device__ __forceinline__ void mx_stage16(uint8_t* box, int lane, int chunk, uint4 u) {
  *reinterpret_cast<uint4*>(box + lane * 128 + ((chunk ^ (lane & 7)) << 4)) = u;
}

template <int KIND>
__device__ __forceinline__ void mx_epilogue_wgrad(const MxParams& p, const MxTile& tl, int quarter, int half,
                                                  int lane, uint32_t taddr, uint8_t* stage_out,
                                                  uint64_t* acc_empty) {
  int x0, y0;
  const CUtensorMap* map = &p.to0;
  if constexpr (KIND == MX_WGRAD_GATEUP) {
    const int NTg = p.I / 256;
    const bool up = tl.nt >= NTg;  // dW_gate or dW_up as [El*d, I]
    if (up) map = &p.to1;
    x0 = (up ? tl.nt - NTg : tl.nt) * 256 + half * 128;
    y0 = tl.el * p.d + tl.m0 + quarter * 32;
  } else {
    x0 = tl.n0 + half * 128;  // dW_down as [El*I, d]
    y0 = tl.el * p.I + tl.m0 + quarter * 32;
  }
  uint32_t r[2][64];
  if (tl.nk > 0) {
    tmem_ld64_issue(taddr, r[0]);
    tmem_ld64_issue(taddr + 64, r[1]);
    tmem_ld64_wait(r[0]);
    tmem_ld64_wait(r[1]);
  } else {
#pragma unroll
    for (int i = 0; i < 64; ++i) r[0][i] = r[1][i] = 0u;
  }
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(acc_empty);
  if (!p.wout32) {
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      if (lane == 0) bulk_wait_read<1>();
      __syncwarp();
      uint8_t* box = stage_out + b * 4096;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint32_t* w = r[b] + 8 * q;
        mx_stage16(box, lane, q,
                   make_uint4(pack_bf16(__uint_as_float(w[0]), __uint_as_float(w[1])),
                              pack_bf16(__uint_as_float(w[2]), __uint_as_float(w[3])),
                              pack_bf16(__uint_as_float(w[4]), __uint_as_float(w[5])),
                              pack_bf16(__uint_as_float(w[6]), __uint_as_float(w[7]))));
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(map, box, x0 + b * 64, y0);
        bulk_commit();
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (lane == 0) bulk_wait_read<1>();
      __syncwarp();
      uint8_t* box = stage_out + (j & 1) * 4096;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint32_t* w = r[j >> 1] + (j & 1) * 32 + 4 * q;
        mx_stage16(box, lane, q, make_uint4(w[0], w[1], w[2], w[3]));
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(map, box, x0 + j * 32, y0);
        bulk_commit();
      }
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
  uint8_t* stage_out = smem + STAGES * SB;  // weight-gradient kinds: 8 KB per epilogue warp; dgrad of W_down: 1 KB
  uint64_t* full = reinterpret_cast<uint64_t*>(stage_out + mx_out_bytes(KIND));
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
        if constexpr (mx_is_wgrad(KIND)) {  // K: the 128-row blocks of each of the expert's segments
          for (int m = 0, nm = p.nseg / p.El; m < nm && ok; ++m) {
            int r0, rows;
            mx_wseg(p, m, tl.el, r0, rows);
            for (int j = 0; j * 128 < rows; ++j) {
              if (!mbar_wait(&empty[stage], phase ^ 1, p.status)) { ok = false; break; }
              mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>(mx_stage_tx(KIND)));
              mx_load<KIND>(p, tl, 0, r0 + j * 128, smem + stage * SB, &full[stage], pol_act, pol_w);
              last_parity[stage] = static_cast<int>(phase);
              if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
          }
        } else {
          for (int kb = 0; kb < tl.nk; ++kb) {
            if (!mbar_wait(&empty[stage], phase ^ 1, p.status)) { ok = false; break; }
            mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>(mx_stage_tx(KIND)));
            mx_load<KIND>(p, tl, kb, 0, smem + stage * SB, &full[stage], pol_act, pol_w);
            last_parity[stage] = static_cast<int>(phase);
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
          }
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
        // weight gradients: K walks the expert's segments; (m, j, rows) track the current block
        int m = 0, j = 0, rows = 0;
        if constexpr (mx_is_wgrad(KIND)) {
          int r0;
          mx_wseg(p, 0, tl.el, r0, rows);
        }
        for (int kb = 0; kb < tl.nk; ++kb) {
          if constexpr (mx_is_wgrad(KIND)) {
            while (j * 128 >= rows) {  // past this segment: the next one with rows (nk counts them)
              int r0;
              ++m;
              j = 0;
              mx_wseg(p, m, tl.el, r0, rows);
            }
          }
          if (!mbar_wait(&full[stage], phase, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * SB);
          const uint32_t b0 = a0 + static_cast<uint32_t>(MX_A_BYTES);
          const uint32_t sf0 = b0 + static_cast<uint32_t>(BN * 128);
          // scale slot of this stage: 16 columns from column 256 on; A in the first 4,
          // B (rows 0..127, then 128..255) in the columns from 8 on
          if constexpr (mx_is_nv(KIND)) {
            // per stage TMEM columns above the accumulators: A's four chunks (4 columns each),
            // then per K = 64 step B's 128-row halves (4 columns each)
            constexpr uint32_t BW = 4 * (BN / 128);  // B columns per K = 64 step
            const uint32_t nfa = tbase + 256 + stage * (16 + 4 * BW), nfb = nfa + 16;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              tc_cp_sf(nfa + 4 * kk, sf0 + 512 * kk);
              tc_cp_sf(nfb + BW * kk, sf0 + 2048 + 512 * kk);
              if constexpr (BN == 256) tc_cp_sf(nfb + BW * kk + 4, sf0 + 4096 + 512 * kk);
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_nvf4(dtm, sdesc_sw128(a0 + kk * 32, 16, 1024), sdesc_sw128(b0 + kk * 32, 16, 1024),
                        idesc_nvf4(128, BN), nfa + 4 * kk, nfb + BW * kk, (kb | kk) != 0 ? 1u : 0u);
            umma_commit(&empty[stage]);
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
            continue;
          }
          const uint32_t sfa_t = tbase + 256 + stage * 16, sfb_t = sfa_t + 8;
          tc_cp_sf(sfa_t, sf0);
          tc_cp_sf(sfb_t, sf0 + 512);
          if constexpr (BN == 256) tc_cp_sf(sfb_t + 4, sf0 + 1024);
          // weight gradients: the last 128-row block issues only the K = 32 steps with real rows
          // (its rows past them up to the next multiple of 32 are zero codes)
          int nkk = 4;
          if constexpr (mx_is_wgrad(KIND)) {
            const int valid = rows - j * 128;
            if (valid < 128) nkk = (valid + 31) / 32;
            ++j;
          }
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            if (kk < nkk)
              umma_mxf8(dtm, sdesc_sw128(a0 + kk * 32, 16, 1024), sdesc_sw128(b0 + kk * 32, 16, 1024),
                        idesc_mxf8(128, BN, static_cast<uint32_t>(kk)), sfa_t, sfb_t, (kb | kk) != 0 ? 1u : 0u);
          umma_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if (tl.nk > 0) umma_commit(&tfull[acc]);
        else mbar_arrive(&tfull[acc]);  // an expert without rows: nothing to wait for
      }
      umma_commit(drain);
      mx_wait_drain(drain, 0);
    }
  } else {  // epilogue warps 2 .. 2 + EPI - 1
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    constexpr int NCH = KIND == MX_GATEUP || KIND == NV_GATEUP ? BN / 64 : BN / 32;  // 32-column chunks of the epilogue
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
      const uint32_t taddr = tbase + (static_cast<uint32_t>(quarter * 32) << 16) + acc * BN;
      if constexpr (mx_is_wgrad(KIND)) {  // releases the accumulator itself, before its stores
        mx_epilogue_wgrad<KIND>(p, tl, quarter, half, lane, taddr + half * 128, stage_out + (warp - 2) * 8192,
                                &tempty[acc]);
        continue;
      }
      mx_epilogue<KIND>(p, tl, row, taddr, cbeg, cend,
                        reinterpret_cast<float*>(stage_out) + (KIND == MX_DGRAD_DOWN ? (warp - 2) * 32 * MX_TPITCH : 0));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
    if constexpr (mx_is_wgrad(KIND)) {
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
    case MX_WGRAD_GATEUP: return mx_launch_kind<MX_WGRAD_GATEUP>(p, grid, st);
    case MX_WGRAD_DOWN: return mx_launch_kind<MX_WGRAD_DOWN>(p, grid, st);
    case NV_GATEUP: return mx_launch_kind<NV_GATEUP>(p, grid, st);
    case NV_DOWN: return mx_launch_kind<NV_DOWN>(p, grid, st);
    case NV_DGRAD_DOWN: return mx_launch_kind<NV_DGRAD_DOWN>(p, grid, st);
    case NV_DGRAD_GATEUP: return mx_launch_kind<NV_DGRAD_GATEUP>(p, grid, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace moe
