// Routing, dispatch and combine kernels of the MoE layer (and their
// backward mirrors).  These are the "schedule table" steps of the MoK pages
// (page 1, "Three design decisions that matter", bullet 1): one routing table
// (counts, prefix sums, a stable per-expert token order) drives the forward
// dispatch and combine and the backward reverse-combine and reverse-dispatch.
// On one GPU the NVLink pull/push becomes an on-device gather.
//
// Every reduction has a fixed order; integer atomics are used only where the
// result does not depend on their order (shared-memory histogram counts).
#include <cfloat>
#include <cmath>

#include "moe_internal.cuh"
#include "ptx.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// top-k + softmax gating, one warp per token, plus a per-block expert histogram.
// Order key: value descending, then expert id ascending; -0 == +0; NaN lowest.
// ---------------------------------------------------------------------------
__device__ __forceinline__ unsigned long long order_key(float v, int e) {
  uint32_t ord;
  if (isnan(v)) {
    ord = 1u;  // below every number, above a removed entry (key 0)
  } else {
    if (v == 0.f) v = 0.f;  // -0 -> +0
    const uint32_t u = __float_as_uint(v);
    ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  }
  return (static_cast<unsigned long long>(ord) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(e));
}

// The router GEMM leaves `splits` fp32 partial sums per logit (fixed K ranges);
// they are added here in split order, then the bias, and the logit is stored.
// NQ = logits per lane (E <= 32 NQ); the loads of one split are all in flight together.
template <int NQ>
__global__ void __launch_bounds__(kTokensPerBlock * 32) k_topk(const float* __restrict__ part, int splits,
                                                               const float* __restrict__ bias,
                                                               float* __restrict__ logits, int T, int E, int k,
                                                               int* __restrict__ ids, float* __restrict__ gates,
                                                               int* __restrict__ hist, int* status) {
  __shared__ int sh[kMaxE];
  for (int i = threadIdx.x; i < E; i += blockDim.x) sh[i] = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kTokensPerBlock + warp;
  if (t < T) {
    float* row = logits + static_cast<size_t>(t) * E;
    const size_t plane = static_cast<size_t>(T) * E;
    const float* pp = part + static_cast<size_t>(t) * E;
    float v[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      const int e = lane + 32 * q;
      v[q] = e < E ? pp[e] : 0.f;
    }
    for (int sp = 1; sp < splits; ++sp) {
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const int e = lane + 32 * q;
        if (e < E) v[q] += pp[sp * plane + e];
      }
    }
    unsigned long long key[NQ];
    bool bad = false;
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      const int e = lane + 32 * q;
      key[q] = 0ull;
      if (e < E) {
        if (bias) v[q] += bias[e];
        row[e] = v[q];
        bad |= !isfinite(v[q]);
        key[q] = order_key(v[q], e);
      }
    }
    int my_e = 0;
    float my_v = 0.f;
    for (int j = 0; j < k; ++j) {
      unsigned long long best = 0ull;
      int bq = -1;
#pragma unroll
      for (int q = 0; q < NQ; ++q)
        if (key[q] > best) { best = key[q]; bq = q; }
      unsigned long long wb = best;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const unsigned long long o = __shfl_xor_sync(0xffffffffu, wb, off);
        wb = o > wb ? o : wb;
      }
      const int e = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(wb & 0xFFFFFFFFull));
      if (bq >= 0 && best == wb) {  // the owning lane removes the winner (ids are unique)
#pragma unroll
        for (int q = 0; q < NQ; ++q)
          if (q == bq) key[q] = 0ull;
      }
      if (lane == j) {  // the winner's logit, back from its key (-0 comes back as +0)
        const uint32_t ord = static_cast<uint32_t>(wb >> 32);
        my_e = e;
        my_v = __uint_as_float((ord & 0x80000000u) ? (ord & 0x7FFFFFFFu) : ~ord);
      }
    }
    // softmax over the selected logits; the first selected is the largest
    const float vmax = __shfl_sync(0xffffffffu, my_v, 0);
    const float ex = lane < k ? expf(my_v - vmax) : 0.f;
    float sum = 0.f;
    for (int j = 0; j < k; ++j) sum += __shfl_sync(0xffffffffu, ex, j);  // fixed order
    if (lane < k) {
      ids[static_cast<size_t>(t) * k + lane] = my_e;
      gates[static_cast<size_t>(t) * k + lane] = ex / sum;
      atomicAdd(&sh[my_e], 1);
    }
    bad = __any_sync(0xffffffffu, bad);
    if (bad && lane == 0) raise_status(status, MOE_ERR_NONFINITE);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < E; i += blockDim.x) hist[static_cast<size_t>(blockIdx.x) * E + i] = sh[i];
}

// ---------------------------------------------------------------------------
// histogram -> per-block bases, counts, offsets, padded offsets (one block).
// hist[b][e] is replaced in place by the exclusive scan over b.
// ---------------------------------------------------------------------------
// inclusive scan across the warp
__device__ __forceinline__ int warp_incl_scan(int x, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x;
}
// exclusive scan of one value per thread across the block (threads in order); *total gets the sum
__device__ __forceinline__ int block_excl_scan(int v, int* wsum, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int x = warp_incl_scan(v, lane);
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int w = warp_incl_scan(lane < nw ? wsum[lane] : 0, lane);
    if (lane < nw) wsum[lane] = w;
  }
  __syncthreads();
  const int r = (warp > 0 ? wsum[warp - 1] : 0) + x - v;
  *total = wsum[nw - 1];
  __syncthreads();  // wsum is reused by the next scan
  return r;
}

// Column scan of the per-block histograms: hist[b][e] becomes the exclusive prefix over blocks
// b' < b (each token block's base inside expert e), counts[e] the total.  One thread per expert
// (a warp reads 32 consecutive experts of a row), sixteen rows' loads in flight; then the expert
// offsets and the padded offsets of the local experts by block-wide scans.
__global__ void __launch_bounds__(1024) k_scan(int* __restrict__ hist, int nblk, int E, int first, int El,
                                               int* __restrict__ counts, int* __restrict__ offsets,
                                               int* __restrict__ poff, int* __restrict__ hdr) {
  __shared__ int sc[kMaxE];
  __shared__ int wsum[32];
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    for (int b0 = 0; b0 < nblk; b0 += 16) {
      int h[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) h[j] = b0 + j < nblk ? hist[static_cast<size_t>(b0 + j) * E + e] : 0;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (b0 + j < nblk) hist[static_cast<size_t>(b0 + j) * E + e] = run;
        run += h[j];
      }
    }
    counts[e] = run;
    sc[e] = run;
  }
  __syncthreads();
  // E <= kMaxE <= blockDim: one expert per thread
  const int e = threadIdx.x;
  const int c = e < E ? sc[e] : 0;
  int total = 0;
  const int off = block_excl_scan(c, wsum, &total);
  if (e < E) offsets[e] = off;
  if (e == 0) offsets[E] = total;
  const bool local = e >= first && e < first + El;
  const int padded = local ? (c + kPad - 1) / kPad * kPad : 0;
  const int poffe = block_excl_scan(padded, wsum, &total);  // local experts are contiguous in e
  if (local) poff[e - first] = poffe;
  if (e == 0) {
    poff[El] = total;
    hdr[HDR_ROWS_P] = total;
    hdr[HDR_MTILES] = total / kPad;
  }
}

// Two-level form for many token blocks (the single block above walks all nblk rows of every
// column): one block per group of kScanGroup rows sums its rows, k_scan turns the group sums
// into exclusive prefixes over groups (and computes counts, offsets, padded offsets), and one
// block per group writes each row's prefix.  Integer sums: the same result as one pass.
__global__ void __launch_bounds__(512) k_scan_group_sums(const int* __restrict__ hist, int nblk, int E,
                                                         int* __restrict__ gsum) {
  const int b0 = blockIdx.x * kScanGroup;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int h[kScanGroup];
#pragma unroll
    for (int j = 0; j < kScanGroup; ++j) h[j] = b0 + j < nblk ? hist[static_cast<size_t>(b0 + j) * E + e] : 0;
    int sum = 0;
#pragma unroll
    for (int j = 0; j < kScanGroup; ++j) sum += h[j];
    gsum[static_cast<size_t>(blockIdx.x) * E + e] = sum;
  }
}
__global__ void __launch_bounds__(512) k_scan_group_apply(int* __restrict__ hist, int nblk, int E,
                                                          const int* __restrict__ gsum) {
  const int b0 = blockIdx.x * kScanGroup;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int h[kScanGroup];
#pragma unroll
    for (int j = 0; j < kScanGroup; ++j) h[j] = b0 + j < nblk ? hist[static_cast<size_t>(b0 + j) * E + e] : 0;
    int run = gsum[static_cast<size_t>(blockIdx.x) * E + e];
#pragma unroll
    for (int j = 0; j < kScanGroup; ++j) {
      if (b0 + j < nblk) hist[static_cast<size_t>(b0 + j) * E + e] = run;
      run += h[j];
    }
  }
}

// ---------------------------------------------------------------------------
// pad-row marks of every segment, before the scatter fills its real rows: rows up to the real
// count rounded up to 16 are ROW_PAD, the rest of the 128-row padding ROW_DEAD; gates 0.
// One block per segment; with macrobatches, segment m * El + el counts cum's difference.
__global__ void __launch_bounds__(128) k_mark_rows(const int* __restrict__ poff, int nseg, int El,
                                                   const int* __restrict__ cnt, const int* __restrict__ cum, int nm,
                                                   int* __restrict__ row_asg, float* __restrict__ row_gate) {
  const int s = blockIdx.x;
  if (s >= nseg) return;
  const int el = s % El, m = s / El;
  const int tot = cnt[el];
  const int rows = cum ? (m + 1 < nm ? cum[(m + 1) * El + el] : tot) - cum[m * El + el] : tot;
  const int live = (rows + 15) & ~15;
  const int r0 = poff[s], r1 = poff[s + 1];
  for (int r = r0 + threadIdx.x; r < r1; r += blockDim.x) {
    row_asg[r] = r - r0 < live ? ROW_PAD : ROW_DEAD;
    row_gate[r] = 0.f;
  }
}

// ---------------------------------------------------------------------------
// stable scatter: one warp per block of tokens, tokens in ascending order.
// row position of (t, j) inside expert e = base[b][e] + #{earlier tokens of b with e}.
// ---------------------------------------------------------------------------
// Ring-streamed layer: the padded rows are grouped by macrobatch, then expert
// (segment m * El + el starts at seg_poff[...]); `cum` counts the expert's
// assignments in earlier macrobatches.  Without macrobatches (mb_of == NULL)
// the segments are the experts' and poff gives their starts.
__global__ void __launch_bounds__(32) k_scatter(const int* __restrict__ ids, const float* __restrict__ gates,
                                                const int* __restrict__ base, const int* __restrict__ offsets,
                                                const int* __restrict__ poff, int T, int E, int k, int first, int El,
                                                int T_mb, const int* __restrict__ mb_of, const int* __restrict__ cum,
                                                int* __restrict__ perm_tok, int* __restrict__ perm_asg,
                                                int* __restrict__ slot_row, int* __restrict__ row_asg,
                                                float* __restrict__ row_gate) {
  __shared__ int run[kMaxE];
  const int b = blockIdx.x, lane = threadIdx.x;
  for (int e = lane; e < E; e += 32) run[e] = base[static_cast<size_t>(b) * E + e];
  __syncwarp();
  for (int i = 0; i < kTokensPerBlock; ++i) {
    const int t = b * kTokensPerBlock + i;
    if (t >= T) break;
    if (lane < k) {
      const int a = t * k + lane;
      const int e = ids[a];
      const int pos = run[e];
      run[e] = pos + 1;  // the k experts of one token are distinct: no two lanes share e
      const int u = offsets[e] + pos;
      perm_tok[u] = t;
      perm_asg[u] = a;
      const int el = e - first;
      if (el >= 0 && el < El) {
        int R;
        if (mb_of) {
          const int sg = mb_of[t / T_mb] * El + el;
          R = poff[sg] + pos - cum[sg];
        } else {
          R = poff[el] + pos;
        }
        slot_row[a] = R;
        row_asg[R] = a;
        row_gate[R] = gates[a];
      } else {
        slot_row[a] = -1;
      }
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------
// dispatch / reverse-combine: dst[R] = src[token(R)], zero rows for live pad rows, dead pad
// rows left as they are.
// ---------------------------------------------------------------------------
// Rows [*lo, *hi) of the padded layout, written at row R + *shift of dst (a
// ring position for the streamed layer; shift NULL = 0).
__global__ void __launch_bounds__(128) k_gather_rows(const __nv_bfloat16* __restrict__ src,
                                                     const int* __restrict__ row_asg, const int* __restrict__ lo,
                                                     const int* __restrict__ hi, const int* __restrict__ shift, int k,
                                                     int d, __nv_bfloat16* __restrict__ dst) {
  const int r0 = __ldg(lo), r1 = __ldg(hi);
  const int sh = shift ? __ldg(shift) : 0;
  const int nv = d / 8;  // 16-byte chunks per row
  for (int64_t R = r0 + blockIdx.x; R < r1; R += gridDim.x) {
    const int a = row_asg[R];
    if (a == ROW_DEAD) continue;  // never read
    uint4* out = reinterpret_cast<uint4*>(dst + (R + sh) * d);
    const uint4* in = a >= 0 ? reinterpret_cast<const uint4*>(src + static_cast<size_t>(a / k) * d) : nullptr;
    // four independent loads in flight per thread before their stores
    for (int i0 = threadIdx.x; i0 < nv; i0 += 4 * blockDim.x) {
      uint4 u[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = i0 + j * blockDim.x;
        u[j] = (in != nullptr && i < nv) ? __ldg(in + i) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = i0 + j * blockDim.x;
        if (i < nv) out[i] = u[j];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// combine: Y[t] = sum_j O'[slot_row[t, j]] in slot order, fp32, stored bf16.
// ---------------------------------------------------------------------------
// Tokens [0, T), or the minibatches [range[0], range[1]) of T_mb tokens each.
__global__ void __launch_bounds__(128) k_combine(const __nv_bfloat16* __restrict__ Op,
                                                 const int* __restrict__ slot_row, int k, int d, int T,
                                                 const int* __restrict__ range, int T_mb,
                                                 __nv_bfloat16* __restrict__ Y) {
  const int t0 = range ? __ldg(range) * T_mb : 0;
  const int t1 = range ? __ldg(range + 1) * T_mb : T;
  __shared__ int rows[kMaxK];
  for (int t = t0 + blockIdx.x; t < t1; t += gridDim.x) {
  __syncthreads();
  if (threadIdx.x < k) rows[threadIdx.x] = slot_row[static_cast<size_t>(t) * k + threadIdx.x];
  __syncthreads();
  for (int i = threadIdx.x * 8; i < d; i += blockDim.x * 8) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < k; ++j) {
      const int R = rows[j];
      if (R < 0) continue;
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(Op + static_cast<size_t>(R) * d + i));
      float2 f;
      f = unpack_bf16(u.x); acc[0] += f.x; acc[1] += f.y;
      f = unpack_bf16(u.y); acc[2] += f.x; acc[3] += f.y;
      f = unpack_bf16(u.z); acc[4] += f.x; acc[5] += f.y;
      f = unpack_bf16(u.w); acc[6] += f.x; acc[7] += f.y;
    }
    uint4 o;
    o.x = pack_bf16(acc[0], acc[1]);
    o.y = pack_bf16(acc[2], acc[3]);
    o.z = pack_bf16(acc[4], acc[5]);
    o.w = pack_bf16(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(Y + static_cast<size_t>(t) * d + i) = o;
  }
  }
}

// ---------------------------------------------------------------------------
// router backward, one warp per token:
//   dg_j = sum over n-tiles of the dgrad epilogue's partials (fixed order)
//   dl_j = g_j (dg_j - sum_m g_m dg_m)
// ---------------------------------------------------------------------------
// dl of each token's k assignments; also the token's rows of the dense dl matrix, the router
// weight gradient's B operand, as two bf16 terms: hi = bf16(dl) in row t, lo = bf16(dl - hi) in
// row Tpad + t (zeros elsewhere), so the tensor cores see dl to about 16 bits.  Warps of tokens
// in [T, Tpad) write the zero rows that pad K to a multiple of 64.
__global__ void __launch_bounds__(256) k_router_bwd(const float* __restrict__ dgpart, const int* __restrict__ slot_row,
                                                    const float* __restrict__ gates, const int* __restrict__ ids, int T,
                                                    int Tpad, int k, int ntn, int E64, float* __restrict__ dlasg,
                                                    __nv_bfloat16* __restrict__ dldense) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= Tpad) return;
  uint4* hi_row = reinterpret_cast<uint4*>(dldense + static_cast<size_t>(t) * E64);
  uint4* lo_row = reinterpret_cast<uint4*>(dldense + (static_cast<size_t>(Tpad) + t) * E64);
  for (int i = lane; i < E64 / 8; i += 32) hi_row[i] = lo_row[i] = make_uint4(0, 0, 0, 0);
  if (t >= T) return;
  float dg = 0.f, g = 0.f;
  if (lane < k) {
    const size_t a = static_cast<size_t>(t) * k + lane;
    const int R = slot_row[a];
    g = gates[a];
    if (R >= 0)
      for (int q = 0; q < ntn; ++q) dg += dgpart[static_cast<size_t>(R) * ntn + q];
  }
  float s = 0.f;
  const float gd = g * dg;
  for (int j = 0; j < k; ++j) s += __shfl_sync(0xffffffffu, gd, j);
  const float dl = g * (dg - s);
  __syncwarp();  // the zero rows are written before the k entries
  if (lane < k) {
    const size_t a = static_cast<size_t>(t) * k + lane;
    dlasg[a] = dl;
    const __nv_bfloat16 hi = __float2bfloat16_rn(dl);
    const int e = ids[a];
    dldense[static_cast<size_t>(t) * E64 + e] = hi;
    dldense[(static_cast<size_t>(Tpad) + t) * E64 + e] = __float2bfloat16_rn(dl - __bfloat162float(hi));
  }
}

// ---------------------------------------------------------------------------
// Router weight gradient of an expert slice.  A token with no local assignment has dg = 0 on
// every slot, hence dl = 0, so only tokens with a local assignment add to dW_r = X^T DL.  They
// are listed in ascending token order (a count per 256-token block, a fixed-order sum of the
// counts before each block and a ballot scan inside it) and the contraction runs over the
// list alone: row a of the compacted DL and X matrices is the a-th listed token.
// ---------------------------------------------------------------------------
constexpr int kActBlock = 256;

__device__ __forceinline__ int has_local_slot(const int* __restrict__ slot_row, int64_t t, int k) {
  int act = 0;
  for (int j = 0; j < k; ++j) act |= __ldg(slot_row + t * k + j) >= 0;
  return act;
}

__global__ void __launch_bounds__(kActBlock) k_active_count(const int* __restrict__ slot_row, int T, int k,
                                                            int* __restrict__ cnt) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kActBlock + threadIdx.x;
  const int n = __syncthreads_count(t < T ? has_local_slot(slot_row, t, k) : 0);
  if (threadIdx.x == 0) cnt[blockIdx.x] = n;
}

// dl of every token (dlasg), and the hi / lo DL rows of the listed tokens at their list index
// a (hi row a, lo row Tpad + a).  cnt[0 .. nb) are the block counts; the last block stores the
// list length in cnt[nb] and zeroes the rows that pad it to a multiple of 64 in both halves.
__global__ void __launch_bounds__(kActBlock) k_router_bwd_compact(
    const float* __restrict__ dgpart, const int* __restrict__ slot_row, const float* __restrict__ gates,
    const int* __restrict__ ids, int T, int Tpad, int k, int ntn, int E64, int* __restrict__ cnt, int nb,
    float* __restrict__ dlasg, __nv_bfloat16* __restrict__ dldense, int* __restrict__ act_list) {
  __shared__ int s_idx[kActBlock];
  __shared__ int s_warp[kActBlock / 32];
  __shared__ int s_base, s_total;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    int before = 0, total = 0;
    for (int i = lane; i < nb; i += 32) {
      const int c = cnt[i];
      total += c;
      if (i < static_cast<int>(blockIdx.x)) before += c;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      before += __shfl_xor_sync(0xffffffffu, before, o);
      total += __shfl_xor_sync(0xffffffffu, total, o);
    }
    if (lane == 0) {
      s_base = before;
      s_total = total;
    }
  }
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kActBlock;
  const int64_t t = t0 + threadIdx.x;
  const int act = t < T ? has_local_slot(slot_row, t, k) : 0;
  const unsigned bal = __ballot_sync(0xffffffffu, act);
  if (lane == 0) s_warp[warp] = __popc(bal);
  __syncthreads();
  int woff = 0;
  for (int w = 0; w < warp; ++w) woff += s_warp[w];
  const int a = act ? s_base + woff + __popc(bal & ((1u << lane) - 1u)) : -1;
  s_idx[threadIdx.x] = a;
  if (a >= 0) act_list[a] = static_cast<int>(t);
  __syncthreads();
  const int n4 = E64 / 8;
  if (blockIdx.x == gridDim.x - 1) {
    const int tot = s_total, pad = (tot + 63) / 64 * 64;
    if (threadIdx.x == 0) cnt[nb] = tot;
    for (int i = threadIdx.x; i < (pad - tot) * n4; i += kActBlock) {
      const int r = tot + i / n4, q = i % n4;
      reinterpret_cast<uint4*>(dldense + static_cast<size_t>(r) * E64)[q] = make_uint4(0, 0, 0, 0);
      reinterpret_cast<uint4*>(dldense + (static_cast<size_t>(Tpad) + r) * E64)[q] = make_uint4(0, 0, 0, 0);
    }
  }
  // a warp per token, 32 tokens per warp
  for (int i = 0; i < 32; ++i) {
    const int tl = warp * 32 + i;
    const int64_t tt = t0 + tl;
    if (tt >= T) break;  // the same for every lane
    float dg = 0.f, g = 0.f;
    if (lane < k) {
      const size_t as = static_cast<size_t>(tt) * k + lane;
      const int R = slot_row[as];
      g = gates[as];
      if (R >= 0)
        for (int q = 0; q < ntn; ++q) dg += dgpart[static_cast<size_t>(R) * ntn + q];
    }
    float sum = 0.f;
    const float gd = g * dg;
    for (int j = 0; j < k; ++j) sum += __shfl_sync(0xffffffffu, gd, j);
    const float dl = g * (dg - sum);
    if (lane < k) dlasg[static_cast<size_t>(tt) * k + lane] = dl;
    const int ar = s_idx[tl];
    if (ar >= 0) {
      uint4* hi_row = reinterpret_cast<uint4*>(dldense + static_cast<size_t>(ar) * E64);
      uint4* lo_row = reinterpret_cast<uint4*>(dldense + (static_cast<size_t>(Tpad) + ar) * E64);
      for (int q = lane; q < n4; q += 32) hi_row[q] = lo_row[q] = make_uint4(0, 0, 0, 0);
      __syncwarp();  // the zero rows are written before the k entries
      if (lane < k) {
        const int e = ids[static_cast<size_t>(tt) * k + lane];
        const __nv_bfloat16 hi = __float2bfloat16_rn(dl);
        dldense[static_cast<size_t>(ar) * E64 + e] = hi;
        dldense[(static_cast<size_t>(Tpad) + ar) * E64 + e] = __float2bfloat16_rn(dl - __bfloat162float(hi));
      }
    }
  }
}

// X rows of the listed tokens, then zero rows up to the next multiple of 64 (a warp per row,
// four 16-byte loads in flight per lane)
__global__ void __launch_bounds__(256) k_gather_active(const __nv_bfloat16* __restrict__ X, int d,
                                                       const int* __restrict__ act_list, const int* __restrict__ act_n,
                                                       int64_t max_rows, __nv_bfloat16* __restrict__ Xa) {
  const int n = __ldg(act_n);
  const int64_t pad = (static_cast<int64_t>(n) + 63) / 64 * 64;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nv = d / 8;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + warp; r < pad && r < max_rows;
       r += static_cast<int64_t>(gridDim.x) * 8) {
    uint4* o = reinterpret_cast<uint4*>(Xa + r * d);
    const uint4* in = r < n ? reinterpret_cast<const uint4*>(X + static_cast<int64_t>(__ldg(act_list + r)) * d)
                            : nullptr;
    for (int c0 = lane; c0 < nv; c0 += 128) {
      uint4 u[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = c0 + 32 * j;
        u[j] = (in != nullptr && c < nv) ? __ldg(in + c) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (c0 + 32 * j < nv) o[c0 + 32 * j] = u[j];
    }
  }
}

// W_r [d, E] -> W_r^T [E, d] (bf16), 32 x 32 tiles
__global__ void __launch_bounds__(256) k_transpose_wr(const __nv_bfloat16* __restrict__ Wr, int d, int E,
                                                      __nv_bfloat16* __restrict__ WrT) {
  __shared__ __nv_bfloat16 tile[32][33];
  const int i0 = blockIdx.y * 32, e0 = blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int r = ty; r < 32; r += 8) {
    const int i = i0 + r, e = e0 + tx;
    if (i < d && e < E) tile[r][tx] = Wr[static_cast<size_t>(i) * E + e];
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    const int e = e0 + r, i = i0 + tx;
    if (i < d && e < E) WrT[static_cast<size_t>(e) * d + i] = tile[tx][r];
  }
}
// The same for E a multiple of 8, with 16-byte global accesses: 64 (d) x 64 (E) tiles; each
// thread loads two 8-element vectors and stores two, through a tile with an odd row pitch (65
// elements) so that both the row-wise writes and the column-wise reads spread over the banks.
__global__ void __launch_bounds__(256) k_transpose_wr_v(const __nv_bfloat16* __restrict__ Wr, int d, int E,
                                                        __nv_bfloat16* __restrict__ WrT) {
  __shared__ __nv_bfloat16 tile[64][65];  // [i][e]
  const int i0 = blockIdx.y * 64, e0 = blockIdx.x * 64;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int c = threadIdx.x + h * 256;  // 512 chunks: row i (64) x chunk (8 elements of e)
    const int r = c >> 3, ch = c & 7;
    const int e = e0 + ch * 8;
    __align__(16) __nv_bfloat16 v[8];
    *reinterpret_cast<uint4*>(v) = e < E ? __ldg(reinterpret_cast<const uint4*>(Wr + static_cast<size_t>(i0 + r) * E + e))
                                         : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int j = 0; j < 8; ++j) tile[r][ch * 8 + j] = v[j];
  }
  __syncthreads();
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int c = threadIdx.x + h * 256;  // 512 chunks: row e (64) x chunk (8 elements of i)
    const int r = c >> 3, ch = c & 7;
    const int e = e0 + r;
    if (e >= E) continue;
    __align__(16) __nv_bfloat16 v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = tile[ch * 8 + j][r];
    *reinterpret_cast<uint4*>(WrT + static_cast<size_t>(e) * d + i0 + ch * 8) = *reinterpret_cast<const uint4*>(v);
  }
}

// ---------------------------------------------------------------------------
// reverse-dispatch: dX[t] = sum_j dX_perm[slot_row[t,j]] + sum_j dl_j W_r[:, e_j]
// (expert terms first, then router terms, each in slot order; fp32; bf16 out).  A router term
// with dl_j = 0 adds nothing and is skipped: in an expert slice that is every slot of a token
// with no local assignment, whose row is then written without reading W_r.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) k_rev_dispatch(const __nv_bfloat16* __restrict__ dxperm,
                                                      const int* __restrict__ slot_row, const int* __restrict__ ids,
                                                      const float* __restrict__ dlasg,
                                                      const __nv_bfloat16* __restrict__ WrT, int k, int d,
                                                      __nv_bfloat16* __restrict__ dX) {
  const int t = blockIdx.x;
  // the token's contributing slots, compacted in slot order: rows with a local expert, and
  // router terms with dl != 0 (so a token with nothing to add only writes zeros)
  __shared__ int rows[kMaxK], eid[kMaxK];
  __shared__ float dl[kMaxK];
  __shared__ int nr, nd;
  if (threadIdx.x < 32) {
    const int j = threadIdx.x;
    int R = -1, e = 0;
    float w = 0.f;
    if (j < k) {
      const size_t a = static_cast<size_t>(t) * k + j;
      R = slot_row[a];
      e = ids[a];
      w = dlasg[a];
    }
    const unsigned mr = __ballot_sync(0xffffffffu, j < k && R >= 0);
    const unsigned md = __ballot_sync(0xffffffffu, j < k && w != 0.f);
    const unsigned below = (1u << j) - 1u;
    if (j < k && R >= 0) rows[__popc(mr & below)] = R;
    if (j < k && w != 0.f) {
      eid[__popc(md & below)] = e;
      dl[__popc(md & below)] = w;
    }
    if (j == 0) {
      nr = __popc(mr);
      nd = __popc(md);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x * 8; i < d; i += blockDim.x * 8) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < nr; ++j) {
      const int R = rows[j];
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(dxperm + static_cast<size_t>(R) * d + i));
      float2 f;
      f = unpack_bf16(u.x); acc[0] += f.x; acc[1] += f.y;
      f = unpack_bf16(u.y); acc[2] += f.x; acc[3] += f.y;
      f = unpack_bf16(u.z); acc[4] += f.x; acc[5] += f.y;
      f = unpack_bf16(u.w); acc[6] += f.x; acc[7] += f.y;
    }
    for (int j = 0; j < nd; ++j) {
      const float w = dl[j];
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(WrT + static_cast<size_t>(eid[j]) * d + i));
      float2 f;
      f = unpack_bf16(u.x); acc[0] = fmaf(w, f.x, acc[0]); acc[1] = fmaf(w, f.y, acc[1]);
      f = unpack_bf16(u.y); acc[2] = fmaf(w, f.x, acc[2]); acc[3] = fmaf(w, f.y, acc[3]);
      f = unpack_bf16(u.z); acc[4] = fmaf(w, f.x, acc[4]); acc[5] = fmaf(w, f.y, acc[5]);
      f = unpack_bf16(u.w); acc[6] = fmaf(w, f.x, acc[6]); acc[7] = fmaf(w, f.y, acc[7]);
    }
    uint4 o;
    o.x = pack_bf16(acc[0], acc[1]);
    o.y = pack_bf16(acc[2], acc[3]);
    o.z = pack_bf16(acc[4], acc[5]);
    o.w = pack_bf16(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(dX + static_cast<size_t>(t) * d + i) = o;
  }
}



// ---------------------------------------------------------------------------
// Ring-streamed layer planner (one thread; M minibatches, El local experts).
//
// Forward: consecutive minibatches are grouped into a macrobatch until its
// padded rows reach min_rows (the gate/up grouped GEMM then has at least two
// full waves of tiles, the MoK pages' heuristic), or until the next minibatch
// would not fit in the ring.  Each macrobatch's padded segment is placed at the
// ring's write pointer; a segment that would run past the end starts at row 0.
// Backward: macrobatches are visited in reverse.  The ones whose segment is
// still intact (no later segment overlapped it) form the first chunk and are
// reused in place; older ones are re-dispatched (replayed) into the ring in
// chunks of consecutive macrobatches that fit in it together.
// ---------------------------------------------------------------------------
__global__ void k_plan(const int* __restrict__ base, const int* __restrict__ counts, int nblk_per_mb, int nblk, int M,
                       int E, int first, int El, int ring_rows, int min_rows, StreamTables tb) {
  __shared__ int open_cnt[kMaxE];  // assignments per expert in the macrobatch being formed
  __shared__ int tot_cnt[kMaxE];   // assignments per expert in the macrobatches already formed
  __shared__ int resident[kMaxMinibatches];
  if (threadIdx.x != 0) return;
  for (int el = 0; el < El; ++el) open_cnt[el] = tot_cnt[el] = 0;
  // count of local expert el in minibatch b: difference of the block-level exclusive scans
  auto mb_count = [&](int b, int el) {
    const int e = first + el;
    const int b1 = (b + 1) * nblk_per_mb;
    const int hi = b1 >= nblk ? counts[e] : base[static_cast<size_t>(b1) * E + e];
    return hi - base[static_cast<size_t>(b * nblk_per_mb) * E + e];
  };
  auto padded = [](int c) { return (c + kPad - 1) / kPad * kPad; };
  int row = 0, wp = 0, nm = 0, b0 = 0;
  auto emit = [&](int b_end) {  // close the open macrobatch = minibatches [b0, b_end)
    const int start = row;
    for (int el = 0; el < El; ++el) {
      const int sg = nm * El + el;
      tb.seg_poff[sg] = row;
      tb.cum[sg] = tot_cnt[el];
      row += padded(open_cnt[el]);
      tot_cnt[el] += open_cnt[el];
      open_cnt[el] = 0;
    }
    const int size = row - start;
    if (wp + size > ring_rows) wp = 0;  // would straddle the end: restart at row 0
    tb.ring_start[nm] = wp;
    tb.shift_fwd[nm] = wp - start;
    wp += size;
    tb.mb_range[2 * nm] = b0;
    tb.mb_range[2 * nm + 1] = b_end;
    ++nm;
    b0 = b_end;
  };
  for (int b = 0; b < M; ++b) {
    if (b > b0) {  // does minibatch b still fit in the ring with the open macrobatch?
      int with_b = 0;
      for (int el = 0; el < El; ++el) with_b += padded(open_cnt[el] + mb_count(b, el));
      if (with_b > ring_rows) emit(b);
    }
    int rows_now = 0;
    for (int el = 0; el < El; ++el) {
      open_cnt[el] += mb_count(b, el);
      rows_now += padded(open_cnt[el]);
    }
    tb.mb_of[b] = nm;
    if (rows_now >= min_rows) emit(b + 1);  // two full waves of gate/up tiles
  }
  if (b0 < M) emit(M);
  for (int m = nm; m < M; ++m) {  // macrobatches not formed: empty segments at the end
    for (int el = 0; el < El; ++el) {
      tb.seg_poff[m * El + el] = row;
      tb.cum[m * El + el] = tot_cnt[el];
    }
    tb.mb_range[2 * m] = tb.mb_range[2 * m + 1] = M;
    tb.shift_fwd[m] = tb.shift_bwd[m] = tb.ring_start[m] = tb.replay[m] = 0;
  }
  tb.seg_poff[M * El] = row;

  // residency after the forward: no later segment overlaps this one in the ring
  auto seg_rows = [&](int m) { return tb.seg_poff[(m + 1) * El] - tb.seg_poff[m * El]; };
  for (int m = 0; m < nm; ++m) {
    const int a0 = tb.ring_start[m], a1 = a0 + seg_rows(m);
    int ok = 1;
    for (int q = m + 1; q < nm && ok; ++q) {
      const int c0 = tb.ring_start[q], c1 = c0 + seg_rows(q);
      if (a1 > a0 && c1 > c0 && c0 < a1 && a0 < c1) ok = 0;
    }
    resident[m] = ok;
  }
  // backward chunks, walking the macrobatches in reverse
  int nc = 0, replayed = 0, resident_rows = 0, m = nm - 1;
  while (m >= 0 && resident[m]) {
    tb.shift_bwd[m] = tb.shift_fwd[m];
    tb.replay[m] = 0;
    resident_rows += seg_rows(m);
    --m;
  }
  if (m + 1 < nm) {
    tb.chunk[0] = m + 1;
    tb.chunk[1] = nm;
    tb.chunk[2] = 1;
    nc = 1;
  }
  while (m >= 0) {
    const int hi = m + 1;
    int rows_c = 0;
    do {
      rows_c += seg_rows(m);
      --m;
    } while (m >= 0 && rows_c + seg_rows(m) <= ring_rows);
    int pos = 0;
    for (int q = m + 1; q < hi; ++q) {
      tb.replay[q] = 1;
      tb.shift_bwd[q] = pos - tb.seg_poff[q * El];
      pos += seg_rows(q);
    }
    replayed += rows_c;
    tb.chunk[4 * nc] = m + 1;
    tb.chunk[4 * nc + 1] = hi;
    tb.chunk[4 * nc + 2] = 1;
    ++nc;
  }
  if (nc == 0) {  // no rows at all: one empty chunk still writes the (zero) gradients
    tb.chunk[0] = tb.chunk[1] = 0;
    tb.chunk[2] = 1;
    nc = 1;
  }
  for (int c = 0; c < M; ++c) {
    if (c < nc) {
      tb.chunk[4 * c + 3] = nc == 1 ? 0 : (c == 0 ? 1 : 2);
    } else {
      tb.chunk[4 * c] = tb.chunk[4 * c + 1] = tb.chunk[4 * c + 2] = tb.chunk[4 * c + 3] = 0;
    }
  }
  tb.plan[PLAN_N_MACRO] = nm;
  tb.plan[PLAN_N_CHUNKS] = nc;
  tb.plan[PLAN_ROWS] = row;
  tb.plan[PLAN_REPLAYED] = replayed;
  tb.plan[PLAN_RESIDENT] = resident_rows;
  tb.plan[PLAN_RING_ROWS] = ring_rows;
}

// Backward chunk c: re-dispatch the X rows of every macrobatch marked for replay
// into the ring at its backward position.  Resident macrobatches are left alone.
__global__ void __launch_bounds__(128) k_replay(const __nv_bfloat16* __restrict__ X, const int* __restrict__ row_asg,
                                                StreamTables tb, int El, int c, int k, int d,
                                                __nv_bfloat16* __restrict__ ring) {
  if (!tb.chunk[4 * c + 2]) return;
  const int m_lo = tb.chunk[4 * c], m_hi = tb.chunk[4 * c + 1];
  const int nv = d / 8;
  for (int m = m_lo; m < m_hi; ++m) {
    if (!tb.replay[m]) continue;
    const int r0 = tb.seg_poff[m * El], r1 = tb.seg_poff[(m + 1) * El];
    const int sh = tb.shift_bwd[m];
    for (int64_t R = r0 + blockIdx.x; R < r1; R += gridDim.x) {
      const int a = row_asg[R];
      if (a == ROW_DEAD) continue;
      uint4* out = reinterpret_cast<uint4*>(ring + (R + sh) * d);
      if (a >= 0) {
        const uint4* in = reinterpret_cast<const uint4*>(X + static_cast<size_t>(a / k) * d);
        for (int i = threadIdx.x; i < nv; i += blockDim.x) out[i] = __ldg(in + i);
      } else {
        const uint4 z = make_uint4(0, 0, 0, 0);
        for (int i = threadIdx.x; i < nv; i += blockDim.x) out[i] = z;
      }
    }
  }
}

// dW_gate / dW_up (bf16) from the fp32 accumulator when the backward used several chunks.
__device__ __forceinline__ void store4(__nv_bfloat16* dst, float4 v) {
  uint2 u;
  u.x = pack_bf16(v.x, v.y);
  u.y = pack_bf16(v.z, v.w);
  *reinterpret_cast<uint2*>(dst) = u;
}
__device__ __forceinline__ void store4(float* dst, float4 v) { *reinterpret_cast<float4*>(dst) = v; }

template <typename OutT>
__global__ void __launch_bounds__(256) k_finish_acc(const float* __restrict__ acc, const int* __restrict__ plan,
                                                    size_t n_each, OutT* __restrict__ dWg, OutT* __restrict__ dWu) {
  if (plan[PLAN_N_CHUNKS] <= 1) return;  // the wgrad epilogue already wrote the gradients
  const size_t n4 = n_each / 4;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < 2 * n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(acc)[i];
    store4(i < n4 ? dWg + 4 * i : dWu + 4 * (i - n4), v);
  }
}

// local views of the routing table for the test hook
__global__ void k_export_routing(const int* __restrict__ counts, const int* __restrict__ offsets,
                                 const int* __restrict__ poff, const int* __restrict__ perm_tok, int first, int El,
                                 int32_t* o_counts, int32_t* o_offsets, int32_t* o_poff, int32_t* o_perm) {
  const int base = offsets[first];
  const int n = offsets[first + El] - base;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i <= El || i < n; i += gridDim.x * blockDim.x) {
    if (i < El && o_counts) o_counts[i] = counts[first + i];
    if (i <= El && o_offsets) o_offsets[i] = offsets[first + i] - base;
    if (i <= El && o_poff) o_poff[i] = poff[i];
    if (i < n && o_perm) o_perm[i] = perm_tok[base + i];
  }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
cudaError_t launch_topk(const Layout& L, const Ctx& c, const float* bias, int splits, cudaStream_t st) {
  const int T = static_cast<int>(L.T);
  if (L.E <= 128)
    k_topk<4><<<L.nblk, kTokensPerBlock * 32, 0, st>>>(c.rpart, splits, bias, c.logits, T, L.E, L.k, c.ids, c.gates,
                                                       c.hist, c.hdr + HDR_STATUS);
  else if (L.E <= 256)
    k_topk<8><<<L.nblk, kTokensPerBlock * 32, 0, st>>>(c.rpart, splits, bias, c.logits, T, L.E, L.k, c.ids, c.gates,
                                                       c.hist, c.hdr + HDR_STATUS);
  else if (L.E <= 384)
    k_topk<12><<<L.nblk, kTokensPerBlock * 32, 0, st>>>(c.rpart, splits, bias, c.logits, T, L.E, L.k, c.ids,
                                                        c.gates, c.hist, c.hdr + HDR_STATUS);
  else
    k_topk<kMaxE / 32><<<L.nblk, kTokensPerBlock * 32, 0, st>>>(c.rpart, splits, bias, c.logits, T, L.E, L.k, c.ids,
                                                                c.gates, c.hist, c.hdr + HDR_STATUS);
  return cudaGetLastError();
}
cudaError_t preload_router_kernels() {
  cudaFuncAttributes a;
  cudaError_t e = cudaSuccess;
  if (e == cudaSuccess) e = cudaFuncGetAttributes(&a, k_transpose_wr);
  if (e == cudaSuccess) e = cudaFuncGetAttributes(&a, k_transpose_wr_v);
  if (e == cudaSuccess) e = cudaFuncGetAttributes(&a, k_topk<4>);
  if (e == cudaSuccess) e = cudaFuncGetAttributes(&a, k_topk<8>);
  if (e == cudaSuccess) e = cudaFuncGetAttributes(&a, k_topk<12>);
  if (e == cudaSuccess) e = cudaFuncGetAttributes(&a, k_topk<kMaxE / 32>);
  return e;
}
cudaError_t launch_scan(const Layout& L, const Ctx& c, cudaStream_t st) {
  // over the group sums when the scan is two-level (launch_scan_groups before, _apply after)
  k_scan<<<1, 1024, 0, st>>>(L.scan_groups ? c.hsum : c.hist, L.scan_groups ? L.scan_groups : L.nblk, L.E, L.first,
                             L.El, c.counts, c.offsets, c.poff, c.hdr);
  return cudaGetLastError();
}
cudaError_t launch_scan_groups(const Layout& L, const Ctx& c, cudaStream_t st) {
  k_scan_group_sums<<<L.scan_groups, 512, 0, st>>>(c.hist, L.nblk, L.E, c.hsum);
  return cudaGetLastError();
}
cudaError_t launch_scan_apply(const Layout& L, const Ctx& c, cudaStream_t st) {
  k_scan_group_apply<<<L.scan_groups, 512, 0, st>>>(c.hist, L.nblk, L.E, c.hsum);
  return cudaGetLastError();
}
cudaError_t launch_scatter(const Layout& L, const Ctx& c, cudaStream_t st) {
  const bool streamed = L.M > 0;
  k_scatter<<<L.nblk, 32, 0, st>>>(c.ids, c.gates, c.hist, c.offsets, streamed ? c.tab.seg_poff : c.poff,
                                   static_cast<int>(L.T), L.E, L.k, L.first, L.El, static_cast<int>(L.T_mb),
                                   streamed ? c.tab.mb_of : nullptr, streamed ? c.tab.cum : nullptr, c.perm_tok,
                                   c.perm_asg, c.slot_row, c.row_asg, c.row_gate);
  return cudaGetLastError();
}
// One thread waits on an mbarrier that nothing arrives at: the bounded wait gives up and
// records MOE_ERR_DEVICE_TIMEOUT in *status (the failure path of every GEMM role).
__global__ void k_wait_probe(int* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbar_init();
  mbar_wait(&bar, 0, status);
}
cudaError_t launch_wait_probe(int* status, cudaStream_t st) {
  k_wait_probe<<<1, 32, 0, st>>>(status);
  return cudaGetLastError();
}
cudaError_t launch_mark_rows(const Layout& L, const Ctx& c, cudaStream_t st) {
  const bool mb = L.M > 0;
  const int nseg = mb ? L.M * L.El : L.El;
  k_mark_rows<<<nseg, 128, 0, st>>>(mb ? c.tab.seg_poff : c.poff, nseg, L.El, c.counts + L.first,
                                    mb ? c.tab.cum : nullptr, mb ? L.M : 1, c.row_asg, c.row_gate);
  return cudaGetLastError();
}
cudaError_t launch_gather_range(const Layout& L, const Ctx& c, const __nv_bfloat16* src, const int* lo, const int* hi,
                                const int* shift, int64_t max_rows, __nv_bfloat16* dst, cudaStream_t st) {
  const int grid = static_cast<int>(max_rows < 148 * 16 ? (max_rows > 0 ? max_rows : 1) : 148 * 16);
  k_gather_rows<<<grid, 128, 0, st>>>(src, c.row_asg, lo, hi, shift, L.k, L.d, dst);
  return cudaGetLastError();
}
cudaError_t launch_gather_rows(const Layout& L, const Ctx& c, const __nv_bfloat16* src, __nv_bfloat16* dst,
                               cudaStream_t st) {
  if (L.M > 0)  // all rows of the stream
    return launch_gather_range(L, c, src, c.tab.seg_poff, c.tab.seg_poff + L.M * L.El, nullptr, L.RP, dst, st);
  return launch_gather_range(L, c, src, c.poff, c.poff + L.El, nullptr, L.RP, dst, st);
}
cudaError_t launch_combine(const Layout& L, const Ctx& c, const __nv_bfloat16* Oprime, __nv_bfloat16* Y,
                           cudaStream_t st, const int* mb_range) {
  const int64_t n = mb_range ? L.T_mb * L.M : L.T;
  const int grid = static_cast<int>(n < 148 * 16 ? (n > 0 ? n : 1) : 148 * 16);
  k_combine<<<grid, 128, 0, st>>>(Oprime, c.slot_row, L.k, L.d, static_cast<int>(L.T), mb_range,
                                  static_cast<int>(L.T_mb), Y);
  return cudaGetLastError();
}
cudaError_t launch_plan(const Layout& L, const Ctx& c, int ring_rows, int min_rows, cudaStream_t st) {
  k_plan<<<1, 32, 0, st>>>(c.hist, c.counts, static_cast<int>(L.T_mb / kTokensPerBlock), L.nblk, L.M, L.E, L.first,
                           L.El, ring_rows, min_rows, c.tab);
  return cudaGetLastError();
}
cudaError_t launch_replay(const Layout& L, const Ctx& c, int chunk, const __nv_bfloat16* X, __nv_bfloat16* ring,
                          int64_t ring_rows, cudaStream_t st) {
  const int grid = static_cast<int>(ring_rows < 148 * 16 ? ring_rows : 148 * 16);
  k_replay<<<grid, 128, 0, st>>>(X, c.row_asg, c.tab, L.El, chunk, L.k, L.d, ring);
  return cudaGetLastError();
}
cudaError_t launch_finish_acc(const Layout& L, const Ctx& c, void* dW_gate, void* dW_up, cudaStream_t st) {
  const size_t n_each = static_cast<size_t>(L.El) * L.d * L.I;
  if (L.w32)
    k_finish_acc<<<148 * 8, 256, 0, st>>>(c.acc32, c.tab.plan, n_each, static_cast<float*>(dW_gate),
                                          static_cast<float*>(dW_up));
  else
    k_finish_acc<<<148 * 8, 256, 0, st>>>(c.acc32, c.tab.plan, n_each, static_cast<__nv_bfloat16*>(dW_gate),
                                          static_cast<__nv_bfloat16*>(dW_up));
  return cudaGetLastError();
}
cudaError_t launch_active_count(const Layout& L, const Ctx& c, cudaStream_t st) {
  const int nb = static_cast<int>((L.T + kActBlock - 1) / kActBlock);
  k_active_count<<<nb, kActBlock, 0, st>>>(c.slot_row, static_cast<int>(L.T), L.k, c.actcnt);
  return cudaGetLastError();
}
cudaError_t launch_gather_active(const Layout& L, const Ctx& c, const __nv_bfloat16* X, cudaStream_t st) {
  const int nb = static_cast<int>((L.T + kActBlock - 1) / kActBlock);
  const int64_t Tpad = (L.T + 63) / 64 * 64;
  const int64_t g = (Tpad + 7) / 8;
  const int grid = static_cast<int>(g < 148 * 8 ? g : 148 * 8);
  k_gather_active<<<grid, 256, 0, st>>>(X, L.d, c.actlist, c.actcnt + nb, Tpad, c.xact);
  return cudaGetLastError();
}
cudaError_t launch_router_bwd(const Layout& L, const Ctx& c, cudaStream_t st, int n_tiles_i) {
  // n_tiles_i: dg partials per row = n-tiles of the dgrad-down GEMM (I / 256 bf16, I / 128 MXFP8)
  const int E64 = (L.E + 63) / 64 * 64;
  const int Tpad = static_cast<int>((L.T + 63) / 64 * 64);
  if (L.rslice) {  // expert slice: DL rows of the listed tokens only (launch_active_count first)
    const int nb = static_cast<int>((L.T + kActBlock - 1) / kActBlock);
    k_router_bwd_compact<<<nb, kActBlock, 0, st>>>(c.dgpart, c.slot_row, c.gates, c.ids, static_cast<int>(L.T), Tpad,
                                                   L.k, n_tiles_i ? n_tiles_i : L.I / 256, E64, c.actcnt, nb,
                                                   c.dlasg, c.dldense, c.actlist);
    return cudaGetLastError();
  }
  k_router_bwd<<<static_cast<unsigned>(Tpad / 8), 256, 0, st>>>(c.dgpart, c.slot_row, c.gates, c.ids,
                                                                 static_cast<int>(L.T), Tpad, L.k,
                                                                 n_tiles_i ? n_tiles_i : L.I / 256, E64, c.dlasg,
                                                                 c.dldense);
  return cudaGetLastError();
}
cudaError_t launch_transpose_wr(const Layout& L, const __nv_bfloat16* W_r, __nv_bfloat16* W_rT, cudaStream_t st) {
  if (L.E % 8 == 0 && L.d % 64 == 0) {
    k_transpose_wr_v<<<dim3((L.E + 63) / 64, L.d / 64), 256, 0, st>>>(W_r, L.d, L.E, W_rT);
  } else {
    dim3 grid((L.E + 31) / 32, (L.d + 31) / 32);
    k_transpose_wr<<<grid, 256, 0, st>>>(W_r, L.d, L.E, W_rT);
  }
  return cudaGetLastError();
}
cudaError_t launch_rev_dispatch(const Layout& L, const Ctx& c, __nv_bfloat16* dX, cudaStream_t st) {
  k_rev_dispatch<<<static_cast<unsigned>(L.T), 128, 0, st>>>(c.dxperm, c.slot_row, c.ids, c.dlasg, c.wrt, L.k, L.d,
                                                              dX);
  return cudaGetLastError();
}
cudaError_t launch_export_routing(const Layout& L, const Ctx& c, int32_t* counts, int32_t* offsets, int32_t* poff,
                                  int32_t* perm, cudaStream_t st) {
  const int64_t n = L.T * L.k + L.El + 1;
  const int grid = static_cast<int>((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024);
  k_export_routing<<<grid, 256, 0, st>>>(c.counts, c.offsets, c.poff, c.perm_tok, L.first, L.El, counts, offsets,
                                         poff, perm);
  return cudaGetLastError();
}

}  // namespace moe
