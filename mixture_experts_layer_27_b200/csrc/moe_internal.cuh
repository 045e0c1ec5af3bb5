// Internal declarations shared by the translation units of libmoe.so:
// the context / workspace layout, the GEMM parameter block and the kernel
// launchers.  Nothing here is part of the public ABI.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "moe.h"

namespace moe {

constexpr int kPad = 128;          // rows of an expert segment are padded to a multiple of this
constexpr int kTokensPerBlock = 16;  // tokens per block of the top-k / scatter kernels
constexpr int kScanGroup = 32;       // histogram rows per group of the two-level expert scan
constexpr int kScanOneLevel = 256;   // up to this many token blocks the scan is one block
constexpr int kMaxE = 512;
constexpr int kMaxK = 16;
constexpr int kMaxMinibatches = 256;  // ring-streamed layer

// ctx header words (int32)
enum HdrWord { HDR_STATUS = 0, HDR_ROWS_P = 1, HDR_MTILES = 2, HDR_WORDS = 64 };

// Plan of a ring-streamed layer (M minibatches grouped into macrobatches), written on
// the device by k_plan and read by every per-macrobatch / per-chunk launch.
enum PlanWord {
  PLAN_N_MACRO = 0,   // macrobatches formed
  PLAN_N_CHUNKS = 1,  // backward wgrad chunks
  PLAN_ROWS = 2,      // padded rows of the whole stream
  PLAN_REPLAYED = 3,  // padded rows re-dispatched in the backward
  PLAN_RESIDENT = 4,  // padded rows the backward found still in the ring
  PLAN_RING_ROWS = 5, // ring capacity in rows
  PLAN_WORDS = 16
};
// Pad rows of an expert segment (its real rows are a prefix): the first ones, up to the next
// multiple of 16 rows, are ROW_PAD, written as zero rows by every producer because the weight
// gradients' last K16 step reads them; the rest are ROW_DEAD, never written and never read.
constexpr int ROW_PAD = -1;
constexpr int ROW_DEAD = -2;

struct StreamTables {
  int* plan;       // [PLAN_WORDS]
  int* mb_of;      // [M]        macrobatch of each minibatch
  int* seg_poff;   // [M*El+1]   padded row where segment (m, el) starts
  int* cum;        // [M*El]     assignments to el in macrobatches before m
  int* mb_range;   // [2M]       minibatches [begin, end) of macrobatch m
  int* shift_fwd;  // [M]        ring row - padded row, forward placement
  int* shift_bwd;  // [M]        ring row - padded row, backward placement
  int* replay;     // [M]        1 if the backward re-dispatches macrobatch m
  int* chunk;      // [4M]       backward chunk c: {m_lo, m_hi, valid, mode}
  int* ring_start; // [M]        forward ring row of macrobatch m
};
constexpr int stream_table_words(int M, int El) { return PLAN_WORDS + M + (M * El + 1) + M * El + 2 * M + 4 * M + 4 * M; }

// Byte offsets of every region of ctx (saved for backward) and ws (scratch).
struct Layout {
  // shape
  int64_t T;
  int d, E, I, k, first, El;
  int64_t RP;     // padded-row capacity: worst case of sum_e ceil(count_e / 128) * 128
  int nblk;       // blocks of the top-k / scatter kernels
  int scan_groups;  // groups of the two-level expert scan (0: one level)
  int M;          // minibatches of a ring-streamed layer (0: one call = one batch)
  int64_t T_mb;   // tokens per minibatch (streamed layer)
  // ctx
  size_t hdr, ids, gates, counts, offsets, poff, perm_tok, perm_asg, slot_row, row_asg, row_gate, xperm, abuf,
      bbuf, stab, xq, xqs, ctx_bytes;
  // ws
  size_t hist, hsum, logits, rpart, hbuf, obuf, dyperm, dabuf, dbbuf, hgbuf, dgpart, dlasg, dldense, wrt, dxperm, acc32, hq, hqs, dyq,
      dyqs, daq, daqs, dbq, dbqs, actcnt, actlist, xact, fctl, ws_bytes;
  // MXFP8 weight gradients: X, dY, dA, dB, Hg quantised along the rows, K-major in 128-row tiles
  // (rowq_index in ptx.cuh) with their scale chunks
  size_t xqt, xqts, dyqt, dyqts, daqt, daqts, dbqt, dbqts, hgqt, hgqts;
  bool mx;   // MXFP8 mode
  bool mxw;  // MXFP8 mode with the weight-gradient GEMMs on MXFP8 as well
  bool w32;  // expert weight gradients written as fp32
  bool rslice;  // an expert slice (El < E): the router weight gradient runs over the listed tokens
  bool nv;      // NVFP4 (moe_fwd_nvfp4 / moe_bwd_nvfp4): xq / xqs, hq / hqs, dyq / dyqs, daq / daqs,
                // dbq / dbqs hold E2M1 codes (two per byte) and E4M3 scale chunks (nv_sf_index); nvh the
                // gate/up GEMM's fp32 H [RP, I], nvdab the dgrad of W_down's fp32 dA, dB; nvsc eight
                // words: amax X, H, dY, [dA | dB] (fp32 bits) and their global scales, in the order
                // amax X, amax H, gs X, gs H, amax dY, amax dAB, gs dY, gs dAB; the prepared weights are
                // the five MXFP8 layouts in NVFP4 and the global scales gate, up, down, [gate | up]
                // (wnvgs, then four amax words at +64)
  size_t nvh, nvsc, wnvgs, nvdab;
  // prepared MXFP8 weights (moe_prepare_weights): fp8 codes and scale chunks
  size_t wgu1, wgu1s, wd2, wd2s, wd3, wd3s, wg4, wg4s, wu4, wu4s, wq_bytes;
};

// Returns false for shapes outside the supported limits.  M > 0: a ring-streamed
// layer of M minibatches of s.T tokens (X_perm lives in the caller's ring).
bool make_layout(const moe_shape& s, Layout* L, int M = 0);

// ---------------------------------------------------------------------------
// grouped GEMM (tcgen05 + TMA), see gemm.cu
// ---------------------------------------------------------------------------
enum GemmKind {
  G_GATEUP = 0,         // [A|B] = X_perm . [W_gate | W_up], SwiGLU epilogue -> A, B, H
  G_DOWN = 1,           // O' = g * (H . W_down)
  G_DGRAD_DOWN = 2,     // dH' = dY_perm . W_down^T, SwiGLU-backward + router-grad epilogue
  G_DGRAD_GATEUP = 3,   // dX_perm = dA . W_gate^T + dB . W_up^T
  G_WGRAD_GATEUP = 4,   // dW_gate = X_perm^T dA, dW_up = X_perm^T dB (per expert)
  G_WGRAD_DOWN = 5,     // dW_down = Hg^T dY_perm (per expert)
  G_ROUTER = 6,         // router logits partials: part[s] = X[:, Ks] . W_r[Ks, :] (fixed K split s)
  G_ROUTER_WGRAD = 7,   // dW_r = X^T . DL_hi + X^T . DL_lo, DL = dl as a dense [T, E] matrix in two bf16 terms
};

struct GemmParams {
  CUtensorMap ta0, ta1, tb0, tb1;  // operand maps
  CUtensorMap to0, to1;            // output maps (TMA stores of the wgrad epilogues)
  CUtensorMap tacc;                // fp32 wgrad accumulator map (ring-streamed backward, several chunks)
  const int* hdr;             // ctx header
  // Padded row space: nseg segments (macrobatch m, local expert el) = m * El + el,
  // segment s covers rows [poff[s], poff[s+1]).  One macrobatch: nseg = El.
  const int* poff;
  int nseg;
  const int* ring_shift;      // per macrobatch: ring row - padded row of X_perm (NULL: X_perm not in a ring)
  const int* chunk;           // wgrad gate/up over a chunk of macrobatches: {m_lo, m_hi, valid, mode}; NULL = all
  // Real (unpadded) rows of a segment, a prefix of it: cnt[el] for one batch; with a ring
  // stream cum[m*El+el] counts el's rows in macrobatches before m (cnt[el] = the total).
  const int* cnt;
  const int* cum;
  float* acc32;               // fp32 accumulator for dW_gate / dW_up when a backward needs several chunks
  const float* row_gate;      // [RP]
  const int* row_asg;         // [RP] assignment of each padded row, ROW_PAD / ROW_DEAD for pad rows
  const __nv_bfloat16* in0;   // epilogue inputs
  const __nv_bfloat16* in1;
  __nv_bfloat16* out0;        // epilogue outputs
  __nv_bfloat16* out1;
  __nv_bfloat16* out2;
  float* outf;
  int El, d, I;
  int T, E, splits;           // router GEMM: tokens, experts, K splits
  int router_bn;              // router GEMM: experts per n-tile (E split evenly over ceil(E / 256) tiles)
  int wout32;                 // wgrad: to0 / to1 are fp32 maps (32 x 32 boxes) and take the unrounded sums
  const int* act_n;           // router wgrad over listed tokens: their number (device); NULL = all T tokens
  int* status;
};

constexpr int GEMM_BM = 128, GEMM_BN = 256, GEMM_BK = 64, GEMM_STAGES = 4;
constexpr int GEMM_THREADS = 192;        // six role warps: producer, MMA issuer, four epilogue warps
constexpr int GEMM_THREADS_SCHED = 224;  // the same plus a tile scheduler warp
constexpr size_t GEMM_A_BYTES = GEMM_BM * GEMM_BK * 2;
constexpr size_t GEMM_B_BYTES = GEMM_BN * GEMM_BK * 2;
constexpr size_t GEMM_STAGE_BYTES = GEMM_A_BYTES + GEMM_B_BYTES;
constexpr size_t GEMM_STAGE_OUT_BYTES = 4 * 32 * 256 * 2;  // wgrad: one 32 x 256 bf16 slice per epilogue warp
// experts per n-tile of the router GEMM: E split evenly over ceil(E / 256) tiles, rounded up to
// the MMA's N granule (16), so that E = 384 runs as two 192-wide tiles instead of 256 + 128
constexpr int router_tile_n(int E) { return ((E + (E + 255) / 256 - 1) / ((E + 255) / 256) + 15) / 16 * 16; }
constexpr int router_splits(int64_t T, int E, int d) {  // K splits of the router GEMM (about one wave)
  const int64_t tiles = ((T + 127) / 128) * ((E + 255) / 256);
  int64_t s = tiles > 0 ? 148 / tiles : 1;
  if (s < 1) s = 1;
  if (s > d / 64) s = d / 64;
  return static_cast<int>(s);
}

// sched: the weight-gradient kinds can decode their tiles in a scheduler warp ahead of the
// roles (worth it when tiles have few K blocks and the epilogue is the critical path); other
// kinds ignore it.
cudaError_t launch_gemm(GemmKind kind, const GemmParams& p, int grid, cudaStream_t st, bool sched = false);
// Loads the kernel of one GEMM kind (and sets its shared-memory attribute) without launching it,
// so that a later launch needs no lazy module loading.
cudaError_t preload_gemm(GemmKind kind);

// Two dependent grouped GEMMs in one persistent launch (gemm.cu): every tile of the first,
// then every tile of the second, as work units that CTAs take from one ticket counter in one
// global order, CTAs that have not started claimed through Cluster Launch Control.  A tile of
// the second GEMM waits (bounded) until every tile of the first has stored its 128 rows.
enum GemmPair {
  PAIR_FWD = 0,    // G_GATEUP then G_DOWN (reads H)
  PAIR_DGRAD = 1,  // G_DGRAD_DOWN then G_DGRAD_GATEUP (reads dA, dB)
};
struct GemmPairParams {
  GemmParams p1;  // the first GEMM's parameters, as for launch_gemm
  GemmParams p2;  // the second GEMM's parameters
  int* ctl;       // gemm_pair_ctl_words(RP) ints, zero before the launch
  int mt_cap;     // m-tile capacity of ctl (RP / 128)
  int skip_first; // test hook: the first GEMM's tiles are not run, so the second GEMM's tiles wait
                  // for rows that nobody writes until their bounded wait gives up
};
constexpr int64_t gemm_pair_ctl_words(int64_t RP) { return 1 + RP / 128; }
// Upper bound of the work units (both GEMMs' tiles at RP rows).
int64_t gemm_pair_units(GemmPair pair, int64_t RP, int d, int I);
cudaError_t launch_gemm_pair(GemmPair pair, const GemmPairParams& p, int64_t grid, cudaStream_t st);

// 2-D bf16 tensor map [outer, inner] (inner contiguous, row pitch in elements), box
// {box_inner, box_outer}, 128-byte swizzle, zero fill out of bounds (moe_api.cu).
bool tmap_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t pitch_elems,
             uint32_t box_inner, uint32_t box_outer);
// Router GEMM: the fp32 partial logits of its router_splits() fixed K splits into rpart
// [splits, T, E], from X [T, d] and W_r^T [E, d] (moe_api.cu).  Shared by moe_fwd and the
// allocation-free router entry point, so both run the same tiles in the same order.
cudaError_t launch_router_logits(const Layout& L, const void* X, const __nv_bfloat16* wrt, float* rpart, int* status,
                                 cudaStream_t st);

// ---------------------------------------------------------------------------
// MXFP8 grouped GEMMs (tcgen05 kind::mxf8f6f4 block_scale), see gemm_mx.cu
// ---------------------------------------------------------------------------
enum MxKind {
  MX_GATEUP = 0,        // [A|B] = Xq . [Wg|Wu]q (2 x (64 gate + 64 up) columns per tile); H quantised in the epilogue
  MX_DOWN = 1,          // O' = g * (Hq . Wd_q)
  MX_DGRAD_DOWN = 2,    // dH' = dYq . Wd_q^T; SwiGLU backward; dA, dB quantised in the epilogue
  MX_DGRAD_GATEUP = 3,  // dX_perm = dAq . Wg_q^T + dBq . Wu_q^T
  MX_WGRAD_GATEUP = 4,  // dW_gate = Xq^T dAq, dW_up = Xq^T dBq per expert, all quantised along its rows
  MX_WGRAD_DOWN = 5,    // dW_down = Hgq^T dYq per expert
  NV_GATEUP = 6,        // NVFP4 (kind::mxf4nvf4): H = silu(A) B from Xq . [Wg|Wu]q, fp32 H and its amax out
  NV_DOWN = 7,          // NVFP4: O' = g * (Hq . Wd_q)
  NV_DGRAD_DOWN = 8,    // NVFP4: dH' = dYq . Wd_q^T; SwiGLU backward; bf16 dA, dB, Hg and fp32 dA, dB (+ amax) out
  NV_DGRAD_GATEUP = 9,  // NVFP4: dX_perm = [dA | dB]q . [Wg | Wu]q^T (K = 2I, one global scale per operand)
};
struct MxParams {
  CUtensorMap ta0, ta1, tb0, tb1;  // fp8 K-major operands, box {128 bytes of K, 128 rows (A) / mx_bn rows (B)}
  const uint8_t* sfa0;             // scale chunks of the A operands (K = the GEMM's contraction)
  const uint8_t* sfa1;
  const uint8_t* sfb0;             // scale chunks of the B operands
  const uint8_t* sfb1;
  const int* poff;                 // padded expert offsets [nseg+1]
  int nseg;
  const float* row_gate;
  const int* row_asg;              // assignment of each padded row, ROW_PAD / ROW_DEAD for pad rows
  const __nv_bfloat16* in0;        // dgrad-down epilogue: saved A, B
  const __nv_bfloat16* in1;
  __nv_bfloat16* out0;
  __nv_bfloat16* out1;
  __nv_bfloat16* out2;
  uint8_t* q0;                     // fp8 epilogue outputs and their scale chunks
  uint8_t* q1;
  uint8_t* qs0;
  uint8_t* qs1;
  float* outf;
  int El, d, I;
  int* status;
  // weight-gradient kinds: operands quantised along the rows (K = rows; rowq layout), the
  // real row count of each local expert, and the gradient outputs as TMA store maps (bf16
  // 64 x 32 boxes, or fp32 32 x 32 boxes with wout32)
  CUtensorMap to0, to1;
  const int* cnt;
  const int* cum;  // ring-streamed layer: real rows of local expert el before segment (m, el), [nseg];
                   // NULL: one segment per expert (nseg = El)
  int wout32;
  // dgrad of W_down with MXFP8 weight gradients: dA, dB and Hg also quantised along the rows,
  // from the fp32 epilogue values, into the rowq layout (C = I) and its scale chunks (the
  // bf16 dA, dB, Hg are then not written: out0..out2 NULL)
  uint8_t* tq[3];
  uint8_t* tqs[3];
  // gate/up GEMM of a ring-streamed macrobatch: the A operand's codes and scale chunks sit at ring
  // row = padded row + *ring_shift (a multiple of 128); NULL: at the padded row
  const int* ring_shift;
  // NVFP4 kinds: global scales of the A operand and of the B operand(s) (gate, up), and the gate/up
  // GEMM's fp32 H with the running amax of |H| (fp32 bits, atomicMax)
  const float* gsa;
  const float* gsb;
  float* hout;
  unsigned* amax;
  float* hout2;  // NV_DGRAD_DOWN: fp32 dB beside hout's fp32 dA
};
__host__ __device__ constexpr bool mx_is_wgrad(int kind) { return kind == MX_WGRAD_GATEUP || kind == MX_WGRAD_DOWN; }
__host__ __device__ constexpr bool mx_is_nv(int kind) {
  return kind == NV_GATEUP || kind == NV_DOWN || kind == NV_DGRAD_DOWN || kind == NV_DGRAD_GATEUP;
}
// Tile width per kind: 128 x 256 tiles (one accumulator, four stages) keep 32 KB of fp8 weights
// per stage in flight; the dgrad of W_down, whose epilogue reads and writes the most, keeps
// 128 x 128 tiles with two accumulators (six stages) so that its epilogue overlaps the MMAs.
// A stage = A tile (128 rows x 128 bytes of K), B tile (BN rows), the A scale chunk and BN/128
// B scale chunks; stages start on 1 KB boundaries (128-byte swizzle atoms).
__host__ __device__ constexpr int mx_bn(int kind) { return kind == MX_DGRAD_DOWN || kind == NV_DGRAD_DOWN ? 128 : 256; }
__host__ __device__ constexpr int mx_accs(int kind) { return mx_bn(kind) == 128 ? 2 : 1; }
// (NVFP4 128 x 128: five stages, its 36 KB stages carrying four scale chunks per operand)
__host__ __device__ constexpr int mx_stages(int kind) {
  return mx_bn(kind) == 128 ? (mx_is_nv(kind) ? 5 : 6) : (mx_is_wgrad(kind) ? 3 : 4);
}
// Epilogue warps: with one accumulator the MMAs of the next tile wait for the epilogue, so it is
// split over eight warps (two per TMEM lane quarter, each taking half of the columns); the
// double-buffered 128 x 128 kind keeps four.
__host__ __device__ constexpr int mx_epi_warps(int kind) { return mx_accs(kind) == 1 ? 8 : 4; }
__host__ __device__ constexpr int mx_threads(int kind) { return 64 + 32 * mx_epi_warps(kind); }
constexpr size_t MX_A_BYTES = 128 * 128;
__host__ __device__ constexpr size_t mx_stage_tx(int kind) {  // bytes one stage receives
  // NVFP4: a 128-byte K slice is 256 values, four 64-deep scale chunks per 128 rows
  return MX_A_BYTES + static_cast<size_t>(mx_bn(kind)) * 128 + 512 * (1 + mx_bn(kind) / 128) * (mx_is_nv(kind) ? 4 : 1);
}
__host__ __device__ constexpr size_t mx_stage_bytes(int kind) { return (mx_stage_tx(kind) + 1023) / 1024 * 1024; }
// weight-gradient kinds: 8 KB per epilogue warp stages its two gradient boxes for the TMA stores;
// the dgrad of W_down: 32 x 33 fp32 words per epilogue warp transpose its 32 x 32 value blocks
constexpr size_t MX_STAGE_OUT_BYTES = 8 * 8192;
__host__ __device__ constexpr size_t mx_out_bytes(int kind) {
  return mx_is_wgrad(kind) ? MX_STAGE_OUT_BYTES : (kind == MX_DGRAD_DOWN ? 4 * 32 * 33 * 4 : 0);
}
__host__ __device__ constexpr size_t mx_smem_bytes(int kind) {
  return mx_stages(kind) * mx_stage_bytes(kind) + mx_out_bytes(kind) + 1024 + 256;
}
constexpr int MX_MAX_STAGES = 6;
cudaError_t launch_gemm_mx(MxKind kind, const MxParams& p, int grid, cudaStream_t st);

// ---------------------------------------------------------------------------
// routing / permutation kernels, see routing.cu
// ---------------------------------------------------------------------------
struct Ctx {  // typed views of ctx + ws for one shape
  int* hdr;
  int *ids, *counts, *offsets, *poff, *perm_tok, *perm_asg, *slot_row, *row_asg;
  float *gates, *row_gate;
  __nv_bfloat16 *xperm, *abuf, *bbuf;
  int* hist;
  int* hsum;  // two-level scan: per group and expert, the group's sum, then its exclusive prefix
  float* logits;
  float* rpart;  // router split-K partials [splits, T, E]
  __nv_bfloat16 *hbuf, *obuf, *dyperm, *dabuf, *dbbuf, *hgbuf, *wrt, *dxperm;
  float *dgpart, *dlasg;
  __nv_bfloat16* dldense;  // [2, Tpad, E64] bf16 (Tpad, E64: T, E rounded up to 64): dl at (token, expert) as
                           // hi and lo bf16 terms, zeros elsewhere
  float* acc32;
  int* actcnt;               // expert slice: token counts per 256-token block, then the list length
  int* actlist;              // expert slice: the tokens with a local assignment, ascending
  __nv_bfloat16* xact;       // expert slice: their X rows [Tpad, d] (rows past the list up to a multiple of 64: 0)
  int* fctl;                 // control block of a persistent GEMM pair (gemm_pair_ctl_words(RP) ints)
  StreamTables tab;
  uint8_t *xq, *xqs, *hq, *hqs, *dyq, *dyqs, *daq, *daqs, *dbq, *dbqs;  // MXFP8 operands and scales
  uint8_t *xqt, *xqts, *dyqt, *dyqts, *daqt, *daqts, *dbqt, *dbqts, *hgqt, *hgqts;  // MXFP8 weight-gradient operands
  float* nvh;       // NVFP4 forward: fp32 H [RP, I]
  float* nvdab;     // NVFP4 backward: fp32 dA, then dB [2, RP, I]
  unsigned* nvsc;   // NVFP4 forward: amax(X), amax(H) (fp32 bits), gs_X, gs_H (fp32)
};
Ctx make_ctx(const Layout& L, void* ctx, void* ws);

cudaError_t launch_topk(const Layout& L, const Ctx& c, const float* bias, int splits, cudaStream_t st);
// Loads the W_r transpose and top-k kernels without launching them (see preload_gemm).
cudaError_t preload_router_kernels();
cudaError_t launch_scan(const Layout& L, const Ctx& c, cudaStream_t st);
cudaError_t launch_scan_groups(const Layout& L, const Ctx& c, cudaStream_t st);
cudaError_t launch_scan_apply(const Layout& L, const Ctx& c, cudaStream_t st);
cudaError_t launch_scatter(const Layout& L, const Ctx& c, cudaStream_t st);
cudaError_t launch_mark_rows(const Layout& L, const Ctx& c, cudaStream_t st);
cudaError_t launch_wait_probe(int* status, cudaStream_t st);
cudaError_t launch_gather_rows(const Layout& L, const Ctx& c, const __nv_bfloat16* src, __nv_bfloat16* dst,
                               cudaStream_t st);
// rows [*lo, *hi) to dst row + *shift (streamed layer)
cudaError_t launch_gather_range(const Layout& L, const Ctx& c, const __nv_bfloat16* src, const int* lo, const int* hi,
                                const int* shift, int64_t max_rows, __nv_bfloat16* dst, cudaStream_t st);
cudaError_t launch_combine(const Layout& L, const Ctx& c, const __nv_bfloat16* Oprime, __nv_bfloat16* Y,
                           cudaStream_t st, const int* mb_range = nullptr);
cudaError_t launch_plan(const Layout& L, const Ctx& c, int ring_rows, int min_rows, cudaStream_t st);
cudaError_t launch_replay(const Layout& L, const Ctx& c, int chunk, const __nv_bfloat16* X, __nv_bfloat16* ring,
                          int64_t ring_rows, cudaStream_t st);
// expert slice: per-block counts of the tokens with a local assignment (before launch_router_bwd)
cudaError_t launch_active_count(const Layout& L, const Ctx& c, cudaStream_t st);
// expert slice: X rows of the listed tokens into c.xact (after launch_router_bwd)
cudaError_t launch_gather_active(const Layout& L, const Ctx& c, const __nv_bfloat16* X, cudaStream_t st);
// the fp32 gate/up accumulator into dW_gate / dW_up (bf16, or fp32 when L.w32)
cudaError_t launch_finish_acc(const Layout& L, const Ctx& c, void* dW_gate, void* dW_up, cudaStream_t st);
cudaError_t launch_router_bwd(const Layout& L, const Ctx& c, cudaStream_t st, int n_tiles_i = 0);
// MXFP8 quantisation, see quant.cu
cudaError_t launch_quant_weight(int mode, const __nv_bfloat16* src0, const __nv_bfloat16* src1, int64_t R_out, int K,
                                int N, uint8_t* q, uint8_t* qs, cudaStream_t st);
cudaError_t launch_gather_rows_mx(const Layout& L, const Ctx& c, const __nv_bfloat16* src, __nv_bfloat16* dst,
                                  uint8_t* q, uint8_t* qs, cudaStream_t st);
// rows [*lo, *hi): bf16 to dst row + *shift (a ring position; shift may be NULL), codes at the row,
// or at the ring position too with shift_codes
cudaError_t launch_gather_range_mx(const Layout& L, const Ctx& c, const __nv_bfloat16* src, const int* lo,
                                   const int* hi, const int* shift, bool shift_codes, int64_t max_rows,
                                   __nv_bfloat16* dst, uint8_t* q, uint8_t* qs, cudaStream_t st);
// Dispatch / reverse-combine with MXFP8 weight gradients: the padded rows gathered from src and
// quantised along d (qd, qds as launch_gather_rows_mx writes them) and along the rows in blocks of
// 32 (qr, qrs: rowq layout), no bf16 copy.
cudaError_t launch_gather_quant2(const Layout& L, const Ctx& c, const __nv_bfloat16* src, uint8_t* qd, uint8_t* qds,
                                 uint8_t* qr, uint8_t* qrs, cudaStream_t st);
// rows [*lo, *hi) only, the codes along d at row + *dshift (a ring position; dshift may be NULL)
cudaError_t launch_gather_quant2_range(const Layout& L, const Ctx& c, const __nv_bfloat16* src, const int* lo,
                                       const int* hi, const int* dshift, uint8_t* qd, uint8_t* qds, uint8_t* qr,
                                       uint8_t* qrs, cudaStream_t st);
// NVFP4 forward (nvfp4.cu): amax of |x| over n bf16 values (n a multiple of 8) into *amax (fp32 bits,
// atomicMax: the caller zeroes it); global scales gs[i] = 2688 / amax[i] (1 for 0) for i < n;
// the dispatch of X quantised along d; H (fp32 [RP, I]) quantised along I; weights quantised
// along K into the forward layouts (paired: the gate/up B operand, 64-row gate / up blocks;
// otherwise W [El][K][N] to rows el * N + n), gs the device scale(s) of src0 (and src1)
cudaError_t launch_nv_amax(const __nv_bfloat16* x, int64_t n, unsigned* amax, cudaStream_t st);
cudaError_t launch_nv_scale(const unsigned* amax, float* gs, int n, cudaStream_t st);
// (dst: the bf16 rows too, or NULL)
cudaError_t launch_nv_gather_x(const Layout& L, const Ctx& c, const __nv_bfloat16* X, const float* gs, uint8_t* q,
                               uint8_t* qs, __nv_bfloat16* dst, cudaStream_t st);
// rows of a row-major bf16 [R, K] quantised along K (the backward's weight layouts)
cudaError_t launch_nv_quant_rows(const __nv_bfloat16* src, int64_t R, int K, const float* gs, uint8_t* q, uint8_t* qs,
                                 cudaStream_t st);
cudaError_t launch_nv_quant_h(const Layout& L, const Ctx& c, const float* h, const float* gs, uint8_t* q, uint8_t* qs,
                              __nv_bfloat16* dst, cudaStream_t st);  // dst: the rows in bf16 too, or NULL
cudaError_t launch_nv_quant_weight(bool paired, const __nv_bfloat16* src0, const __nv_bfloat16* src1, int El, int K,
                                   int N, const float* gs, uint8_t* q, uint8_t* qs, cudaStream_t st);
cudaError_t launch_transpose_wr(const Layout& L, const __nv_bfloat16* W_r, __nv_bfloat16* W_rT, cudaStream_t st);
cudaError_t launch_rev_dispatch(const Layout& L, const Ctx& c, __nv_bfloat16* dX, cudaStream_t st);
cudaError_t launch_export_routing(const Layout& L, const Ctx& c, int32_t* counts, int32_t* offsets,
                                  int32_t* poff, int32_t* perm, cudaStream_t st);

}  // namespace moe
