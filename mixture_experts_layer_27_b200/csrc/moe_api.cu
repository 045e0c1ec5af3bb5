// Host side of libmoe.so: argument validation, the ctx / workspace layout,
// TMA tensor-map encoding and the launch sequences of moe_fwd / moe_bwd.
// Every step of the layer runs in this library's kernels; the host only
// enqueues work and never waits on the device (except in moe_get_error).
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>
#include <vector>

#include "ep_internal.cuh"
#include "moe_internal.cuh"

namespace moe {

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool make_layout(const moe_shape& s, Layout* L, int M) {
  if (s.T < 0 || s.d <= 0 || s.E <= 0 || s.I <= 0 || s.top_k <= 0) return false;
  if (s.E > kMaxE || s.top_k > kMaxK || s.top_k > s.E) return false;
  if (s.d % 256 || s.I % 256) return false;
  if (s.wgrad_dtype != MOE_WGRAD_BF16 && s.wgrad_dtype != MOE_WGRAD_FP32) return false;
  const int El = s.num_local_experts == 0 ? s.E - s.first_local_expert : s.num_local_experts;
  if (s.first_local_expert < 0 || El <= 0 || s.first_local_expert + El > s.E) return false;
  if (M < 0 || M > kMaxMinibatches) return false;
  if (M > 0 && (s.T % kTokensPerBlock != 0 || s.T == 0)) return false;  // minibatches of whole token blocks
  const int64_t T_all = M > 0 ? s.T * M : s.T;
  if (T_all * static_cast<int64_t>(s.top_k) >= (int64_t(1) << 31)) return false;
  L->T = T_all;
  L->M = M;
  L->T_mb = s.T;
  L->d = s.d;
  L->E = s.E;
  L->I = s.I;
  L->k = s.top_k;
  L->first = s.first_local_expert;
  L->El = El;
  L->w32 = s.wgrad_dtype == MOE_WGRAD_FP32;
  // a token has at most min(k, El) local assignments; every (macrobatch, expert) segment pads < 128 rows
  const int64_t A = T_all * (s.top_k < El ? s.top_k : El);
  const int64_t nseg = static_cast<int64_t>(El) * (M > 0 ? M : 1);
  L->RP = static_cast<int64_t>(align_up(static_cast<size_t>(A + int64_t(kPad - 1) * nseg), kPad));
  if (L->RP < kPad) L->RP = kPad;
  if (L->RP * static_cast<int64_t>(s.d > s.I ? s.d : s.I) >= (int64_t(1) << 40)) return false;
  L->nblk = static_cast<int>((T_all + kTokensPerBlock - 1) / kTokensPerBlock);
  if (L->nblk < 1) L->nblk = 1;
  L->scan_groups = L->nblk > kScanOneLevel ? (L->nblk + kScanGroup - 1) / kScanGroup : 0;

  const size_t RP = static_cast<size_t>(L->RP), T = static_cast<size_t>(T_all), k = s.top_k;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, 256);
    return at;
  };
  L->mx = s.prec == MOE_MXFP8 || s.prec == MOE_MXFP8_ALL;
  L->mxw = s.prec == MOE_MXFP8_ALL;
  L->nv = s.prec == MOE_NVFP4;
  // row-quantised operands are addressed by TMA as RP / 128 * C lines (a signed 32-bit coordinate)
  if (L->mxw && (L->RP / 128) * static_cast<int64_t>(s.d > s.I ? s.d : s.I) >= (int64_t(1) << 31)) return false;
  L->hdr = take(HDR_WORDS * 4);
  L->ids = take(T * k * 4);
  L->gates = take(T * k * 4);
  L->counts = take(static_cast<size_t>(s.E) * 4);
  L->offsets = take(static_cast<size_t>(s.E + 1) * 4);
  L->poff = take(static_cast<size_t>(El + 1) * 4);
  L->perm_tok = take(T * k * 4);
  L->perm_asg = take(T * k * 4);
  L->slot_row = take(T * k * 4);
  L->row_asg = take(RP * 4);
  L->row_gate = take(RP * 4);
  // streamed layer: X_perm lives in the caller's ring; MXFP8 weight gradients keep X quantised instead
  L->xperm = take(M > 0 || s.prec == MOE_MXFP8_ALL ? 0 : RP * s.d * 2);
  L->abuf = take(RP * s.I * 2);
  L->bbuf = take(RP * s.I * 2);
  L->stab = take(M > 0 ? static_cast<size_t>(stream_table_words(M, El)) * 4 : 0);
  const size_t mxd = L->mx ? RP * s.d : 0, mxi = L->mx ? RP * s.I : 0;  // fp8 bytes; scales are 1/32 of that
  // the one-batch MXFP8 forward's X codes (a ring-streamed layer keeps them in the caller's ring)
  // (NVFP4: two codes per byte and one scale byte per 16 values)
  L->xq = take(M > 0 ? 0 : (L->nv ? RP * s.d / 2 : mxd));
  L->xqs = take(M > 0 ? 0 : (L->nv ? RP * s.d / 16 : mxd / 32));
  const size_t wxd = L->mxw ? RP * s.d : 0, wxi = L->mxw ? RP * s.I : 0;
  L->xqt = take(wxd);  // X along the rows, from the forward's dispatch for the weight gradients
  L->xqts = take(wxd / 32);
  L->ctx_bytes = o;

  o = 0;
  L->hist = take(static_cast<size_t>(L->nblk) * s.E * 4);
  L->hsum = take(static_cast<size_t>(L->scan_groups) * s.E * 4);
  L->logits = take(T * s.E * 4);
  L->rpart = take(static_cast<size_t>(router_splits(T_all, s.E, s.d)) * T * s.E * 4);
  L->hbuf = take(RP * s.I * 2);
  L->obuf = take(RP * s.d * 2);
  L->dyperm = take(RP * s.d * 2);
  L->dabuf = take(RP * s.I * 2);
  L->dbbuf = take(RP * s.I * 2);
  L->hgbuf = take(RP * s.I * 2);
  L->dgpart = take(RP * (s.I / 128) * 4);  // dg partials per n-tile of the dgrad-down GEMM (256 wide bf16, 128 MXFP8)
  L->dlasg = take(T * k * 4);
  L->dldense = take(2 * align_up(static_cast<size_t>(T), 64) * align_up(static_cast<size_t>(s.E), 64) * 2);
  L->rslice = El < s.E;
  L->actcnt = take(L->rslice ? ((T + 255) / 256 + 1) * 4 : 0);
  L->actlist = take(L->rslice ? T * 4 : 0);
  L->xact = take(L->rslice ? align_up(T, 64) * s.d * 2 : 0);
  L->wrt = take(static_cast<size_t>(s.E) * s.d * 2);
  L->dxperm = take(RP * s.d * 2);
  L->acc32 = take(M > 0 ? 2 * static_cast<size_t>(El) * s.d * s.I * 4 : 0);
  L->hq = take(L->nv ? RP * s.I / 2 : mxi);
  L->hqs = take(L->nv ? RP * s.I / 16 : mxi / 32);
  L->nvh = take(L->nv ? RP * s.I * 4 : 0);
  L->nvsc = take(L->nv ? 256 : 0);
  L->dyq = take(L->nv ? RP * s.d / 2 : mxd);
  L->dyqs = take(L->nv ? RP * s.d / 16 : mxd / 32);
  L->daq = take(L->nv ? RP * s.I / 2 : mxi);
  L->daqs = take(L->nv ? RP * s.I / 16 : mxi / 32);
  L->dbq = take(L->nv ? RP * s.I / 2 : mxi);
  L->dbqs = take(L->nv ? RP * s.I / 16 : mxi / 32);
  L->nvdab = take(L->nv ? 2 * RP * s.I * 4 : 0);
  L->fctl = take(L->mx ? 0 : static_cast<size_t>(gemm_pair_ctl_words(L->RP)) * 4);
  L->dyqt = take(wxd);
  L->dyqts = take(wxd / 32);
  L->daqt = take(wxi);
  L->daqts = take(wxi / 32);
  L->dbqt = take(wxi);
  L->dbqts = take(wxi / 32);
  L->hgqt = take(wxi);
  L->hgqts = take(wxi / 32);
  L->ws_bytes = o;
  // prepared weights: [W_gate|W_up paired, K = d] [W_down^T, K = I] [W_down, K = d] [W_gate, K = I] [W_up, K = I]
  o = 0;
  // NVFP4: the same five layouts at half a byte per value and a scale byte per 16, then the four
  // global scales (and their amax words)
  const size_t w1 = static_cast<size_t>(El) * s.d * s.I;
  const size_t wb = L->nv ? w1 / 2 : w1, wsb = L->nv ? w1 / 16 : w1 / 32, wbwd = 1;
  L->wgu1 = take(2 * wb);
  L->wgu1s = take(2 * wsb);
  L->wd2 = take(wb);
  L->wd2s = take(wsb);
  L->wd3 = take(wbwd * wb);
  L->wd3s = take(wbwd * wsb);
  L->wg4 = take(wbwd * wb);
  L->wg4s = take(wbwd * wsb);
  L->wu4 = take(wbwd * wb);
  L->wu4s = take(wbwd * wsb);
  L->wnvgs = take(L->nv ? 256 : 0);
  L->wq_bytes = o;
  return true;
}

Ctx make_ctx(const Layout& L, void* ctx, void* ws) {
  auto C = [&](size_t off) { return static_cast<char*>(ctx) + off; };
  auto W = [&](size_t off) { return static_cast<char*>(ws) + off; };
  Ctx c;
  c.hdr = reinterpret_cast<int*>(C(L.hdr));
  c.ids = reinterpret_cast<int*>(C(L.ids));
  c.gates = reinterpret_cast<float*>(C(L.gates));
  c.counts = reinterpret_cast<int*>(C(L.counts));
  c.offsets = reinterpret_cast<int*>(C(L.offsets));
  c.poff = reinterpret_cast<int*>(C(L.poff));
  c.perm_tok = reinterpret_cast<int*>(C(L.perm_tok));
  c.perm_asg = reinterpret_cast<int*>(C(L.perm_asg));
  c.slot_row = reinterpret_cast<int*>(C(L.slot_row));
  c.row_asg = reinterpret_cast<int*>(C(L.row_asg));
  c.row_gate = reinterpret_cast<float*>(C(L.row_gate));
  c.xperm = reinterpret_cast<__nv_bfloat16*>(C(L.xperm));
  c.abuf = reinterpret_cast<__nv_bfloat16*>(C(L.abuf));
  c.bbuf = reinterpret_cast<__nv_bfloat16*>(C(L.bbuf));
  c.tab = StreamTables{};
  if (L.M > 0) {
    int* t = reinterpret_cast<int*>(C(L.stab));
    const int M = L.M, El = L.El;
    c.tab.plan = t;        t += PLAN_WORDS;
    c.tab.mb_of = t;       t += M;
    c.tab.seg_poff = t;    t += M * El + 1;
    c.tab.cum = t;         t += M * El;
    c.tab.mb_range = t;    t += 2 * M;
    c.tab.shift_fwd = t;   t += M;
    c.tab.shift_bwd = t;   t += M;
    c.tab.replay = t;      t += M;
    c.tab.chunk = t;       t += 4 * M;
    c.tab.ring_start = t;
  }
  c.acc32 = nullptr;
  c.fctl = nullptr;
  c.actcnt = c.actlist = nullptr;
  c.xact = nullptr;
  c.xq = L.mx || L.nv ? reinterpret_cast<uint8_t*>(C(L.xq)) : nullptr;
  c.xqs = L.mx || L.nv ? reinterpret_cast<uint8_t*>(C(L.xqs)) : nullptr;
  c.nvh = (ws && L.nv) ? reinterpret_cast<float*>(W(L.nvh)) : nullptr;
  c.nvsc = (ws && L.nv) ? reinterpret_cast<unsigned*>(W(L.nvsc)) : nullptr;
  c.nvdab = (ws && L.nv) ? reinterpret_cast<float*>(W(L.nvdab)) : nullptr;
  c.hq = c.hqs = c.dyq = c.dyqs = c.daq = c.daqs = c.dbq = c.dbqs = nullptr;
  c.xqt = c.xqts = c.dyqt = c.dyqts = c.daqt = c.daqts = c.dbqt = c.dbqts = c.hgqt = c.hgqts = nullptr;
  if (L.mxw) {
    c.xqt = reinterpret_cast<uint8_t*>(C(L.xqt));
    c.xqts = reinterpret_cast<uint8_t*>(C(L.xqts));
  }
  if (ws && L.mxw) {
    c.dyqt = reinterpret_cast<uint8_t*>(W(L.dyqt));
    c.dyqts = reinterpret_cast<uint8_t*>(W(L.dyqts));
    c.daqt = reinterpret_cast<uint8_t*>(W(L.daqt));
    c.daqts = reinterpret_cast<uint8_t*>(W(L.daqts));
    c.dbqt = reinterpret_cast<uint8_t*>(W(L.dbqt));
    c.dbqts = reinterpret_cast<uint8_t*>(W(L.dbqts));
    c.hgqt = reinterpret_cast<uint8_t*>(W(L.hgqt));
    c.hgqts = reinterpret_cast<uint8_t*>(W(L.hgqts));
  }
  if (ws && (L.mx || L.nv)) {
    c.hq = reinterpret_cast<uint8_t*>(W(L.hq));
    c.hqs = reinterpret_cast<uint8_t*>(W(L.hqs));
    c.dyq = reinterpret_cast<uint8_t*>(W(L.dyq));
    c.dyqs = reinterpret_cast<uint8_t*>(W(L.dyqs));
    c.daq = reinterpret_cast<uint8_t*>(W(L.daq));
    c.daqs = reinterpret_cast<uint8_t*>(W(L.daqs));
    c.dbq = reinterpret_cast<uint8_t*>(W(L.dbq));
    c.dbqs = reinterpret_cast<uint8_t*>(W(L.dbqs));
  }
  if (ws) {
    c.hist = reinterpret_cast<int*>(W(L.hist));
    c.hsum = reinterpret_cast<int*>(W(L.hsum));
    c.logits = reinterpret_cast<float*>(W(L.logits));
    c.rpart = reinterpret_cast<float*>(W(L.rpart));
    c.hbuf = reinterpret_cast<__nv_bfloat16*>(W(L.hbuf));
    c.obuf = reinterpret_cast<__nv_bfloat16*>(W(L.obuf));
    c.dyperm = reinterpret_cast<__nv_bfloat16*>(W(L.dyperm));
    c.dabuf = reinterpret_cast<__nv_bfloat16*>(W(L.dabuf));
    c.dbbuf = reinterpret_cast<__nv_bfloat16*>(W(L.dbbuf));
    c.hgbuf = reinterpret_cast<__nv_bfloat16*>(W(L.hgbuf));
    c.dgpart = reinterpret_cast<float*>(W(L.dgpart));
    c.dlasg = reinterpret_cast<float*>(W(L.dlasg));
    c.dldense = reinterpret_cast<__nv_bfloat16*>(W(L.dldense));
    c.wrt = reinterpret_cast<__nv_bfloat16*>(W(L.wrt));
    c.dxperm = reinterpret_cast<__nv_bfloat16*>(W(L.dxperm));
    c.acc32 = L.M > 0 ? reinterpret_cast<float*>(W(L.acc32)) : nullptr;
    c.fctl = !L.mx ? reinterpret_cast<int*>(W(L.fctl)) : nullptr;
    if (L.rslice) {
      c.actcnt = reinterpret_cast<int*>(W(L.actcnt));
      c.actlist = reinterpret_cast<int*>(W(L.actlist));
      c.xact = reinterpret_cast<__nv_bfloat16*>(W(L.xact));
    }
  }
  return c;
}

// ---------------------------------------------------------------------------
// TMA tensor maps (driver entry point fetched through the runtime, so the
// library does not link libcuda directly)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 tensor [outer, inner] (inner contiguous, row pitch in elements),
// box {box_inner, box_outer}, 128-byte swizzle, zero fill out of bounds.
bool tmap_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t pitch_elems,
                    uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {pitch_elems * 2};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D fp8 (byte) tensor [outer, inner], box {128, 128}, 128-byte swizzle.
static bool tmap_fp8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner};
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D fp32 tensor [outer, inner] (dense rows), box {32, 32} (128-byte rows), 128-byte swizzle.
static bool tmap_f32(CUtensorMap* m, void* base, uint64_t inner, uint64_t outer) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * 4};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output map of an expert weight gradient [outer, inner]: bf16 in 64 x 32 boxes, or fp32 in
// 32 x 32 boxes when the layer writes the unrounded sums.
static bool tmap_wgrad_out(const Layout& L, CUtensorMap* m, void* base, uint64_t inner, uint64_t outer) {
  return L.w32 ? tmap_f32(m, base, inner, outer) : tmap_2d(m, base, inner, outer, inner, 64, 32);
}

static int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess)
      n = 148;
  }
  return n;
}

// ---------------------------------------------------------------------------
// optional per-kernel timing: each launch bracketed by CUDA events on its stream
// ---------------------------------------------------------------------------
enum KernelId {
  K_ROUTER_LOGITS, K_TOPK, K_SCAN, K_SCATTER, K_DISPATCH, K_GEMM_GATEUP, K_GEMM_DOWN, K_COMBINE,
  K_REV_COMBINE, K_GEMM_DGRAD_DOWN, K_ROUTER_BWD, K_ROUTER_WGRAD, K_TRANSPOSE_WR, K_GEMM_DGRAD_GATEUP, K_REV_DISPATCH,
  K_GEMM_WGRAD_GATEUP, K_GEMM_WGRAD_DOWN, K_PLAN, K_REPLAY, K_FINISH_ACC, K_QUANT_WEIGHTS, K_MARK_ROWS,
  K_ACTIVE_COUNT, K_GATHER_ACTIVE, K_SCAN_GROUPS, K_SCAN_APPLY, K_PAIR_FWD, K_PAIR_DGRAD, K_MX_WGRAD_GATEUP, K_MX_WGRAD_DOWN,
  K_NV_SCALE, K_NV_GATEUP, K_NV_QUANT_H, K_NV_DOWN, K_NV_DGRAD_DOWN, K_NV_QUANT_DAB, K_NV_DGRAD_GATEUP, K_NUM
};
static const char* kKernelNames[K_NUM] = {
    "router_logits", "topk_gating", "hist_scan", "stable_scatter", "dispatch", "gemm_gateup_swiglu",
    "gemm_down_combw", "combine", "reverse_combine", "gemm_dgrad_down_swiglu_bwd", "router_bwd", "router_wgrad",
    "transpose_wr", "gemm_dgrad_gateup", "reverse_dispatch", "gemm_wgrad_gateup", "gemm_wgrad_down",
    "stream_plan", "ring_replay", "wgrad_accumulator_finish", "quantize_weights", "mark_pad_rows",
    "router_token_count", "router_token_gather", "hist_scan_group_sums", "hist_scan_group_apply",
    "gemm_gateup_down_persistent", "gemm_dgrads_persistent", "gemm_wgrad_gateup_mx", "gemm_wgrad_down_mx",
    "nvfp4_amax_scale", "gemm_gateup_swiglu_nvfp4", "nvfp4_quantize_h", "gemm_down_combw_nvfp4",
    "gemm_dgrad_down_swiglu_bwd_nvfp4", "nvfp4_quantize_da_db", "gemm_dgrad_gateup_nvfp4"};

struct ProfRec {
  int kid;
  cudaEvent_t a, b;
};
static std::mutex g_mu;
static bool g_prof_on = false;
static std::vector<ProfRec> g_prof;
static std::vector<cudaEvent_t> g_pool;
static std::atomic<unsigned long long> g_launches{0};

static cudaEvent_t pool_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// Launches one kernel through `fn`, counting it and (when enabled) timing it.
template <class F>
static cudaError_t timed(int kid, cudaStream_t st, F fn) {
  cudaEvent_t a = nullptr, b = nullptr;
  if (g_prof_on) {
    std::lock_guard<std::mutex> lk(g_mu);
    a = pool_event();
    b = pool_event();
    if (a && b) cudaEventRecord(a, st);
  }
  const cudaError_t e = fn();
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (g_prof_on && a && b) {
    cudaEventRecord(b, st);
    std::lock_guard<std::mutex> lk(g_mu);
    g_prof.push_back({kid, a, b});
  }
  return e;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

cudaError_t launch_router_logits(const Layout& L, const void* X, const __nv_bfloat16* wrt, float* rpart, int* status,
                                 cudaStream_t st) {
  const int splits = router_splits(L.T, L.E, L.d);
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  if (!tmap_2d(&p.ta0, X, L.d, static_cast<uint64_t>(L.T), L.d, 64, 128) ||
      !tmap_2d(&p.tb0, wrt, L.d, static_cast<uint64_t>(L.E), L.d, 64, 256))
    return cudaErrorInvalidValue;
  p.ta1 = p.ta0;
  p.tb1 = p.tb0;
  p.El = L.El;
  p.d = L.d;
  p.I = L.I;
  p.T = static_cast<int>(L.T);
  p.E = L.E;
  p.splits = splits;
  p.router_bn = router_tile_n(L.E);
  p.outf = rpart;
  p.status = status;
  const int64_t tiles = ((L.T + 127) / 128) * ((L.E + 255) / 256) * splits;
  const int grid = static_cast<int>(tiles < num_sms() ? tiles : num_sms());
  return launch_gemm(G_ROUTER, p, grid, st);
}

static GemmParams base_params(const Layout& L, const Ctx& c, int* status) {
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.hdr = c.hdr;
  p.poff = c.poff;
  p.cnt = c.counts + L.first;
  p.row_gate = c.row_gate;
  p.row_asg = c.row_asg;
  p.El = L.El;
  p.d = L.d;
  p.I = L.I;
  p.nseg = L.El;
  p.wout32 = L.w32 ? 1 : 0;
  p.status = status;
  return p;
}

static MxParams mx_params(const Layout& L, const Ctx& c, int* status) {
  MxParams p;
  std::memset(&p, 0, sizeof(p));
  p.poff = c.poff;
  p.nseg = L.El;
  p.row_gate = c.row_gate;
  p.row_asg = c.row_asg;
  p.El = L.El;
  p.d = L.d;
  p.I = L.I;
  p.status = status;
  return p;
}

// dW_r = X^T . DL on the tensor cores (both operands MN-major: d and E are contiguous, the
// contraction runs over tokens, twice: the hi and the lo bf16 terms of dl); fp32 out, one CTA
// per 128 x 256 tile, fixed K order.  In an expert slice the tokens are the listed ones
// (c.xact, compacted DL rows, their number on the device).
static cudaError_t launch_router_wgrad(const Layout& L, const Ctx& c, const void* X, float* dW_r, int* status,
                                       cudaStream_t st) {
  GemmParams p = base_params(L, c, status);
  const uint64_t E64 = align_up(static_cast<size_t>(L.E), 64);
  const uint64_t Tpad = align_up(static_cast<size_t>(L.T), 64);
  if (L.rslice) {
    if (!tmap_2d(&p.ta0, c.xact, L.d, Tpad, L.d, 64, 64)) return cudaErrorInvalidValue;
    p.act_n = c.actcnt + (L.T + 255) / 256;
  } else if (!tmap_2d(&p.ta0, X, L.d, static_cast<uint64_t>(L.T), L.d, 64, 64)) {
    return cudaErrorInvalidValue;
  }
  if (!tmap_2d(&p.tb0, c.dldense, E64, 2 * Tpad, E64, 64, 64)) return cudaErrorInvalidValue;
  p.ta1 = p.ta0;
  p.tb1 = p.tb0;
  p.outf = dW_r;
  p.T = static_cast<int>(L.T);
  p.E = L.E;
  p.splits = 1;
  const int tiles = (L.d / 128) * ((L.E + 255) / 256);
  const int grid = tiles < num_sms() ? tiles : num_sms();
  return launch_gemm(G_ROUTER_WGRAD, p, grid, st);
}

#define MOE_TRY(x)                                   \
  do {                                               \
    if ((x) != cudaSuccess) return MOE_ERR_CUDA;     \
  } while (0)
#define MOE_TMAP(x)                                  \
  do {                                               \
    if (!(x)) return MOE_ERR_CUDA;                   \
  } while (0)
#define MOE_TRY_STATUS(x)                            \
  do {                                               \
    const moe_status s_ = (x);                       \
    if (s_ != MOE_OK) return s_;                     \
  } while (0)

}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_ctx_size(const moe_shape* s) {
  Layout L;
  if (!s || !make_layout(*s, &L)) return 0;
  return L.ctx_bytes;
}

size_t moe_workspace_size(const moe_shape* s) {
  Layout L;
  if (!s || !make_layout(*s, &L)) return 0;
  return L.ws_bytes;
}

const char* moe_status_string(moe_status st) {
  switch (st) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape or mode";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "ctx or workspace too small";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case MOE_ERR_NONFINITE: return "non-finite router logit";
    case MOE_ERR_EXCHANGE: return "expert-parallel exchange tables do not fit together";
  }
  return "unknown status";
}

static bool is_mx_prec(int32_t prec) { return prec == MOE_MXFP8 || prec == MOE_MXFP8_ALL; }

static moe_status check_shape_mx(const moe_shape* s, Layout* L) {
  if (!s) return MOE_ERR_INVALID_ARG;
  if (!is_mx_prec(s->prec)) return MOE_ERR_INVALID_ARG;
  if (s->T < 0 || s->d <= 0 || s->E <= 0 || s->I <= 0 || s->top_k <= 0 || s->first_local_expert < 0 ||
      s->num_local_experts < 0)
    return MOE_ERR_INVALID_ARG;
  if (!make_layout(*s, L)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

static moe_status check_shape(const moe_shape* s, Layout* L) {
  if (!s) return MOE_ERR_INVALID_ARG;
  if (s->T < 0 || s->d <= 0 || s->E <= 0 || s->I <= 0 || s->top_k <= 0 || s->first_local_expert < 0 ||
      s->num_local_experts < 0)
    return MOE_ERR_INVALID_ARG;
  if (s->prec != MOE_BF16 && !is_mx_prec(s->prec)) return MOE_ERR_INVALID_ARG;
  if (is_mx_prec(s->prec)) return MOE_ERR_UNSUPPORTED;
  if (!make_layout(*s, L)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

// Router GEMM, top-k gating, histogram + scan (+ the stream plan) and the stable scatter.
static moe_status route_tokens(const Layout& L, const Ctx& c, const void* X, const void* W_r, const float* bias,
                               int ring_rows, cudaStream_t st) {
  const int grid = num_sms();
  int* status = c.hdr + HDR_STATUS;
  MOE_TRY(timed(K_TRANSPOSE_WR, st, [&] {
    return launch_transpose_wr(L, static_cast<const __nv_bfloat16*>(W_r), c.wrt, st);
  }));
  const int splits = router_splits(L.T, L.E, L.d);
  MOE_TRY(timed(K_ROUTER_LOGITS, st, [&] { return launch_router_logits(L, X, c.wrt, c.rpart, status, st); }));
  MOE_TRY(timed(K_TOPK, st, [&] { return launch_topk(L, c, bias, splits, st); }));
  if (L.scan_groups) MOE_TRY(timed(K_SCAN_GROUPS, st, [&] { return launch_scan_groups(L, c, st); }));
  MOE_TRY(timed(K_SCAN, st, [&] { return launch_scan(L, c, st); }));
  if (L.scan_groups) MOE_TRY(timed(K_SCAN_APPLY, st, [&] { return launch_scan_apply(L, c, st); }));
  if (L.M > 0) {
    // two full waves of the gate/up GEMM: (rows / 128) * (I / 128) >= 2 * SMs
    const int min_rows = static_cast<int>((2LL * grid * 128) / (L.I / 128));
    MOE_TRY(timed(K_PLAN, st, [&] { return launch_plan(L, c, ring_rows, min_rows, st); }));
  }
  MOE_TRY(timed(K_MARK_ROWS, st, [&] { return launch_mark_rows(L, c, st); }));  // pad rows: live / dead
  MOE_TRY(timed(K_SCATTER, st, [&] { return launch_scatter(L, c, st); }));
  return MOE_OK;
}

moe_status moe_fwd(const moe_shape* s, const void* X, const void* W_r, const float* bias, const void* W_gate,
                   const void* W_up, const void* W_down, void* Y, void* ctx, size_t ctx_bytes, void* ws,
                   size_t ws_bytes, void* stream) {
  Layout L;
  const moe_status cs = check_shape(s, &L);
  if (cs != MOE_OK) return cs;
  const bool tok = s->T > 0;  // with no tokens, X and Y may be empty (NULL)
  if ((tok && (!X || !Y)) || !W_r || !W_gate || !W_up || !W_down || !ctx || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(W_r) || !aligned16(W_gate) || !aligned16(W_up) || !aligned16(W_down) ||
      !aligned16(Y) || !aligned16(ctx) || !aligned16(ws) || (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)))
    return MOE_ERR_INVALID_ARG;
  if (ctx_bytes < L.ctx_bytes || ws_bytes < L.ws_bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ctx c = make_ctx(L, ctx, ws);
  MOE_TRY(cudaMemsetAsync(c.hdr, 0, HDR_WORDS * 4, st));  // clears the status word
  if (L.T == 0) return MOE_OK;

  const auto* Xb = static_cast<const __nv_bfloat16*>(X);
  const int grid = num_sms();
  int* status = c.hdr + HDR_STATUS;
  const uint64_t RP = static_cast<uint64_t>(L.RP);
  // 1-4. router GEMM (tensor cores, fixed K splits), top-k gating, histogram + scan, stable scatter
  {
    const moe_status r = route_tokens(L, c, X, W_r, bias, 0, st);
    if (r != MOE_OK) return r;
  }
  // 4. dispatch into the expert-contiguous layout
  MOE_TRY(timed(K_DISPATCH, st, [&] { return launch_gather_rows(L, c, Xb, c.xperm, st); }));

  // 5. grouped gate/up GEMM with the SwiGLU epilogue
  {
    GemmParams p = base_params(L, c, status);
    MOE_TMAP(tmap_2d(&p.ta0, c.xperm, L.d, RP, L.d, 64, 128));
    MOE_TMAP(tmap_2d(&p.tb0, W_gate, L.I, static_cast<uint64_t>(L.El) * L.d, L.I, 64, 64));
    MOE_TMAP(tmap_2d(&p.tb1, W_up, L.I, static_cast<uint64_t>(L.El) * L.d, L.I, 64, 64));
    p.ta1 = p.ta0;
    p.out0 = c.abuf;
    p.out1 = c.bbuf;
    p.out2 = c.hbuf;
    MOE_TRY(timed(K_GEMM_GATEUP, st, [&] { return launch_gemm(G_GATEUP, p, grid, st); }));
  }
  // 6. grouped down GEMM with the combine-weight epilogue
  {
    GemmParams p = base_params(L, c, status);
    MOE_TMAP(tmap_2d(&p.ta0, c.hbuf, L.I, RP, L.I, 64, 128));
    MOE_TMAP(tmap_2d(&p.tb0, W_down, L.d, static_cast<uint64_t>(L.El) * L.I, L.d, 64, 64));
    p.ta1 = p.ta0;
    p.tb1 = p.tb0;
    p.out0 = c.obuf;
    MOE_TRY(timed(K_GEMM_DOWN, st, [&] { return launch_gemm(G_DOWN, p, grid, st); }));
  }
  // 7. combine
  MOE_TRY(timed(K_COMBINE, st, [&] { return launch_combine(L, c, c.obuf, static_cast<__nv_bfloat16*>(Y), st); }));
  return MOE_OK;
}

// Two dependent grouped GEMMs as one persistent launch (a CTA per SM, a second wave claimed
// through Cluster Launch Control by the CTAs that run first).
static cudaError_t run_gemm_pair(const Layout& L, const Ctx& c, GemmPair pair, const GemmParams& p1,
                                 const GemmParams& p2, cudaStream_t st, bool skip_first = false) {
  GemmPairParams f;
  f.p1 = p1;
  f.p2 = p2;
  f.ctl = c.fctl;
  f.mt_cap = static_cast<int>(L.RP / 128);
  f.skip_first = skip_first ? 1 : 0;
  cudaError_t e = cudaMemsetAsync(c.fctl, 0, static_cast<size_t>(gemm_pair_ctl_words(L.RP)) * 4, st);
  if (e != cudaSuccess) return e;
  const int64_t units = gemm_pair_units(pair, L.RP, L.d, L.I);
  const int64_t grid = units < 2LL * num_sms() ? units : 2LL * num_sms();
  return launch_gemm_pair(pair, f, grid, st);
}

// The forward with its two grouped GEMMs in one persistent launch: the same routing, dispatch
// and combine launches as moe_fwd around it.  skip_first: the test hook of GemmPairParams.
static moe_status fwd_persistent_impl(const moe_shape* s, const void* X, const void* W_r, const float* bias,
                                      const void* W_gate, const void* W_up, const void* W_down, void* Y, void* ctx,
                                      size_t ctx_bytes, void* ws, size_t ws_bytes, void* stream, bool skip_first) {
  Layout L;
  const moe_status cs = check_shape(s, &L);
  if (cs != MOE_OK) return cs;
  const bool tok = s->T > 0;
  if ((tok && (!X || !Y)) || !W_r || !W_gate || !W_up || !W_down || !ctx || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(W_r) || !aligned16(W_gate) || !aligned16(W_up) || !aligned16(W_down) ||
      !aligned16(Y) || !aligned16(ctx) || !aligned16(ws) || (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)))
    return MOE_ERR_INVALID_ARG;
  if (ctx_bytes < L.ctx_bytes || ws_bytes < L.ws_bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ctx c = make_ctx(L, ctx, ws);
  MOE_TRY(cudaMemsetAsync(c.hdr, 0, HDR_WORDS * 4, st));
  if (L.T == 0) return MOE_OK;

  int* status = c.hdr + HDR_STATUS;
  const uint64_t RP = static_cast<uint64_t>(L.RP);
  {
    const moe_status r = route_tokens(L, c, X, W_r, bias, 0, st);
    if (r != MOE_OK) return r;
  }
  MOE_TRY(timed(K_DISPATCH, st, [&] {
    return launch_gather_rows(L, c, static_cast<const __nv_bfloat16*>(X), c.xperm, st);
  }));
  GemmParams gu = base_params(L, c, status);
  MOE_TMAP(tmap_2d(&gu.ta0, c.xperm, L.d, RP, L.d, 64, 128));
  MOE_TMAP(tmap_2d(&gu.tb0, W_gate, L.I, static_cast<uint64_t>(L.El) * L.d, L.I, 64, 64));
  MOE_TMAP(tmap_2d(&gu.tb1, W_up, L.I, static_cast<uint64_t>(L.El) * L.d, L.I, 64, 64));
  gu.ta1 = gu.ta0;
  gu.out0 = c.abuf;
  gu.out1 = c.bbuf;
  gu.out2 = c.hbuf;
  GemmParams dn = base_params(L, c, status);
  MOE_TMAP(tmap_2d(&dn.ta0, c.hbuf, L.I, RP, L.I, 64, 128));
  MOE_TMAP(tmap_2d(&dn.tb0, W_down, L.d, static_cast<uint64_t>(L.El) * L.I, L.d, 64, 64));
  dn.ta1 = dn.ta0;
  dn.tb1 = dn.tb0;
  dn.out0 = c.obuf;
  MOE_TRY(timed(K_PAIR_FWD, st, [&] { return run_gemm_pair(L, c, PAIR_FWD, gu, dn, st, skip_first); }));
  MOE_TRY(timed(K_COMBINE, st, [&] { return launch_combine(L, c, c.obuf, static_cast<__nv_bfloat16*>(Y), st); }));
  return MOE_OK;
}

moe_status moe_fwd_persistent(const moe_shape* s, const void* X, const void* W_r, const float* bias,
                              const void* W_gate, const void* W_up, const void* W_down, void* Y, void* ctx,
                              size_t ctx_bytes, void* ws, size_t ws_bytes, void* stream) {
  return fwd_persistent_impl(s, X, W_r, bias, W_gate, W_up, W_down, Y, ctx, ctx_bytes, ws, ws_bytes, stream, false);
}

moe_status moe_debug_pair_wait(const moe_shape* s, const void* X, const void* W_r, const float* bias,
                               const void* W_gate, const void* W_up, const void* W_down, void* Y, void* ctx,
                               size_t ctx_bytes, void* ws, size_t ws_bytes, void* stream) {
  return fwd_persistent_impl(s, X, W_r, bias, W_gate, W_up, W_down, Y, ctx, ctx_bytes, ws, ws_bytes, stream, true);
}

// 10. router backward: dl (and, in an expert slice, the list of tokens with a local
// assignment and their X rows), then dW_r = X^T DL on the tensor cores.
static moe_status router_backward(const Layout& L, const Ctx& c, const void* X, float* dW_r, int* status,
                                  cudaStream_t st, int n_tiles_i = 0) {
  if (L.rslice) MOE_TRY(timed(K_ACTIVE_COUNT, st, [&] { return launch_active_count(L, c, st); }));
  MOE_TRY(timed(K_ROUTER_BWD, st, [&] { return launch_router_bwd(L, c, st, n_tiles_i); }));
  if (L.rslice)
    MOE_TRY(timed(K_GATHER_ACTIVE, st, [&] {
      return launch_gather_active(L, c, static_cast<const __nv_bfloat16*>(X), st);
    }));
  MOE_TRY(timed(K_ROUTER_WGRAD, st, [&] { return launch_router_wgrad(L, c, X, dW_r, status, st); }));
  return MOE_OK;
}

// Expert weight gradients from the saved X_perm and the backward's dA, dB, Hg, dY_perm:
// gate/up, then down (write-bound; separate launches keep the HBM traffic one-directional).
// With at most 256 rows per expert on average (four 64-row K blocks) a tile's MMAs are short
// and the gradient stores of the epilogue set the pace: the tiles are then decoded ahead by a
// scheduler warp (launch_gemm's sched flag).
static moe_status launch_wgrads(const Layout& L, const Ctx& c, int* status, void* dW_gate, void* dW_up,
                                void* dW_down, cudaStream_t st) {
  const int grid = num_sms();
  const bool sched = L.M == 0 && L.T * L.k <= 256LL * L.E;
  const uint64_t RP = static_cast<uint64_t>(L.RP), El = static_cast<uint64_t>(L.El);
  {
    GemmParams p = base_params(L, c, status);
    MOE_TMAP(tmap_2d(&p.ta0, c.xperm, L.d, RP, L.d, 64, 64));
    MOE_TMAP(tmap_2d(&p.tb0, c.dabuf, L.I, RP, L.I, 64, 64));
    MOE_TMAP(tmap_2d(&p.tb1, c.dbbuf, L.I, RP, L.I, 64, 64));
    MOE_TMAP(tmap_wgrad_out(L, &p.to0, dW_gate, L.I, El * L.d));
    MOE_TMAP(tmap_wgrad_out(L, &p.to1, dW_up, L.I, El * L.d));
    p.ta1 = p.ta0;
    MOE_TRY(timed(K_GEMM_WGRAD_GATEUP, st, [&] { return launch_gemm(G_WGRAD_GATEUP, p, grid, st, sched); }));
  }
  {
    GemmParams p = base_params(L, c, status);
    MOE_TMAP(tmap_2d(&p.ta0, c.hgbuf, L.I, RP, L.I, 64, 64));
    MOE_TMAP(tmap_2d(&p.tb0, c.dyperm, L.d, RP, L.d, 64, 64));
    MOE_TMAP(tmap_wgrad_out(L, &p.to0, dW_down, L.d, El * L.I));
    p.to1 = p.to0;
    p.ta1 = p.ta0;
    p.tb1 = p.tb0;
    MOE_TRY(timed(K_GEMM_WGRAD_DOWN, st, [&] { return launch_gemm(G_WGRAD_DOWN, p, grid, st, sched); }));
  }
  return MOE_OK;
}

// Zero expert and router weight gradients (a backward with no tokens).
static moe_status zero_wgrads(const Layout& L, void* dW_gate, void* dW_up, void* dW_down, float* dW_r,
                              cudaStream_t st) {
  const size_t wexp = static_cast<size_t>(L.El) * L.d * L.I * (L.w32 ? 4 : 2);
  MOE_TRY(cudaMemsetAsync(dW_gate, 0, wexp, st));
  MOE_TRY(cudaMemsetAsync(dW_up, 0, wexp, st));
  MOE_TRY(cudaMemsetAsync(dW_down, 0, wexp, st));
  MOE_TRY(cudaMemsetAsync(dW_r, 0, static_cast<size_t>(L.d) * L.E * 4, st));
  return MOE_OK;
}

// persistent: both dgrads as one persistent launch (the router backward then runs after them).
static moe_status bwd_impl(const moe_shape* s, const void* X, const void* W_r, const void* W_gate, const void* W_up,
                           const void* W_down, const void* dY, void* ctx, size_t ctx_bytes, void* dX, void* dW_gate,
                           void* dW_up, void* dW_down, float* dW_r, void* ws, size_t ws_bytes, void* stream,
                           bool persistent) {
  Layout L;
  const moe_status cs = check_shape(s, &L);
  if (cs != MOE_OK) return cs;
  const bool tok = s->T > 0;  // with no tokens, X, dY and dX may be empty (NULL)
  if ((tok && (!X || !dY || !dX)) || !W_r || !W_gate || !W_up || !W_down || !ctx || !dW_gate || !dW_up ||
      !dW_down || !dW_r || !ws)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(W_r) || !aligned16(W_gate) || !aligned16(W_up) || !aligned16(W_down) ||
      !aligned16(dY) || !aligned16(ctx) || !aligned16(dX) || !aligned16(dW_gate) || !aligned16(dW_up) ||
      !aligned16(dW_down) || !aligned16(dW_r) || !aligned16(ws))
    return MOE_ERR_INVALID_ARG;
  if (ctx_bytes < L.ctx_bytes || ws_bytes < L.ws_bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ctx c = make_ctx(L, ctx, ws);
  if (L.T == 0) return zero_wgrads(L, dW_gate, dW_up, dW_down, dW_r, st);  // no tokens: all zero
  const int grid = num_sms();
  int* status = c.hdr + HDR_STATUS;
  const uint64_t RP = static_cast<uint64_t>(L.RP);
  const uint64_t El = static_cast<uint64_t>(L.El);

  // 8. reverse-combine: dY into the expert-contiguous layout
  MOE_TRY(timed(K_REV_COMBINE, st, [&] { return launch_gather_rows(L, c, static_cast<const __nv_bfloat16*>(dY), c.dyperm, st); }));
  // 9. dgrad of the down projection + SwiGLU backward + router-gate gradient partials
  GemmParams p9 = base_params(L, c, status);
  MOE_TMAP(tmap_2d(&p9.ta0, c.dyperm, L.d, RP, L.d, 64, 128));
  MOE_TMAP(tmap_2d(&p9.tb0, W_down, L.d, El * L.I, L.d, 64, 256));
  p9.ta1 = p9.ta0;
  p9.tb1 = p9.tb0;
  p9.in0 = c.abuf;
  p9.in1 = c.bbuf;
  p9.out0 = c.dabuf;
  p9.out1 = c.dbbuf;
  p9.out2 = c.hgbuf;
  p9.outf = c.dgpart;
  // 11. dgrad of gate/up
  GemmParams p11 = base_params(L, c, status);
  MOE_TMAP(tmap_2d(&p11.ta0, c.dabuf, L.I, RP, L.I, 64, 128));
  MOE_TMAP(tmap_2d(&p11.ta1, c.dbbuf, L.I, RP, L.I, 64, 128));
  MOE_TMAP(tmap_2d(&p11.tb0, W_gate, L.I, El * L.d, L.I, 64, 256));
  MOE_TMAP(tmap_2d(&p11.tb1, W_up, L.I, El * L.d, L.I, 64, 256));
  p11.out0 = c.dxperm;
  if (persistent) {
    MOE_TRY(timed(K_PAIR_DGRAD, st, [&] { return run_gemm_pair(L, c, PAIR_DGRAD, p9, p11, st); }));
    // 10. router backward: dl, then dW_r = X^T DL (tensor cores); W_r^T for the dX router term
    MOE_TRY_STATUS(router_backward(L, c, X, dW_r, status, st));
    MOE_TRY(timed(K_TRANSPOSE_WR, st, [&] {
      return launch_transpose_wr(L, static_cast<const __nv_bfloat16*>(W_r), c.wrt, st);
    }));
  } else {
    MOE_TRY(timed(K_GEMM_DGRAD_DOWN, st, [&] { return launch_gemm(G_DGRAD_DOWN, p9, grid, st); }));
    // 10. router backward: dl, then dW_r = X^T DL (tensor cores); W_r^T for the dX router term
    MOE_TRY_STATUS(router_backward(L, c, X, dW_r, status, st));
    MOE_TRY(timed(K_TRANSPOSE_WR, st, [&] {
      return launch_transpose_wr(L, static_cast<const __nv_bfloat16*>(W_r), c.wrt, st);
    }));
    MOE_TRY(timed(K_GEMM_DGRAD_GATEUP, st, [&] { return launch_gemm(G_DGRAD_GATEUP, p11, grid, st); }));
  }
  // 12. reverse-dispatch (+ router term dl W_r^T)
  MOE_TRY(timed(K_REV_DISPATCH, st, [&] { return launch_rev_dispatch(L, c, static_cast<__nv_bfloat16*>(dX), st); }));
  // 13. wgrad
  return launch_wgrads(L, c, status, dW_gate, dW_up, dW_down, st);
}

moe_status moe_bwd(const moe_shape* s, const void* X, const void* W_r, const void* W_gate, const void* W_up,
                   const void* W_down, const void* dY, void* ctx, size_t ctx_bytes, void* dX, void* dW_gate,
                   void* dW_up, void* dW_down, float* dW_r, void* ws, size_t ws_bytes, void* stream) {
  return bwd_impl(s, X, W_r, W_gate, W_up, W_down, dY, ctx, ctx_bytes, dX, dW_gate, dW_up, dW_down, dW_r, ws,
                  ws_bytes, stream, false);
}

moe_status moe_bwd_persistent(const moe_shape* s, const void* X, const void* W_r, const void* W_gate,
                              const void* W_up, const void* W_down, const void* dY, void* ctx, size_t ctx_bytes,
                              void* dX, void* dW_gate, void* dW_up, void* dW_down, float* dW_r, void* ws,
                              size_t ws_bytes, void* stream) {
  return bwd_impl(s, X, W_r, W_gate, W_up, W_down, dY, ctx, ctx_bytes, dX, dW_gate, dW_up, dW_down, dW_r, ws,
                  ws_bytes, stream, true);
}

moe_status moe_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_prof_on = on != 0;
  return MOE_OK;
}

int moe_profile_read(int max_kernels, double* total_ms, int* launches) {
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  std::lock_guard<std::mutex> lk(g_mu);
  for (int i = 0; i < max_kernels && i < K_NUM; ++i) {
    if (total_ms) total_ms[i] = 0.0;
    if (launches) launches[i] = 0;
  }
  for (const ProfRec& r : g_prof) {
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess && r.kid < max_kernels) {
      if (total_ms) total_ms[r.kid] += ms;
      if (launches) launches[r.kid] += 1;
    }
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_prof.clear();
  return K_NUM;
}

const char* moe_kernel_name(int kernel_id) {
  return (kernel_id >= 0 && kernel_id < K_NUM) ? kKernelNames[kernel_id] : "";
}

unsigned long long moe_kernel_launches(void) { return g_launches.load(); }

// ---------------------------------------------------------------------------
// Ring-streamed layer: M minibatches of shape->T tokens through a fixed ring
// ---------------------------------------------------------------------------
// prec: MOE_BF16 for the bf16 entry points, MOE_MXFP8 for the MXFP8 ones (MOE_MXFP8 or
// MOE_MXFP8_ALL shapes), -1 for any (sizes, debug).
static moe_status check_stream(const moe_shape* s, int32_t M, Layout* L, int32_t prec = MOE_BF16) {
  if (!s || M <= 0) return MOE_ERR_INVALID_ARG;
  if (s->prec != MOE_BF16 && !is_mx_prec(s->prec)) return MOE_ERR_INVALID_ARG;
  if (prec == MOE_BF16 && s->prec != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (prec == MOE_MXFP8 && !is_mx_prec(s->prec)) return MOE_ERR_UNSUPPORTED;
  if (!make_layout(*s, L, M)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

// Worst-case padded rows of one minibatch: every macrobatch must fit in the ring.
static int64_t minibatch_rows(const Layout& L) {
  const int64_t kl = L.k < L.El ? L.k : L.El;
  return static_cast<int64_t>(align_up(static_cast<size_t>(L.T_mb * kl + int64_t(kPad - 1) * L.El), kPad));
}

size_t moe_stream_ctx_size(const moe_shape* s, int32_t M) {
  Layout L;
  if (check_stream(s, M, &L, -1) != MOE_OK) return 0;
  return L.ctx_bytes;
}

size_t moe_stream_workspace_size(const moe_shape* s, int32_t M) {
  Layout L;
  if (check_stream(s, M, &L, -1) != MOE_OK) return 0;
  return L.ws_bytes;
}

// Bytes of the caller's ring per row: the bf16 row (the bf16 weight gradients' operand, replayed),
// and in MXFP8 its codes along d and their scales (ring_rows bf16 rows, then ring_rows code rows,
// then their scale chunks); with MXFP8 weight gradients the codes only (X's codes along the rows
// are kept at their padded rows, so nothing is replayed).
static size_t ring_row_bytes(const Layout& L) {
  const size_t codes = L.mx ? static_cast<size_t>(L.d) + L.d / 32 : 0;
  return (L.mxw ? 0 : static_cast<size_t>(L.d) * 2) + codes;
}
// Rows of a ring of ring_bytes; in MXFP8 a multiple of 128 (the scale chunks cover 128-row tiles).
static int64_t ring_rows_of(const Layout& L, size_t ring_bytes) {
  const int64_t r = static_cast<int64_t>(ring_bytes / ring_row_bytes(L));
  return L.mx ? r / 128 * 128 : r;
}

size_t moe_stream_min_ring_bytes(const moe_shape* s) {
  Layout L;
  if (check_stream(s, 1, &L, -1) != MOE_OK) return 0;
  return static_cast<size_t>(minibatch_rows(L)) * ring_row_bytes(L);
}

moe_status moe_fwd_stream(const moe_shape* s, int32_t M, const void* X, const void* W_r, const float* bias,
                          const void* W_gate, const void* W_up, const void* W_down, void* Y, void* ctx,
                          size_t ctx_bytes, void* ring, size_t ring_bytes, void* ws, size_t ws_bytes, void* stream) {
  Layout L;
  const moe_status cs = check_stream(s, M, &L);
  if (cs != MOE_OK) return cs;
  if (!X || !Y || !W_r || !W_gate || !W_up || !W_down || !ctx || !ring || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(W_r) || !aligned16(W_gate) || !aligned16(W_up) || !aligned16(W_down) ||
      !aligned16(Y) || !aligned16(ctx) || !aligned16(ring) || !aligned16(ws) ||
      (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)))
    return MOE_ERR_INVALID_ARG;
  const int64_t ring_rows = static_cast<int64_t>(ring_bytes / (static_cast<size_t>(L.d) * 2));
  if (ctx_bytes < L.ctx_bytes || ws_bytes < L.ws_bytes || ring_rows < minibatch_rows(L) ||
      ring_rows >= (int64_t(1) << 31))
    return MOE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ctx c = make_ctx(L, ctx, ws);
  MOE_TRY(cudaMemsetAsync(c.hdr, 0, HDR_WORDS * 4, st));
  {
    const moe_status r = route_tokens(L, c, X, W_r, bias, static_cast<int>(ring_rows), st);
    if (r != MOE_OK) return r;
  }
  int* status = c.hdr + HDR_STATUS;
  const uint64_t RP = static_cast<uint64_t>(L.RP);
  const int El = L.El;
  CUtensorMap ring_map, wg_map, wu_map, h_map, wd_map;
  MOE_TMAP(tmap_2d(&ring_map, ring, L.d, static_cast<uint64_t>(ring_rows), L.d, 64, 128));
  MOE_TMAP(tmap_2d(&wg_map, W_gate, L.I, static_cast<uint64_t>(El) * L.d, L.I, 64, 64));
  MOE_TMAP(tmap_2d(&wu_map, W_up, L.I, static_cast<uint64_t>(El) * L.d, L.I, 64, 64));
  MOE_TMAP(tmap_2d(&h_map, c.hbuf, L.I, RP, L.I, 64, 128));
  MOE_TMAP(tmap_2d(&wd_map, W_down, L.d, static_cast<uint64_t>(El) * L.I, L.d, 64, 64));
  // Macrobatches walk the ring forward.  The host enqueues M of them (the most
  // the plan can form); launches past the plan's count find empty segments and exit.
  for (int m = 0; m < M; ++m) {
    const int* seg = c.tab.seg_poff + m * El;
    MOE_TRY(timed(K_DISPATCH, st, [&] {
      return launch_gather_range(L, c, static_cast<const __nv_bfloat16*>(X), seg, seg + El, c.tab.shift_fwd + m,
                                 ring_rows, static_cast<__nv_bfloat16*>(ring), st);
    }));
    GemmParams p = base_params(L, c, status);
    p.poff = seg;
    p.nseg = El;
    p.ta0 = ring_map;
    p.ta1 = ring_map;
    p.tb0 = wg_map;
    p.tb1 = wu_map;
    p.ring_shift = c.tab.shift_fwd + m;
    p.out0 = c.abuf;
    p.out1 = c.bbuf;
    p.out2 = c.hbuf;
    GemmParams q = base_params(L, c, status);
    q.poff = seg;
    q.nseg = El;
    q.ta0 = q.ta1 = h_map;
    q.tb0 = q.tb1 = wd_map;
    q.out0 = c.obuf;
    // gate/up then down as one persistent launch (the down tiles start while the macrobatch's
    // last gate/up tiles run; measured 2-3% faster per step than two launches at n = 512-2368)
    MOE_TRY(timed(K_PAIR_FWD, st, [&] { return run_gemm_pair(L, c, PAIR_FWD, p, q, st); }));
    MOE_TRY(timed(K_COMBINE, st, [&] {
      return launch_combine(L, c, c.obuf, static_cast<__nv_bfloat16*>(Y), st, c.tab.mb_range + 2 * m);
    }));
  }
  return MOE_OK;
}

static moe_status stream_wgrads(const Layout& L, const Ctx& c, int* status, const void* X, void* ring,
                                int64_t ring_rows, void* dW_gate, void* dW_up, void* dW_down, cudaStream_t st);
static moe_status launch_wgrads_mx(const Layout& L, const Ctx& c, int* status, void* dW_gate, void* dW_up,
                                   void* dW_down, cudaStream_t st);

moe_status moe_bwd_stream(const moe_shape* s, int32_t M, const void* X, const void* W_r, const void* W_gate,
                          const void* W_up, const void* W_down, const void* dY, void* ctx, size_t ctx_bytes, void* dX,
                          void* dW_gate, void* dW_up, void* dW_down, float* dW_r, void* ring, size_t ring_bytes,
                          void* ws, size_t ws_bytes, void* stream) {
  Layout L;
  const moe_status cs = check_stream(s, M, &L);
  if (cs != MOE_OK) return cs;
  if (!X || !dY || !dX || !W_r || !W_gate || !W_up || !W_down || !ctx || !dW_gate || !dW_up || !dW_down || !dW_r ||
      !ring || !ws)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(W_r) || !aligned16(W_gate) || !aligned16(W_up) || !aligned16(W_down) ||
      !aligned16(dY) || !aligned16(ctx) || !aligned16(dX) || !aligned16(dW_gate) || !aligned16(dW_up) ||
      !aligned16(dW_down) || !aligned16(dW_r) || !aligned16(ring) || !aligned16(ws))
    return MOE_ERR_INVALID_ARG;
  const int64_t ring_rows = static_cast<int64_t>(ring_bytes / (static_cast<size_t>(L.d) * 2));
  if (ctx_bytes < L.ctx_bytes || ws_bytes < L.ws_bytes || ring_rows < minibatch_rows(L) ||
      ring_rows >= (int64_t(1) << 31))
    return MOE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ctx c = make_ctx(L, ctx, ws);
  int* status = c.hdr + HDR_STATUS;
  const uint64_t RP = static_cast<uint64_t>(L.RP);
  const uint64_t El = static_cast<uint64_t>(L.El);
  const int nseg = L.M * L.El;

  // dgrad path over every row of the stream (no X_perm needed)
  MOE_TRY(timed(K_REV_COMBINE, st, [&] {
    return launch_gather_rows(L, c, static_cast<const __nv_bfloat16*>(dY), c.dyperm, st);
  }));
  // dgrad of W_down (SwiGLU backward, router-gate partials) then dgrad of gate/up, as one
  // persistent launch over every row of the stream; the router backward follows it
  GemmParams p9 = base_params(L, c, status);
  p9.poff = c.tab.seg_poff;
  p9.cum = c.tab.cum;
  p9.nseg = nseg;
  MOE_TMAP(tmap_2d(&p9.ta0, c.dyperm, L.d, RP, L.d, 64, 128));
  MOE_TMAP(tmap_2d(&p9.tb0, W_down, L.d, El * L.I, L.d, 64, 256));
  p9.ta1 = p9.ta0;
  p9.tb1 = p9.tb0;
  p9.in0 = c.abuf;
  p9.in1 = c.bbuf;
  p9.out0 = c.dabuf;
  p9.out1 = c.dbbuf;
  p9.out2 = c.hgbuf;
  p9.outf = c.dgpart;
  GemmParams p11 = base_params(L, c, status);
  p11.poff = c.tab.seg_poff;
  p11.cum = c.tab.cum;
  p11.nseg = nseg;
  MOE_TMAP(tmap_2d(&p11.ta0, c.dabuf, L.I, RP, L.I, 64, 128));
  MOE_TMAP(tmap_2d(&p11.ta1, c.dbbuf, L.I, RP, L.I, 64, 128));
  MOE_TMAP(tmap_2d(&p11.tb0, W_gate, L.I, El * L.d, L.I, 64, 256));
  MOE_TMAP(tmap_2d(&p11.tb1, W_up, L.I, El * L.d, L.I, 64, 256));
  p11.out0 = c.dxperm;
  MOE_TRY(timed(K_PAIR_DGRAD, st, [&] { return run_gemm_pair(L, c, PAIR_DGRAD, p9, p11, st); }));
  MOE_TRY_STATUS(router_backward(L, c, X, dW_r, status, st));
  MOE_TRY(timed(K_TRANSPOSE_WR, st, [&] {
    return launch_transpose_wr(L, static_cast<const __nv_bfloat16*>(W_r), c.wrt, st);
  }));
  MOE_TRY(timed(K_REV_DISPATCH, st, [&] { return launch_rev_dispatch(L, c, static_cast<__nv_bfloat16*>(dX), st); }));
  return stream_wgrads(L, c, status, X, ring, ring_rows, dW_gate, dW_up, dW_down, st);
}

// Weight gradients of a ring-streamed backward: W_down's over every row of the stream (Hg and
// dY_perm), W_gate / W_up's walking the ring in reverse, chunk by chunk (replaying the macrobatches
// the forward overwrote), into the fp32 accumulator, then rounded once.
static moe_status stream_wgrads(const Layout& L, const Ctx& c, int* status, const void* X, void* ring,
                                int64_t ring_rows, void* dW_gate, void* dW_up, void* dW_down, cudaStream_t st) {
  const int grid = num_sms();
  const uint64_t RP = static_cast<uint64_t>(L.RP), El = static_cast<uint64_t>(L.El);
  const int nseg = L.M * L.El;
  {  // wgrad of W_down: Hg and dY_perm cover the whole stream
    GemmParams p = base_params(L, c, status);
    p.poff = c.tab.seg_poff;
    p.cum = c.tab.cum;
    p.nseg = nseg;
    MOE_TMAP(tmap_2d(&p.ta0, c.hgbuf, L.I, RP, L.I, 64, 64));
    MOE_TMAP(tmap_2d(&p.tb0, c.dyperm, L.d, RP, L.d, 64, 64));
    MOE_TMAP(tmap_wgrad_out(L, &p.to0, dW_down, L.d, El * L.I));
    p.to1 = p.to0;
    p.ta1 = p.ta0;
    p.tb1 = p.tb0;
    MOE_TRY(timed(K_GEMM_WGRAD_DOWN, st, [&] { return launch_gemm(G_WGRAD_DOWN, p, grid, st); }));
  }
  // wgrad of W_gate / W_up needs X_perm: walk the ring in reverse, chunk by chunk
  {
    GemmParams p = base_params(L, c, status);
    p.poff = c.tab.seg_poff;
    p.cum = c.tab.cum;
    p.nseg = nseg;
    p.ring_shift = c.tab.shift_bwd;
    p.acc32 = c.acc32;
    MOE_TMAP(tmap_2d(&p.ta0, ring, L.d, static_cast<uint64_t>(ring_rows), L.d, 64, 64));
    MOE_TMAP(tmap_2d(&p.tb0, c.dabuf, L.I, RP, L.I, 64, 64));
    MOE_TMAP(tmap_2d(&p.tb1, c.dbbuf, L.I, RP, L.I, 64, 64));
    MOE_TMAP(tmap_wgrad_out(L, &p.to0, dW_gate, L.I, El * L.d));
    MOE_TMAP(tmap_wgrad_out(L, &p.to1, dW_up, L.I, El * L.d));
    MOE_TMAP(tmap_f32(&p.tacc, c.acc32, L.I, 2 * El * L.d));  // fp32 accumulator [2 * El * d, I]
    p.ta1 = p.ta0;
    for (int ch = 0; ch < L.M; ++ch) {
      MOE_TRY(timed(K_REPLAY, st, [&] {
        return launch_replay(L, c, ch, static_cast<const __nv_bfloat16*>(X), static_cast<__nv_bfloat16*>(ring),
                             ring_rows, st);
      }));
      p.chunk = c.tab.chunk + 4 * ch;
      MOE_TRY(timed(K_GEMM_WGRAD_GATEUP, st, [&] { return launch_gemm(G_WGRAD_GATEUP, p, grid, st); }));
    }
  }
  MOE_TRY(timed(K_FINISH_ACC, st, [&] { return launch_finish_acc(L, c, dW_gate, dW_up, st); }));
  return MOE_OK;
}

// MXFP8 ring-streamed layer: the bf16 stream's macrobatches, ring and backward chunks, with the
// gate/up, down and both dgrad GEMMs on the MX engine.  The forward's dispatch writes each
// macrobatch's rows to the ring in bf16 (the weight gradients' operand, replayed as in the bf16
// stream) and their codes along d to the same ring rows of the ring's code region (the gate/up
// GEMM's operand; ring positions are multiples of 128 rows, so the scale chunks stay whole).
static moe_status check_stream_mx_args(const moe_shape* s, int32_t M, Layout* L, const void* wq, size_t wq_bytes,
                                       size_t ctx_bytes, size_t ws_bytes, size_t ring_bytes, int64_t* ring_rows) {
  const moe_status cs = check_stream(s, M, L, MOE_MXFP8);
  if (cs != MOE_OK) return cs;
  if (!wq || !aligned16(wq)) return MOE_ERR_INVALID_ARG;
  *ring_rows = ring_rows_of(*L, ring_bytes);
  if (ctx_bytes < L->ctx_bytes || ws_bytes < L->ws_bytes || wq_bytes < L->wq_bytes ||
      *ring_rows < minibatch_rows(*L) || *ring_rows >= (int64_t(1) << 31))
    return MOE_ERR_WORKSPACE_TOO_SMALL;
  return MOE_OK;
}

moe_status moe_fwd_stream_mx(const moe_shape* s, int32_t M, const void* X, const void* W_r, const float* bias,
                             const void* wq, size_t wq_bytes, void* Y, void* ctx, size_t ctx_bytes, void* ring,
                             size_t ring_bytes, void* ws, size_t ws_bytes, void* stream) {
  Layout L;
  int64_t ring_rows = 0;
  if (!s) return MOE_ERR_INVALID_ARG;
  if (!X || !Y || !W_r || !ctx || !ring || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(W_r) || !aligned16(Y) || !aligned16(ctx) || !aligned16(ring) || !aligned16(ws) ||
      (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)))
    return MOE_ERR_INVALID_ARG;
  const moe_status cs = check_stream_mx_args(s, M, &L, wq, wq_bytes, ctx_bytes, ws_bytes, ring_bytes, &ring_rows);
  if (cs != MOE_OK) return cs;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ctx c = make_ctx(L, ctx, ws);
  MOE_TRY(cudaMemsetAsync(c.hdr, 0, HDR_WORDS * 4, st));
  {
    const moe_status r = route_tokens(L, c, X, W_r, bias, static_cast<int>(ring_rows), st);
    if (r != MOE_OK) return r;
  }
  const int grid = num_sms();
  int* status = c.hdr + HDR_STATUS;
  const uint64_t RP = static_cast<uint64_t>(L.RP), El = static_cast<uint64_t>(L.El);
  const auto* w = static_cast<const uint8_t*>(wq);
  // the ring: ring_rows bf16 rows (not with MXFP8 weight gradients), their codes, the codes' scale chunks
  uint8_t* ring_q = static_cast<uint8_t*>(ring) + (L.mxw ? 0 : static_cast<size_t>(ring_rows) * L.d * 2);
  uint8_t* ring_qs = ring_q + static_cast<size_t>(ring_rows) * L.d;
  CUtensorMap xq_map, wgu_map, hq_map, wd_map;
  MOE_TMAP(tmap_fp8(&xq_map, ring_q, L.d, static_cast<uint64_t>(ring_rows), 128));
  MOE_TMAP(tmap_fp8(&wgu_map, w + L.wgu1, L.d, El * 2 * L.I, mx_bn(MX_GATEUP)));
  MOE_TMAP(tmap_fp8(&hq_map, c.hq, L.I, RP, 128));
  MOE_TMAP(tmap_fp8(&wd_map, w + L.wd2, L.I, El * L.d, mx_bn(MX_DOWN)));
  // Macrobatches walk the ring forward; launches past the plan's count find empty segments and exit.
  for (int m = 0; m < M; ++m) {
    const int* seg = c.tab.seg_poff + m * L.El;
    MOE_TRY(timed(K_DISPATCH, st, [&] {
      if (L.mxw)  // codes along d to the ring, codes along the rows (weight gradients) at the padded rows
        return launch_gather_quant2_range(L, c, static_cast<const __nv_bfloat16*>(X), seg, seg + L.El,
                                          c.tab.shift_fwd + m, ring_q, ring_qs, c.xqt, c.xqts, st);
      return launch_gather_range_mx(L, c, static_cast<const __nv_bfloat16*>(X), seg, seg + L.El,
                                    c.tab.shift_fwd + m, true, ring_rows, static_cast<__nv_bfloat16*>(ring), ring_q,
                                    ring_qs, st);
    }));
    {
      MxParams p = mx_params(L, c, status);
      p.poff = seg;
      p.ring_shift = c.tab.shift_fwd + m;
      p.ta0 = p.ta1 = xq_map;
      p.tb0 = p.tb1 = wgu_map;
      p.sfa0 = p.sfa1 = ring_qs;
      p.sfb0 = p.sfb1 = w + L.wgu1s;
      p.out0 = c.abuf;
      p.out1 = c.bbuf;
      p.q0 = c.hq;
      p.qs0 = c.hqs;
      MOE_TRY(timed(K_GEMM_GATEUP, st, [&] { return launch_gemm_mx(MX_GATEUP, p, grid, st); }));
    }
    {
      MxParams p = mx_params(L, c, status);
      p.poff = seg;
      p.ta0 = p.ta1 = hq_map;
      p.tb0 = p.tb1 = wd_map;
      p.sfa0 = p.sfa1 = c.hqs;
      p.sfb0 = p.sfb1 = w + L.wd2s;
      p.out0 = c.obuf;
      MOE_TRY(timed(K_GEMM_DOWN, st, [&] { return launch_gemm_mx(MX_DOWN, p, grid, st); }));
    }
    MOE_TRY(timed(K_COMBINE, st, [&] {
      return launch_combine(L, c, c.obuf, static_cast<__nv_bfloat16*>(Y), st, c.tab.mb_range + 2 * m);
    }));
  }
  return MOE_OK;
}

moe_status moe_bwd_stream_mx(const moe_shape* s, int32_t M, const void* X, const void* W_r, const void* wq,
                             size_t wq_bytes, const void* dY, void* ctx, size_t ctx_bytes, void* dX, void* dW_gate,
                             void* dW_up, void* dW_down, float* dW_r, void* ring, size_t ring_bytes, void* ws,
                             size_t ws_bytes, void* stream) {
  Layout L;
  int64_t ring_rows = 0;
  if (!s) return MOE_ERR_INVALID_ARG;
  if (!X || !dY || !dX || !W_r || !ctx || !dW_gate || !dW_up || !dW_down || !dW_r || !ring || !ws)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(W_r) || !aligned16(dY) || !aligned16(ctx) || !aligned16(dX) ||
      !aligned16(dW_gate) || !aligned16(dW_up) || !aligned16(dW_down) || !aligned16(dW_r) || !aligned16(ring) ||
      !aligned16(ws))
    return MOE_ERR_INVALID_ARG;
  const moe_status cs = check_stream_mx_args(s, M, &L, wq, wq_bytes, ctx_bytes, ws_bytes, ring_bytes, &ring_rows);
  if (cs != MOE_OK) return cs;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ctx c = make_ctx(L, ctx, ws);
  const int grid = num_sms();
  int* status = c.hdr + HDR_STATUS;
  const uint64_t RP = static_cast<uint64_t>(L.RP), El = static_cast<uint64_t>(L.El);
  const int nseg = L.M * L.El;
  const auto* w = static_cast<const uint8_t*>(wq);
  // reverse-combine over every row of the stream: codes along d (the dgrad of W_down's operand) and
  // bf16 (the W_down weight gradient's operand), or codes along the rows with MXFP8 weight gradients
  MOE_TRY(timed(K_REV_COMBINE, st, [&] {
    if (L.mxw)
      return launch_gather_quant2(L, c, static_cast<const __nv_bfloat16*>(dY), c.dyq, c.dyqs, c.dyqt, c.dyqts, st);
    return launch_gather_rows_mx(L, c, static_cast<const __nv_bfloat16*>(dY), c.dyperm, c.dyq, c.dyqs, st);
  }));
  {
    MxParams p = mx_params(L, c, status);
    p.poff = c.tab.seg_poff;
    p.nseg = nseg;
    MOE_TMAP(tmap_fp8(&p.ta0, c.dyq, L.d, RP, 128));
    MOE_TMAP(tmap_fp8(&p.tb0, w + L.wd3, L.d, El * L.I, mx_bn(MX_DGRAD_DOWN)));
    p.ta1 = p.ta0;
    p.tb1 = p.tb0;
    p.sfa0 = p.sfa1 = c.dyqs;
    p.sfb0 = p.sfb1 = w + L.wd3s;
    p.in0 = c.abuf;
    p.in1 = c.bbuf;
    if (L.mxw) {  // dA, dB, Hg along the rows, from fp32, for the MXFP8 weight gradients
      p.tq[0] = c.daqt;
      p.tq[1] = c.dbqt;
      p.tq[2] = c.hgqt;
      p.tqs[0] = c.daqts;
      p.tqs[1] = c.dbqts;
      p.tqs[2] = c.hgqts;
    } else {
      p.out0 = c.dabuf;
      p.out1 = c.dbbuf;
      p.out2 = c.hgbuf;
    }
    p.q0 = c.daq;
    p.qs0 = c.daqs;
    p.q1 = c.dbq;
    p.qs1 = c.dbqs;
    p.outf = c.dgpart;
    MOE_TRY(timed(K_GEMM_DGRAD_DOWN, st, [&] { return launch_gemm_mx(MX_DGRAD_DOWN, p, grid, st); }));
  }
  MOE_TRY_STATUS(router_backward(L, c, X, dW_r, status, st, L.I / mx_bn(MX_DGRAD_DOWN)));
  MOE_TRY(timed(K_TRANSPOSE_WR, st, [&] {
    return launch_transpose_wr(L, static_cast<const __nv_bfloat16*>(W_r), c.wrt, st);
  }));
  {
    MxParams p = mx_params(L, c, status);
    p.poff = c.tab.seg_poff;
    p.nseg = nseg;
    MOE_TMAP(tmap_fp8(&p.ta0, c.daq, L.I, RP, 128));
    MOE_TMAP(tmap_fp8(&p.ta1, c.dbq, L.I, RP, 128));
    MOE_TMAP(tmap_fp8(&p.tb0, w + L.wg4, L.I, El * L.d, mx_bn(MX_DGRAD_GATEUP)));
    MOE_TMAP(tmap_fp8(&p.tb1, w + L.wu4, L.I, El * L.d, mx_bn(MX_DGRAD_GATEUP)));
    p.sfa0 = c.daqs;
    p.sfa1 = c.dbqs;
    p.sfb0 = w + L.wg4s;
    p.sfb1 = w + L.wu4s;
    p.out0 = c.dxperm;
    MOE_TRY(timed(K_GEMM_DGRAD_GATEUP, st, [&] { return launch_gemm_mx(MX_DGRAD_GATEUP, p, grid, st); }));
  }
  MOE_TRY(timed(K_REV_DISPATCH, st, [&] { return launch_rev_dispatch(L, c, static_cast<__nv_bfloat16*>(dX), st); }));
  // MXFP8 weight gradients over every segment of the stream (no replay: X's codes along the rows
  // are kept at the padded rows), or bf16 ones exactly as the bf16 stream: W_down's over every row,
  // gate/up's walking the ring in reverse, chunk by chunk, into the fp32 accumulator
  if (L.mxw) return launch_wgrads_mx(L, c, status, dW_gate, dW_up, dW_down, st);
  return stream_wgrads(L, c, status, X, ring, ring_rows, dW_gate, dW_up, dW_down, st);
}

moe_status moe_debug_stream_plan(const moe_shape* s, int32_t M, const void* ctx, int32_t* tables, void* stream) {
  Layout L;
  const moe_status cs = check_stream(s, M, &L, -1);
  if (cs != MOE_OK) return cs;
  if (!ctx || !tables) return MOE_ERR_INVALID_ARG;
  MOE_TRY(cudaMemcpyAsync(tables, static_cast<const char*>(ctx) + L.stab,
                          static_cast<size_t>(stream_table_words(M, L.El)) * 4, cudaMemcpyDeviceToDevice,
                          static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// MXFP8 mode
// ---------------------------------------------------------------------------
static moe_status check_shape_nv(const moe_shape* s, Layout* L) {
  if (!s) return MOE_ERR_INVALID_ARG;
  if (s->prec != MOE_NVFP4) return MOE_ERR_INVALID_ARG;
  if (s->T < 0 || s->d <= 0 || s->E <= 0 || s->I <= 0 || s->top_k <= 0 || s->first_local_expert < 0 ||
      s->num_local_experts < 0)
    return MOE_ERR_INVALID_ARG;
  if (!make_layout(*s, L)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

size_t moe_weights_size(const moe_shape* s) {
  Layout L;
  if (s && s->prec == MOE_NVFP4) return check_shape_nv(s, &L) == MOE_OK ? L.wq_bytes : 0;
  if (check_shape_mx(s, &L) != MOE_OK) return 0;
  return L.wq_bytes;
}

// NVFP4 weights: amax of each tensor (the local experts' W_gate, W_up, W_down), their global
// scales, then the gate/up B operand (K = d, 64-row gate / up blocks) and W_down^T (K = I).
static moe_status prepare_weights_nv(const moe_shape* s, const void* W_gate, const void* W_up, const void* W_down,
                                     void* wq, size_t wq_bytes, cudaStream_t st) {
  Layout L;
  const moe_status cs = check_shape_nv(s, &L);
  if (cs != MOE_OK) return cs;
  if (!W_gate || !W_up || !W_down || !wq) return MOE_ERR_INVALID_ARG;
  if (!aligned16(W_gate) || !aligned16(W_up) || !aligned16(W_down) || !aligned16(wq)) return MOE_ERR_INVALID_ARG;
  if (wq_bytes < L.wq_bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  auto* w = static_cast<uint8_t*>(wq);
  float* gs = reinterpret_cast<float*>(w + L.wnvgs);
  unsigned* amx = reinterpret_cast<unsigned*>(w + L.wnvgs + 64);
  const auto* g = static_cast<const __nv_bfloat16*>(W_gate);
  const auto* u = static_cast<const __nv_bfloat16*>(W_up);
  const auto* dn = static_cast<const __nv_bfloat16*>(W_down);
  const int64_t n = static_cast<int64_t>(L.El) * L.d * L.I;
  MOE_TRY(cudaMemsetAsync(amx, 0, 4 * sizeof(unsigned), st));
  MOE_TRY(timed(K_QUANT_WEIGHTS, st, [&] {  // gate, up, down, and [gate | up] for the dgrad of gate/up
    cudaError_t e = launch_nv_amax(g, n, amx, st);
    if (e == cudaSuccess) e = launch_nv_amax(u, n, amx + 1, st);
    if (e == cudaSuccess) e = launch_nv_amax(dn, n, amx + 2, st);
    if (e == cudaSuccess) e = launch_nv_amax(g, n, amx + 3, st);
    if (e == cudaSuccess) e = launch_nv_amax(u, n, amx + 3, st);
    if (e == cudaSuccess) e = launch_nv_scale(amx, gs, 4, st);
    return e;
  }));
  MOE_TRY(timed(K_QUANT_WEIGHTS, st, [&] {
    return launch_nv_quant_weight(true, g, u, L.El, L.d, L.I, gs, w + L.wgu1, w + L.wgu1s, st);
  }));
  MOE_TRY(timed(K_QUANT_WEIGHTS, st, [&] {
    return launch_nv_quant_weight(false, dn, nullptr, L.El, L.I, L.d, gs + 2, w + L.wd2, w + L.wd2s, st);
  }));
  // the backward's layouts, as stored: W_down [El*I, d] (K = d), W_gate, W_up [El*d, I] (K = I)
  MOE_TRY(timed(K_QUANT_WEIGHTS, st, [&] {
    cudaError_t e = launch_nv_quant_rows(dn, static_cast<int64_t>(L.El) * L.I, L.d, gs + 2, w + L.wd3, w + L.wd3s, st);
    if (e == cudaSuccess)
      e = launch_nv_quant_rows(g, static_cast<int64_t>(L.El) * L.d, L.I, gs + 3, w + L.wg4, w + L.wg4s, st);
    if (e == cudaSuccess)
      e = launch_nv_quant_rows(u, static_cast<int64_t>(L.El) * L.d, L.I, gs + 3, w + L.wu4, w + L.wu4s, st);
    return e;
  }));
  return MOE_OK;
}

moe_status moe_prepare_weights(const moe_shape* s, const void* W_gate, const void* W_up, const void* W_down, void* wq,
                               size_t wq_bytes, void* stream) {
  if (s && s->prec == MOE_NVFP4)
    return prepare_weights_nv(s, W_gate, W_up, W_down, wq, wq_bytes, static_cast<cudaStream_t>(stream));
  Layout L;
  const moe_status cs = check_shape_mx(s, &L);
  if (cs != MOE_OK) return cs;
  if (!W_gate || !W_up || !W_down || !wq) return MOE_ERR_INVALID_ARG;
  if (!aligned16(W_gate) || !aligned16(W_up) || !aligned16(W_down) || !aligned16(wq)) return MOE_ERR_INVALID_ARG;
  if (wq_bytes < L.wq_bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto* w = static_cast<uint8_t*>(wq);
  const auto* g = static_cast<const __nv_bfloat16*>(W_gate);
  const auto* u = static_cast<const __nv_bfloat16*>(W_up);
  const auto* dn = static_cast<const __nv_bfloat16*>(W_down);
  const int64_t El = L.El;
  MOE_TRY(timed(K_QUANT_WEIGHTS, st, [&] {  // gate/up for the forward: K = d, 64-row gate/up pairs
    return launch_quant_weight(2, g, u, El * 2 * L.I, L.d, L.I, w + L.wgu1, w + L.wgu1s, st);
  }));
  MOE_TRY(timed(K_QUANT_WEIGHTS, st, [&] {  // down for the forward: K = I (transposed)
    return launch_quant_weight(1, dn, nullptr, El * L.d, L.I, L.d, w + L.wd2, w + L.wd2s, st);
  }));
  MOE_TRY(timed(K_QUANT_WEIGHTS, st, [&] {  // down for the backward: K = d (as stored)
    return launch_quant_weight(0, dn, nullptr, El * L.I, L.d, 0, w + L.wd3, w + L.wd3s, st);
  }));
  MOE_TRY(timed(K_QUANT_WEIGHTS, st, [&] {  // gate for the backward: K = I (as stored)
    return launch_quant_weight(0, g, nullptr, El * L.d, L.I, 0, w + L.wg4, w + L.wg4s, st);
  }));
  MOE_TRY(timed(K_QUANT_WEIGHTS, st, [&] {  // up for the backward: K = I (as stored)
    return launch_quant_weight(0, u, nullptr, El * L.d, L.I, 0, w + L.wu4, w + L.wu4s, st);
  }));
  return MOE_OK;
}


// The row segments an MXFP8 weight gradient contracts over: one per local expert, or in a
// ring-streamed layer one per (macrobatch, expert) with the real rows counted by the stream plan.
static void wgrad_segments(const Layout& L, const Ctx& c, MxParams& p) {
  if (L.M > 0) {
    p.poff = c.tab.seg_poff;
    p.nseg = L.M * L.El;
    p.cum = c.tab.cum;
  }
}

// MXFP8 weight gradients from operands quantised along the rows (blocks of 32 rows of one expert,
// K-major in 128-row tiles): X by the forward's dispatch, dY by the reverse-combine, dA, dB and Hg
// by the dgrad of W_down from its fp32 values.  One grouped GEMM for gate/up and one for down;
// gradients leave through TMA box stores (bf16, or fp32 with MOE_WGRAD_FP32).
static moe_status launch_wgrads_mx(const Layout& L, const Ctx& c, int* status, void* dW_gate, void* dW_up,
                                   void* dW_down, cudaStream_t st) {
  const int grid = num_sms();
  const uint64_t RP = static_cast<uint64_t>(L.RP), El = static_cast<uint64_t>(L.El);
  {
    MxParams p = mx_params(L, c, status);
    // row-quantised operands, 128-row-tile-major: lines of 128 codes, RP / 128 tiles of d (or I) lines
    MOE_TMAP(tmap_fp8(&p.ta0, c.xqt, 128, RP / 128 * L.d, 128));
    MOE_TMAP(tmap_fp8(&p.tb0, c.daqt, 128, RP / 128 * L.I, 256));
    MOE_TMAP(tmap_fp8(&p.tb1, c.dbqt, 128, RP / 128 * L.I, 256));
    MOE_TMAP(tmap_wgrad_out(L, &p.to0, dW_gate, L.I, El * L.d));
    MOE_TMAP(tmap_wgrad_out(L, &p.to1, dW_up, L.I, El * L.d));
    wgrad_segments(L, c, p);
    p.ta1 = p.ta0;
    p.sfa0 = p.sfa1 = c.xqts;
    p.sfb0 = c.daqts;
    p.sfb1 = c.dbqts;
    p.cnt = c.counts + L.first;
    p.wout32 = L.w32 ? 1 : 0;
    MOE_TRY(timed(K_MX_WGRAD_GATEUP, st, [&] { return launch_gemm_mx(MX_WGRAD_GATEUP, p, grid, st); }));
  }
  {
    MxParams p = mx_params(L, c, status);
    MOE_TMAP(tmap_fp8(&p.ta0, c.hgqt, 128, RP / 128 * L.I, 128));
    MOE_TMAP(tmap_fp8(&p.tb0, c.dyqt, 128, RP / 128 * L.d, 256));
    MOE_TMAP(tmap_wgrad_out(L, &p.to0, dW_down, L.d, El * L.I));
    wgrad_segments(L, c, p);
    p.ta1 = p.ta0;
    p.tb1 = p.tb0;
    p.to1 = p.to0;
    p.sfa0 = p.sfa1 = c.hgqts;
    p.sfb0 = p.sfb1 = c.dyqts;
    p.cnt = c.counts + L.first;
    p.wout32 = L.w32 ? 1 : 0;
    MOE_TRY(timed(K_MX_WGRAD_DOWN, st, [&] { return launch_gemm_mx(MX_WGRAD_DOWN, p, grid, st); }));
  }
  return MOE_OK;
}

moe_status moe_debug_mx_wgrad_operand(const moe_shape* s, const void* ctx, const void* ws, int32_t which,
                                      void* codes, void* scales, void* stream) {
  Layout L;
  const moe_status cs = check_shape_mx(s, &L);
  if (cs != MOE_OK) return cs;
  if (!L.mxw || !ctx || !ws || !codes || !scales || which < 0 || which > 4) return MOE_ERR_INVALID_ARG;
  const size_t off[5][2] = {{L.xqt, L.xqts}, {L.dyqt, L.dyqts}, {L.daqt, L.daqts}, {L.dbqt, L.dbqts},
                            {L.hgqt, L.hgqts}};
  const size_t n = static_cast<size_t>(L.RP) * (which < 2 ? L.d : L.I);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const char* w = static_cast<const char*>(which == 0 ? ctx : ws);  // X's codes are saved in ctx
  MOE_TRY(cudaMemcpyAsync(codes, w + off[which][0], n, cudaMemcpyDeviceToDevice, st));
  MOE_TRY(cudaMemcpyAsync(scales, w + off[which][1], n / 32, cudaMemcpyDeviceToDevice, st));
  return MOE_OK;
}

int64_t moe_padded_rows(const moe_shape* s) {
  Layout L;
  if (!s || !make_layout(*s, &L)) return 0;
  return L.RP;
}

moe_status moe_fwd_mx(const moe_shape* s, const void* X, const void* W_r, const float* bias, const void* wq,
                      size_t wq_bytes, void* Y, void* ctx, size_t ctx_bytes, void* ws, size_t ws_bytes,
                      void* stream) {
  Layout L;
  const moe_status cs = check_shape_mx(s, &L);
  if (cs != MOE_OK) return cs;
  const bool tok = s->T > 0;
  if ((tok && (!X || !Y)) || !W_r || !wq || !ctx || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(W_r) || !aligned16(wq) || !aligned16(Y) || !aligned16(ctx) || !aligned16(ws) ||
      (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)))
    return MOE_ERR_INVALID_ARG;
  if (ctx_bytes < L.ctx_bytes || ws_bytes < L.ws_bytes || wq_bytes < L.wq_bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ctx c = make_ctx(L, ctx, ws);
  MOE_TRY(cudaMemsetAsync(c.hdr, 0, HDR_WORDS * 4, st));
  if (L.T == 0) return MOE_OK;
  {
    const moe_status r = route_tokens(L, c, X, W_r, bias, 0, st);
    if (r != MOE_OK) return r;
  }
  MOE_TRY(timed(K_DISPATCH, st, [&] {
    if (L.mxw)  // along d for the gate/up GEMM and along the rows for the weight gradients
      return launch_gather_quant2(L, c, static_cast<const __nv_bfloat16*>(X), c.xq, c.xqs, c.xqt, c.xqts, st);
    return launch_gather_rows_mx(L, c, static_cast<const __nv_bfloat16*>(X), c.xperm, c.xq, c.xqs, st);
  }));
  const int grid = num_sms();
  int* status = c.hdr + HDR_STATUS;
  const uint64_t RP = static_cast<uint64_t>(L.RP), El = static_cast<uint64_t>(L.El);
  const auto* w = static_cast<const uint8_t*>(wq);
  {
    MxParams p = mx_params(L, c, status);
    MOE_TMAP(tmap_fp8(&p.ta0, c.xq, L.d, RP, 128));
    MOE_TMAP(tmap_fp8(&p.tb0, w + L.wgu1, L.d, El * 2 * L.I, mx_bn(MX_GATEUP)));
    p.ta1 = p.ta0;
    p.tb1 = p.tb0;
    p.sfa0 = p.sfa1 = c.xqs;
    p.sfb0 = p.sfb1 = w + L.wgu1s;
    p.out0 = c.abuf;
    p.out1 = c.bbuf;
    p.q0 = c.hq;
    p.qs0 = c.hqs;
    MOE_TRY(timed(K_GEMM_GATEUP, st, [&] { return launch_gemm_mx(MX_GATEUP, p, grid, st); }));
  }
  {
    MxParams p = mx_params(L, c, status);
    MOE_TMAP(tmap_fp8(&p.ta0, c.hq, L.I, RP, 128));
    MOE_TMAP(tmap_fp8(&p.tb0, w + L.wd2, L.I, El * L.d, mx_bn(MX_DOWN)));
    p.ta1 = p.ta0;
    p.tb1 = p.tb0;
    p.sfa0 = p.sfa1 = c.hqs;
    p.sfb0 = p.sfb1 = w + L.wd2s;
    p.out0 = c.obuf;
    MOE_TRY(timed(K_GEMM_DOWN, st, [&] { return launch_gemm_mx(MX_DOWN, p, grid, st); }));
  }
  MOE_TRY(timed(K_COMBINE, st, [&] { return launch_combine(L, c, c.obuf, static_cast<__nv_bfloat16*>(Y), st); }));
  return MOE_OK;
}

// NVFP4 forward: routing as in moe_fwd; X's global scale from its amax; the dispatch quantises
// X along d; the gate/up GEMM writes H in fp32 and its amax; H's global scale; H quantised along
// I; the down GEMM (combine weight in its epilogue); the combine.
moe_status moe_fwd_nvfp4(const moe_shape* s, const void* X, const void* W_r, const float* bias, const void* wq,
                         size_t wq_bytes, void* Y, void* ctx, size_t ctx_bytes, void* ws, size_t ws_bytes,
                         void* stream) {
  Layout L;
  const moe_status cs = check_shape_nv(s, &L);
  if (cs != MOE_OK) return cs;
  const bool tok = s->T > 0;
  if ((tok && (!X || !Y)) || !W_r || !wq || !ctx || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(W_r) || !aligned16(wq) || !aligned16(Y) || !aligned16(ctx) || !aligned16(ws) ||
      (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)))
    return MOE_ERR_INVALID_ARG;
  if (ctx_bytes < L.ctx_bytes || ws_bytes < L.ws_bytes || wq_bytes < L.wq_bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ctx c = make_ctx(L, ctx, ws);
  MOE_TRY(cudaMemsetAsync(c.hdr, 0, HDR_WORDS * 4, st));
  if (L.T == 0) return MOE_OK;
  MOE_TRY(cudaMemsetAsync(c.nvsc, 0, 4 * sizeof(unsigned), st));  // amax X, amax H, gs X, gs H
  {
    const moe_status r = route_tokens(L, c, X, W_r, bias, 0, st);
    if (r != MOE_OK) return r;
  }
  unsigned* amx = c.nvsc;                               // [amax X, amax H]
  float* gsv = reinterpret_cast<float*>(c.nvsc + 2);    // [gs X, gs H]
  const auto* w = static_cast<const uint8_t*>(wq);
  const float* gsw = reinterpret_cast<const float*>(w + L.wnvgs);  // [gate, up, down]
  const auto* Xb = static_cast<const __nv_bfloat16*>(X);
  MOE_TRY(timed(K_NV_SCALE, st, [&] {
    const cudaError_t e = launch_nv_amax(Xb, L.T * static_cast<int64_t>(L.d), amx, st);
    return e != cudaSuccess ? e : launch_nv_scale(amx, gsv, 1, st);
  }));
  // X's codes for the gate/up GEMM, and X_perm in bf16 for the weight gradients
  MOE_TRY(timed(K_DISPATCH, st, [&] { return launch_nv_gather_x(L, c, Xb, gsv, c.xq, c.xqs, c.xperm, st); }));
  const int grid = num_sms();
  int* status = c.hdr + HDR_STATUS;
  const uint64_t RP = static_cast<uint64_t>(L.RP), El = static_cast<uint64_t>(L.El);
  {
    MxParams p = mx_params(L, c, status);
    MOE_TMAP(tmap_fp8(&p.ta0, c.xq, L.d / 2, RP, 128));
    MOE_TMAP(tmap_fp8(&p.tb0, w + L.wgu1, L.d / 2, El * 2 * L.I, mx_bn(NV_GATEUP)));
    p.ta1 = p.ta0;
    p.tb1 = p.tb0;
    p.sfa0 = p.sfa1 = c.xqs;
    p.sfb0 = p.sfb1 = w + L.wgu1s;
    p.gsa = gsv;
    p.gsb = gsw;
    p.hout = c.nvh;
    p.amax = amx + 1;
    p.out0 = c.abuf;  // A, B (bf16) saved for the backward
    p.out1 = c.bbuf;
    MOE_TRY(timed(K_NV_GATEUP, st, [&] { return launch_gemm_mx(NV_GATEUP, p, grid, st); }));
  }
  MOE_TRY(timed(K_NV_QUANT_H, st, [&] {
    const cudaError_t e = launch_nv_scale(amx + 1, gsv + 1, 1, st);
    return e != cudaSuccess ? e : launch_nv_quant_h(L, c, c.nvh, gsv + 1, c.hq, c.hqs, nullptr, st);
  }));
  {
    MxParams p = mx_params(L, c, status);
    MOE_TMAP(tmap_fp8(&p.ta0, c.hq, L.I / 2, RP, 128));
    MOE_TMAP(tmap_fp8(&p.tb0, w + L.wd2, L.I / 2, El * L.d, mx_bn(NV_DOWN)));
    p.ta1 = p.ta0;
    p.tb1 = p.tb0;
    p.sfa0 = p.sfa1 = c.hqs;
    p.sfb0 = p.sfb1 = w + L.wd2s;
    p.gsa = gsv + 1;
    p.gsb = gsw + 2;
    p.out0 = c.obuf;
    MOE_TRY(timed(K_NV_DOWN, st, [&] { return launch_gemm_mx(NV_DOWN, p, grid, st); }));
  }
  MOE_TRY(timed(K_COMBINE, st, [&] { return launch_combine(L, c, c.obuf, static_cast<__nv_bfloat16*>(Y), st); }));
  return MOE_OK;
}

// NVFP4 backward: the reverse-combine quantises dY along d (its global scale from an amax pass)
// and keeps its bf16 rows; the dgrad of W_down (SwiGLU backward and router-gate gradient in its
// epilogue) writes bf16 dA, dB, Hg and fp32 dA, dB with their joint amax; the router backward;
// [dA | dB] quantised along I under one scale; the dgrad of gate/up over K = 2I; the reverse
// dispatch; the weight gradients from the bf16 operands.
moe_status moe_bwd_nvfp4(const moe_shape* s, const void* X, const void* W_r, const void* wq, size_t wq_bytes,
                         const void* dY, void* ctx, size_t ctx_bytes, void* dX, void* dW_gate, void* dW_up,
                         void* dW_down, float* dW_r, void* ws, size_t ws_bytes, void* stream) {
  Layout L;
  const moe_status cs = check_shape_nv(s, &L);
  if (cs != MOE_OK) return cs;
  const bool tok = s->T > 0;
  if ((tok && (!X || !dY || !dX)) || !W_r || !wq || !ctx || !dW_gate || !dW_up || !dW_down || !dW_r || !ws)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(W_r) || !aligned16(wq) || !aligned16(dY) || !aligned16(ctx) || !aligned16(dX) ||
      !aligned16(dW_gate) || !aligned16(dW_up) || !aligned16(dW_down) || !aligned16(dW_r) || !aligned16(ws))
    return MOE_ERR_INVALID_ARG;
  if (ctx_bytes < L.ctx_bytes || ws_bytes < L.ws_bytes || wq_bytes < L.wq_bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ctx c = make_ctx(L, ctx, ws);
  if (L.T == 0) return zero_wgrads(L, dW_gate, dW_up, dW_down, dW_r, st);
  const int grid = num_sms();
  int* status = c.hdr + HDR_STATUS;
  const uint64_t RP = static_cast<uint64_t>(L.RP), El = static_cast<uint64_t>(L.El);
  const auto* w = static_cast<const uint8_t*>(wq);
  const float* gsw = reinterpret_cast<const float*>(w + L.wnvgs);  // [gate, up, down, gate | up]
  unsigned* amx = c.nvsc + 4;                                      // [amax dY, amax dA | dB]
  float* gsv = reinterpret_cast<float*>(c.nvsc + 6);               // [gs dY, gs dA | dB]
  const auto* dYb = static_cast<const __nv_bfloat16*>(dY);
  MOE_TRY(cudaMemsetAsync(amx, 0, 2 * sizeof(unsigned), st));
  MOE_TRY(timed(K_NV_SCALE, st, [&] {
    const cudaError_t e = launch_nv_amax(dYb, L.T * static_cast<int64_t>(L.d), amx, st);
    return e != cudaSuccess ? e : launch_nv_scale(amx, gsv, 1, st);
  }));
  MOE_TRY(timed(K_REV_COMBINE, st, [&] { return launch_nv_gather_x(L, c, dYb, gsv, c.dyq, c.dyqs, c.dyperm, st); }));
  {
    MxParams p = mx_params(L, c, status);
    MOE_TMAP(tmap_fp8(&p.ta0, c.dyq, L.d / 2, RP, 128));
    MOE_TMAP(tmap_fp8(&p.tb0, w + L.wd3, L.d / 2, El * L.I, mx_bn(NV_DGRAD_DOWN)));
    p.ta1 = p.ta0;
    p.tb1 = p.tb0;
    p.sfa0 = p.sfa1 = c.dyqs;
    p.sfb0 = p.sfb1 = w + L.wd3s;
    p.in0 = c.abuf;
    p.in1 = c.bbuf;
    p.out2 = c.hgbuf;  // dA, dB reach bf16 through their quantiser below
    p.hout = c.nvdab;
    p.hout2 = c.nvdab + RP * L.I;
    p.amax = amx + 1;
    p.gsa = gsv;
    p.gsb = gsw + 2;
    p.outf = c.dgpart;
    MOE_TRY(timed(K_NV_DGRAD_DOWN, st, [&] { return launch_gemm_mx(NV_DGRAD_DOWN, p, grid, st); }));
  }
  MOE_TRY_STATUS(router_backward(L, c, X, dW_r, status, st, L.I / mx_bn(NV_DGRAD_DOWN)));
  MOE_TRY(timed(K_TRANSPOSE_WR, st, [&] {
    return launch_transpose_wr(L, static_cast<const __nv_bfloat16*>(W_r), c.wrt, st);
  }));
  MOE_TRY(timed(K_NV_QUANT_DAB, st, [&] {
    cudaError_t e = launch_nv_scale(amx + 1, gsv + 1, 1, st);
    if (e == cudaSuccess) e = launch_nv_quant_h(L, c, c.nvdab, gsv + 1, c.daq, c.daqs, c.dabuf, st);
    if (e == cudaSuccess) e = launch_nv_quant_h(L, c, c.nvdab + RP * L.I, gsv + 1, c.dbq, c.dbqs, c.dbbuf, st);
    return e;
  }));
  {
    MxParams p = mx_params(L, c, status);
    MOE_TMAP(tmap_fp8(&p.ta0, c.daq, L.I / 2, RP, 128));
    MOE_TMAP(tmap_fp8(&p.ta1, c.dbq, L.I / 2, RP, 128));
    MOE_TMAP(tmap_fp8(&p.tb0, w + L.wg4, L.I / 2, El * L.d, mx_bn(NV_DGRAD_GATEUP)));
    MOE_TMAP(tmap_fp8(&p.tb1, w + L.wu4, L.I / 2, El * L.d, mx_bn(NV_DGRAD_GATEUP)));
    p.sfa0 = c.daqs;
    p.sfa1 = c.dbqs;
    p.sfb0 = w + L.wg4s;
    p.sfb1 = w + L.wu4s;
    p.gsa = gsv + 1;
    p.gsb = gsw + 3;
    p.out0 = c.dxperm;
    MOE_TRY(timed(K_NV_DGRAD_GATEUP, st, [&] { return launch_gemm_mx(NV_DGRAD_GATEUP, p, grid, st); }));
  }
  MOE_TRY(timed(K_REV_DISPATCH, st, [&] { return launch_rev_dispatch(L, c, static_cast<__nv_bfloat16*>(dX), st); }));
  return launch_wgrads(L, c, status, dW_gate, dW_up, dW_down, st);
}

// Byte offsets of the NVFP4 buffers, for tests: out[0..1] X codes and scales (ctx), out[2..4] H
// codes, scales, fp32 H (workspace), out[5] the workspace's scale words, out[6..9] gate/up codes
// and scales, W_down^T codes and scales, out[10] the weights' global scales (prepared weights),
// out[11..14] dY codes and scales, dA codes and scales (workspace), out[15..16] dB codes and
// scales (workspace), out[17..22] W_down (K = d), W_gate (K = I), W_up (K = I) codes and scales
// (prepared weights).
moe_status moe_debug_nv_offsets(const moe_shape* s, int64_t* out) {
  Layout L;
  const moe_status cs = check_shape_nv(s, &L);
  if (cs != MOE_OK) return cs;
  if (!out) return MOE_ERR_INVALID_ARG;
  const size_t v[23] = {L.xq,  L.xqs,  L.hq,  L.hqs,  L.nvh,  L.nvsc, L.wgu1, L.wgu1s, L.wd2, L.wd2s, L.wnvgs, L.dyq,
                        L.dyqs, L.daq, L.daqs, L.dbq, L.dbqs, L.wd3, L.wd3s, L.wg4, L.wg4s, L.wu4, L.wu4s};
  for (int i = 0; i < 23; ++i) out[i] = static_cast<int64_t>(v[i]);
  return MOE_OK;
}

moe_status moe_bwd_mx(const moe_shape* s, const void* X, const void* W_r, const void* wq, size_t wq_bytes,
                      const void* dY, void* ctx, size_t ctx_bytes, void* dX, void* dW_gate, void* dW_up,
                      void* dW_down, float* dW_r, void* ws, size_t ws_bytes, void* stream) {
  Layout L;
  const moe_status cs = check_shape_mx(s, &L);
  if (cs != MOE_OK) return cs;
  const bool tok = s->T > 0;
  if ((tok && (!X || !dY || !dX)) || !W_r || !wq || !ctx || !dW_gate || !dW_up || !dW_down || !dW_r || !ws)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(W_r) || !aligned16(wq) || !aligned16(dY) || !aligned16(ctx) || !aligned16(dX) ||
      !aligned16(dW_gate) || !aligned16(dW_up) || !aligned16(dW_down) || !aligned16(dW_r) || !aligned16(ws))
    return MOE_ERR_INVALID_ARG;
  if (ctx_bytes < L.ctx_bytes || ws_bytes < L.ws_bytes || wq_bytes < L.wq_bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ctx c = make_ctx(L, ctx, ws);
  if (L.T == 0) return zero_wgrads(L, dW_gate, dW_up, dW_down, dW_r, st);
  const int grid = num_sms();
  int* status = c.hdr + HDR_STATUS;
  const uint64_t RP = static_cast<uint64_t>(L.RP), El = static_cast<uint64_t>(L.El);
  const auto* w = static_cast<const uint8_t*>(wq);
  MOE_TRY(timed(K_REV_COMBINE, st, [&] {
    if (L.mxw)  // along d for the dgrad of W_down and along the rows for the weight gradients
      return launch_gather_quant2(L, c, static_cast<const __nv_bfloat16*>(dY), c.dyq, c.dyqs, c.dyqt, c.dyqts, st);
    return launch_gather_rows_mx(L, c, static_cast<const __nv_bfloat16*>(dY), c.dyperm, c.dyq, c.dyqs, st);
  }));
  {
    MxParams p = mx_params(L, c, status);
    MOE_TMAP(tmap_fp8(&p.ta0, c.dyq, L.d, RP, 128));
    MOE_TMAP(tmap_fp8(&p.tb0, w + L.wd3, L.d, El * L.I, mx_bn(MX_DGRAD_DOWN)));
    p.ta1 = p.ta0;
    p.tb1 = p.tb0;
    p.sfa0 = p.sfa1 = c.dyqs;
    p.sfb0 = p.sfb1 = w + L.wd3s;
    p.in0 = c.abuf;
    p.in1 = c.bbuf;
    if (L.mxw) {  // dA, dB, Hg quantised along the rows here, from fp32, for the MXFP8 weight gradients
      p.tq[0] = c.daqt;
      p.tq[1] = c.dbqt;
      p.tq[2] = c.hgqt;
      p.tqs[0] = c.daqts;
      p.tqs[1] = c.dbqts;
      p.tqs[2] = c.hgqts;
      } else {  // bf16 operands of the bf16 weight gradients
      p.out0 = c.dabuf;
      p.out1 = c.dbbuf;
      p.out2 = c.hgbuf;
    }
    p.q0 = c.daq;
    p.qs0 = c.daqs;
    p.q1 = c.dbq;
    p.qs1 = c.dbqs;
    p.outf = c.dgpart;
    MOE_TRY(timed(K_GEMM_DGRAD_DOWN, st, [&] { return launch_gemm_mx(MX_DGRAD_DOWN, p, grid, st); }));
  }
  MOE_TRY_STATUS(router_backward(L, c, X, dW_r, status, st, L.I / mx_bn(MX_DGRAD_DOWN)));
  MOE_TRY(timed(K_TRANSPOSE_WR, st, [&] {
    return launch_transpose_wr(L, static_cast<const __nv_bfloat16*>(W_r), c.wrt, st);
  }));
  {
    MxParams p = mx_params(L, c, status);
    MOE_TMAP(tmap_fp8(&p.ta0, c.daq, L.I, RP, 128));
    MOE_TMAP(tmap_fp8(&p.ta1, c.dbq, L.I, RP, 128));
    MOE_TMAP(tmap_fp8(&p.tb0, w + L.wg4, L.I, El * L.d, mx_bn(MX_DGRAD_GATEUP)));
    MOE_TMAP(tmap_fp8(&p.tb1, w + L.wu4, L.I, El * L.d, mx_bn(MX_DGRAD_GATEUP)));
    p.sfa0 = c.daqs;
    p.sfa1 = c.dbqs;
    p.sfb0 = w + L.wg4s;
    p.sfb1 = w + L.wu4s;
    p.out0 = c.dxperm;
    MOE_TRY(timed(K_GEMM_DGRAD_GATEUP, st, [&] { return launch_gemm_mx(MX_DGRAD_GATEUP, p, grid, st); }));
  }
  MOE_TRY(timed(K_REV_DISPATCH, st, [&] { return launch_rev_dispatch(L, c, static_cast<__nv_bfloat16*>(dX), st); }));
  // weight gradients contract over tokens: from the bf16 operands on the bf16 engine, or
  // (MOE_MXFP8_ALL) on MXFP8 from the operands quantised along the rows
  if (!L.mxw) return launch_wgrads(L, c, status, dW_gate, dW_up, dW_down, st);
  return launch_wgrads_mx(L, c, status, dW_gate, dW_up, dW_down, st);
}

moe_status moe_get_error(void* ctx, void* stream) {
  if (!ctx) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  int code = 0;
  if (cudaMemcpy(&code, static_cast<char*>(ctx) + HDR_STATUS * 4, 4, cudaMemcpyDeviceToHost) != cudaSuccess)
    return MOE_ERR_CUDA;
  const int zero = 0;
  if (code != 0 && cudaMemcpy(static_cast<char*>(ctx) + HDR_STATUS * 4, &zero, 4, cudaMemcpyHostToDevice) != cudaSuccess)
    return MOE_ERR_CUDA;
  return static_cast<moe_status>(code);
}

moe_status moe_debug_routing(const moe_shape* s, const void* ctx, int32_t* ids, float* gates, int32_t* counts,
                             int32_t* offsets, int32_t* padded_offsets, int32_t* perm, int32_t* slot_row,
                             void* stream) {
  Layout L;
  const moe_status cs = check_shape(s, &L);
  if (cs != MOE_OK) return cs;
  if (!ctx) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ctx c = make_ctx(L, const_cast<void*>(ctx), nullptr);
  const size_t tk = static_cast<size_t>(L.T) * L.k * 4;
  if (L.T == 0) return MOE_OK;
  if (ids) MOE_TRY(cudaMemcpyAsync(ids, c.ids, tk, cudaMemcpyDeviceToDevice, st));
  if (gates) MOE_TRY(cudaMemcpyAsync(gates, c.gates, tk, cudaMemcpyDeviceToDevice, st));
  if (slot_row) MOE_TRY(cudaMemcpyAsync(slot_row, c.slot_row, tk, cudaMemcpyDeviceToDevice, st));
  if (counts || offsets || padded_offsets || perm)
    MOE_TRY(launch_export_routing(L, c, counts, offsets, padded_offsets, perm, st));
  return MOE_OK;
}

moe_status moe_debug_router_grad(const moe_shape* s, const void* ws, float* dl, void* stream) {
  Layout L;
  const moe_status cs = check_shape(s, &L);
  if (cs != MOE_OK) return cs;
  if (!ws || !dl) return MOE_ERR_INVALID_ARG;
  if (L.T == 0) return MOE_OK;
  MOE_TRY(cudaMemcpyAsync(dl, static_cast<const char*>(ws) + L.dlasg, static_cast<size_t>(L.T) * L.k * 4,
                          cudaMemcpyDeviceToDevice, static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_debug_bounded_wait(const moe_shape* s, void* ctx, size_t ctx_bytes, void* stream) {
  Layout L;
  const moe_status cs = check_shape(s, &L);
  if (cs != MOE_OK) return cs;
  if (!ctx || !aligned16(ctx)) return MOE_ERR_INVALID_ARG;
  if (ctx_bytes < L.ctx_bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  const Ctx c = make_ctx(L, ctx, nullptr);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MOE_TRY(cudaMemsetAsync(c.hdr + HDR_STATUS, 0, 4, st));  // a clear status word: the wait must run out
  MOE_TRY(launch_wait_probe(c.hdr + HDR_STATUS, st));
  return MOE_OK;
}

moe_status moe_debug_logits(const moe_shape* s, const void* ws, float* logits, void* stream) {
  Layout L;
  const moe_status cs = check_shape(s, &L);
  if (cs != MOE_OK) return cs;
  if (!ws || !logits) return MOE_ERR_INVALID_ARG;
  if (L.T == 0) return MOE_OK;
  MOE_TRY(cudaMemcpyAsync(logits, static_cast<const char*>(ws) + L.logits, static_cast<size_t>(L.T) * L.E * 4,
                          cudaMemcpyDeviceToDevice, static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Expert parallelism across R ranks (exchange kernels in ep.cu)
// ---------------------------------------------------------------------------
namespace {
struct EpSetup {
  Layout Ls;       // the source role: this rank's T tokens, routed over all E experts
  Layout Lo;       // the owner role: rows from all R ranks for the local experts
  EpBuf B;         // exchange buffer regions
  size_t ctx_o;    // owner ctx at ctx + ctx_o, then the per-source row counts table
  size_t base_off;
  size_t ws_o;     // owner workspace at ws + ws_o
  size_t ctx_bytes, ws_bytes;
  int El, first, R, rank;
  int64_t TK;
};

moe_status ep_setup(const moe_shape* s, int32_t R, int32_t rank, EpSetup* S) {
  if (!s) return MOE_ERR_INVALID_ARG;
  if (s->prec != MOE_BF16) return is_mx_prec(s->prec) ? MOE_ERR_UNSUPPORTED : MOE_ERR_INVALID_ARG;
  if (R < 1 || R > kEpMaxRanks || rank < 0 || rank >= R || s->E <= 0 || s->E % R) return MOE_ERR_INVALID_ARG;
  if (s->T < 0 || s->T * static_cast<int64_t>(R) * s->top_k >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  const int El = s->E / R;
  moe_shape src = *s, own = *s;
  // source role: a one-expert "slice" keeps its padded-row buffers small; its router weight
  // gradient contracts over all of its tokens (every assignment has an owner somewhere)
  src.first_local_expert = 0;
  src.num_local_experts = 1;
  own.T = s->T * R;
  own.first_local_expert = rank * El;
  own.num_local_experts = El;
  if (!make_layout(src, &S->Ls) || !make_layout(own, &S->Lo)) return MOE_ERR_UNSUPPORTED;
  S->Ls.rslice = false;
  S->B = ep_buffer_layout(s->T, s->top_k, s->E, s->d, R);
  S->ctx_o = align_up(S->Ls.ctx_bytes, 256);
  S->base_off = align_up(S->ctx_o + S->Lo.ctx_bytes, 256);
  S->ctx_bytes = S->base_off + static_cast<size_t>(El) * (R + 1) * 4;
  S->ws_o = align_up(S->Ls.ws_bytes, 256);
  S->ws_bytes = S->ws_o + S->Lo.ws_bytes;
  S->El = El;
  S->first = rank * El;
  S->R = R;
  S->rank = rank;
  S->TK = s->T * static_cast<int64_t>(s->top_k);
  return MOE_OK;
}

moe_status ep_peers(const EpSetup& S, void* const* bufs, EpPeers* P) {
  if (!bufs) return MOE_ERR_INVALID_ARG;
  std::memset(P, 0, sizeof(*P));
  for (int r = 0; r < S.R; ++r) {
    if (!bufs[r] || (reinterpret_cast<uintptr_t>(bufs[r]) & 255u)) return MOE_ERR_INVALID_ARG;
    P->base[r] = static_cast<uint8_t*>(bufs[r]);
  }
  return MOE_OK;
}

// The source role's view: routing table regions in this rank's exchange buffer, slot_row the
// identity (receive regions are indexed by assignment), the router gradient's dg from recv_dg.
Ctx ep_source_ctx(const EpSetup& S, void* ctx, void* ws, uint8_t* mine) {
  Ctx c = make_ctx(S.Ls, ctx, ws);
  c.counts = reinterpret_cast<int*>(mine + S.B.counts);
  c.offsets = reinterpret_cast<int*>(mine + S.B.offsets);
  c.perm_asg = reinterpret_cast<int*>(mine + S.B.perm_asg);
  c.gates = reinterpret_cast<float*>(mine + S.B.gates);
  c.dgpart = reinterpret_cast<float*>(mine + S.B.recv_dg);
  c.dxperm = reinterpret_cast<__nv_bfloat16*>(mine + S.B.recv_dx);
  return c;
}

moe_status ep_check(const moe_shape* s, int32_t R, int32_t rank, void* const* bufs, void* ctx, size_t ctx_bytes,
                    void* ws, size_t ws_bytes, bool need_ws, EpSetup* S, EpPeers* P) {
  const moe_status e = ep_setup(s, R, rank, S);
  if (e != MOE_OK) return e;
  if (!ctx || !aligned16(ctx) || (need_ws && (!ws || !aligned16(ws)))) return MOE_ERR_INVALID_ARG;
  if (ctx_bytes < S->ctx_bytes || (need_ws && ws_bytes < S->ws_bytes)) return MOE_ERR_WORKSPACE_TOO_SMALL;
  return ep_peers(*S, bufs, P);
}
}  // namespace

extern "C" {

size_t moe_ep_buffer_size(const moe_shape* s, int32_t R) {
  EpSetup S;
  return ep_setup(s, R, 0, &S) == MOE_OK ? S.B.bytes : 0;
}
size_t moe_ep_ctx_size(const moe_shape* s, int32_t R) {
  EpSetup S;
  return ep_setup(s, R, 0, &S) == MOE_OK ? S.ctx_bytes : 0;
}
size_t moe_ep_workspace_size(const moe_shape* s, int32_t R) {
  EpSetup S;
  return ep_setup(s, R, 0, &S) == MOE_OK ? S.ws_bytes : 0;
}

moe_status moe_ep_fwd_route(const moe_shape* s, int32_t R, int32_t rank, void* const* bufs, const void* X,
                            const void* W_r, const float* bias, void* ctx, size_t ctx_bytes, void* ws, size_t ws_bytes,
                            int32_t epoch, void* stream) {
  EpSetup S;
  EpPeers P;
  const moe_status e = ep_check(s, R, rank, bufs, ctx, ctx_bytes, ws, ws_bytes, true, &S, &P);
  if (e != MOE_OK) return e;
  if ((s->T > 0 && !X) || !W_r || !aligned16(X) || !aligned16(W_r) || (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)))
    return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* mine = P.base[rank];
  const Ctx c = ep_source_ctx(S, ctx, ws, mine);
  MOE_TRY(cudaMemsetAsync(c.hdr, 0, HDR_WORDS * 4, st));  // clears the status word
  {  // the owner role's row layout starts empty: if this step's plan does not run (a wait gave
     // up), its GEMMs and exchange kernels see no rows
    const Ctx co = make_ctx(S.Lo, static_cast<char*>(ctx) + S.ctx_o, nullptr);
    MOE_TRY(cudaMemsetAsync(co.poff, 0, static_cast<size_t>(S.El + 1) * 4, st));
    MOE_TRY(cudaMemsetAsync(co.counts, 0, static_cast<size_t>(s->E) * 4, st));
    MOE_TRY(cudaMemsetAsync(co.hdr, 0, HDR_WORDS * 4, st));
  }
  if (S.Ls.T == 0) {
    MOE_TRY(cudaMemsetAsync(mine + S.B.counts, 0, static_cast<size_t>(s->E) * 4, st));
    MOE_TRY(cudaMemsetAsync(mine + S.B.offsets, 0, static_cast<size_t>(s->E + 1) * 4, st));
  } else {
    MOE_TRY_STATUS(route_tokens(S.Ls, c, X, W_r, bias, 0, st));  // table straight into the exchange buffer
    MOE_TRY(cudaMemcpyAsync(mine + S.B.x, X, static_cast<size_t>(S.Ls.T) * s->d * 2, cudaMemcpyDeviceToDevice, st));
    MOE_TRY(launch_ep_identity(c.slot_row, S.TK, st));
  }
  MOE_TRY(launch_ep_signal(P, R, rank, false, S.B.flags, EPF_FWD_READY, epoch, st));
  return MOE_OK;
}

moe_status moe_ep_fwd_experts(const moe_shape* s, int32_t R, int32_t rank, void* const* bufs, const void* W_gate,
                              const void* W_up, const void* W_down, void* ctx, size_t ctx_bytes, void* ws,
                              size_t ws_bytes, int32_t epoch, void* stream) {
  EpSetup S;
  EpPeers P;
  const moe_status e = ep_check(s, R, rank, bufs, ctx, ctx_bytes, ws, ws_bytes, true, &S, &P);
  if (e != MOE_OK) return e;
  if (!W_gate || !W_up || !W_down || !aligned16(W_gate) || !aligned16(W_up) || !aligned16(W_down))
    return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Layout& L = S.Lo;
  int* status = static_cast<int*>(ctx) + HDR_STATUS;  // the source role's status word leads ctx
  const Ctx c = make_ctx(L, static_cast<char*>(ctx) + S.ctx_o, static_cast<char*>(ws) + S.ws_o);
  int* base = reinterpret_cast<int*>(static_cast<char*>(ctx) + S.base_off);
  const int TK = static_cast<int>(S.TK);
  const uint64_t RP = static_cast<uint64_t>(L.RP);
  // every source has published its table and rows: pull them
  MOE_TRY(launch_ep_wait(P, R, rank, false, S.B.flags, EPF_FWD_READY, epoch, status, st));
  MOE_TRY(launch_ep_plan(P, R, S.B.counts, S.first, S.El, L.RP, c.counts, c.poff, base, c.hdr, status, st));
  MOE_TRY(timed(K_MARK_ROWS, st, [&] { return launch_mark_rows(L, c, st); }));
  MOE_TRY(launch_ep_table(P, R, S.B, S.first, S.El, TK, c.poff, base, c.row_asg, c.row_gate, status, st));
  MOE_TRY(timed(K_DISPATCH, st, [&] {
    return launch_ep_gather(P, S.B.x, TK, L.k, L.d, c.poff, L.El, c.row_asg, L.RP, c.xperm, status, st);
  }));
  // the owner's gate/up and down GEMMs as one persistent launch
  GemmParams gu = base_params(L, c, status);
  MOE_TMAP(tmap_2d(&gu.ta0, c.xperm, L.d, RP, L.d, 64, 128));
  MOE_TMAP(tmap_2d(&gu.tb0, W_gate, L.I, static_cast<uint64_t>(L.El) * L.d, L.I, 64, 64));
  MOE_TMAP(tmap_2d(&gu.tb1, W_up, L.I, static_cast<uint64_t>(L.El) * L.d, L.I, 64, 64));
  gu.ta1 = gu.ta0;
  gu.out0 = c.abuf;
  gu.out1 = c.bbuf;
  gu.out2 = c.hbuf;
  GemmParams dn = base_params(L, c, status);
  MOE_TMAP(tmap_2d(&dn.ta0, c.hbuf, L.I, RP, L.I, 64, 128));
  MOE_TMAP(tmap_2d(&dn.tb0, W_down, L.d, static_cast<uint64_t>(L.El) * L.I, L.d, 64, 64));
  dn.ta1 = dn.ta0;
  dn.tb1 = dn.tb0;
  dn.out0 = c.obuf;
  MOE_TRY(timed(K_PAIR_FWD, st, [&] { return run_gemm_pair(L, c, PAIR_FWD, gu, dn, st); }));
  // push each output row back to its source's slot, then tell every source
  MOE_TRY(timed(K_COMBINE, st, [&] {
    return launch_ep_push_rows(P, S.B.recv_o, TK, L.d, c.poff, L.El, c.row_asg, L.RP, c.obuf, status, st);
  }));
  MOE_TRY(launch_ep_signal(P, R, rank, true, S.B.flags, EPF_DONE + rank, epoch, st));
  return MOE_OK;
}

moe_status moe_ep_fwd_combine(const moe_shape* s, int32_t R, int32_t rank, void* const* bufs, void* Y, void* ctx,
                              size_t ctx_bytes, int32_t epoch, void* stream) {
  EpSetup S;
  EpPeers P;
  const moe_status e = ep_check(s, R, rank, bufs, ctx, ctx_bytes, nullptr, 0, false, &S, &P);
  if (e != MOE_OK) return e;
  if ((s->T > 0 && !Y) || !aligned16(Y)) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* mine = P.base[rank];
  const Ctx c = ep_source_ctx(S, ctx, nullptr, mine);
  MOE_TRY(launch_ep_wait(P, R, rank, true, S.B.flags, EPF_DONE, epoch, c.hdr + HDR_STATUS, st));
  if (S.Ls.T == 0) return MOE_OK;
  MOE_TRY(timed(K_COMBINE, st, [&] {
    return launch_combine(S.Ls, c, reinterpret_cast<const __nv_bfloat16*>(mine + S.B.recv_o),
                          static_cast<__nv_bfloat16*>(Y), st);
  }));
  return MOE_OK;
}

moe_status moe_ep_bwd_publish(const moe_shape* s, int32_t R, int32_t rank, void* const* bufs, const void* dY,
                              void* ctx, size_t ctx_bytes, int32_t epoch, void* stream) {
  EpSetup S;
  EpPeers P;
  const moe_status e = ep_check(s, R, rank, bufs, ctx, ctx_bytes, nullptr, 0, false, &S, &P);
  if (e != MOE_OK) return e;
  if ((s->T > 0 && !dY) || !aligned16(dY)) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (S.Ls.T > 0)
    MOE_TRY(cudaMemcpyAsync(P.base[rank] + S.B.dy, dY, static_cast<size_t>(S.Ls.T) * s->d * 2,
                            cudaMemcpyDeviceToDevice, st));
  MOE_TRY(launch_ep_signal(P, R, rank, false, S.B.flags, EPF_BWD_READY, epoch, st));
  return MOE_OK;
}

moe_status moe_ep_bwd_experts(const moe_shape* s, int32_t R, int32_t rank, void* const* bufs, const void* W_gate,
                              const void* W_up, const void* W_down, void* dW_gate, void* dW_up, void* dW_down,
                              void* ctx, size_t ctx_bytes, void* ws, size_t ws_bytes, int32_t epoch, void* stream) {
  EpSetup S;
  EpPeers P;
  const moe_status e = ep_check(s, R, rank, bufs, ctx, ctx_bytes, ws, ws_bytes, true, &S, &P);
  if (e != MOE_OK) return e;
  if (!W_gate || !W_up || !W_down || !dW_gate || !dW_up || !dW_down || !aligned16(W_gate) || !aligned16(W_up) ||
      !aligned16(W_down) || !aligned16(dW_gate) || !aligned16(dW_up) || !aligned16(dW_down))
    return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Layout& L = S.Lo;
  int* status = static_cast<int*>(ctx) + HDR_STATUS;
  const Ctx c = make_ctx(L, static_cast<char*>(ctx) + S.ctx_o, static_cast<char*>(ws) + S.ws_o);
  const int TK = static_cast<int>(S.TK);
  const uint64_t RP = static_cast<uint64_t>(L.RP), El = static_cast<uint64_t>(L.El);
  MOE_TRY(launch_ep_wait(P, R, rank, false, S.B.flags, EPF_BWD_READY, epoch, status, st));
  // pull reverse-combine: dY rows from every source
  MOE_TRY(timed(K_REV_COMBINE, st, [&] {
    return launch_ep_gather(P, S.B.dy, TK, L.k, L.d, c.poff, L.El, c.row_asg, L.RP, c.dyperm, status, st);
  }));
  // the owner's dgrad of W_down (SwiGLU backward, router-gate partials) and dgrad of gate/up as
  // one persistent launch
  GemmParams p9 = base_params(L, c, status);
  MOE_TMAP(tmap_2d(&p9.ta0, c.dyperm, L.d, RP, L.d, 64, 128));
  MOE_TMAP(tmap_2d(&p9.tb0, W_down, L.d, El * L.I, L.d, 64, 256));
  p9.ta1 = p9.ta0;
  p9.tb1 = p9.tb0;
  p9.in0 = c.abuf;
  p9.in1 = c.bbuf;
  p9.out0 = c.dabuf;
  p9.out1 = c.dbbuf;
  p9.out2 = c.hgbuf;
  p9.outf = c.dgpart;
  GemmParams p11 = base_params(L, c, status);
  MOE_TMAP(tmap_2d(&p11.ta0, c.dabuf, L.I, RP, L.I, 64, 128));
  MOE_TMAP(tmap_2d(&p11.ta1, c.dbbuf, L.I, RP, L.I, 64, 128));
  MOE_TMAP(tmap_2d(&p11.tb0, W_gate, L.I, El * L.d, L.I, 64, 256));
  MOE_TMAP(tmap_2d(&p11.tb1, W_up, L.I, El * L.d, L.I, 64, 256));
  p11.out0 = c.dxperm;
  MOE_TRY(timed(K_PAIR_DGRAD, st, [&] { return run_gemm_pair(L, c, PAIR_DGRAD, p9, p11, st); }));
  // push each row's router-gate gradient back to its source
  MOE_TRY(timed(K_ROUTER_BWD, st, [&] {
    return launch_ep_push_dg(P, S.B.recv_dg, TK, c.poff, L.El, c.row_asg, c.dgpart, L.I / 256, L.RP, status, st);
  }));
  // push reverse-dispatch: dX rows to their sources, then tell every source
  MOE_TRY(timed(K_REV_DISPATCH, st, [&] {
    return launch_ep_push_rows(P, S.B.recv_dx, TK, L.d, c.poff, L.El, c.row_asg, L.RP, c.dxperm, status, st);
  }));
  MOE_TRY(launch_ep_signal(P, R, rank, true, S.B.flags, EPF_DONE + R + rank, epoch, st));
  return launch_wgrads(L, c, status, dW_gate, dW_up, dW_down, st);
}

moe_status moe_ep_bwd_finish(const moe_shape* s, int32_t R, int32_t rank, void* const* bufs, const void* X,
                             const void* W_r, void* dX, float* dW_r, void* ctx, size_t ctx_bytes, void* ws,
                             size_t ws_bytes, int32_t epoch, void* stream) {
  EpSetup S;
  EpPeers P;
  const moe_status e = ep_check(s, R, rank, bufs, ctx, ctx_bytes, ws, ws_bytes, true, &S, &P);
  if (e != MOE_OK) return e;
  if ((s->T > 0 && (!X || !dX)) || !W_r || !dW_r || !aligned16(X) || !aligned16(dX) || !aligned16(W_r) ||
      !aligned16(dW_r))
    return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Layout& L = S.Ls;
  const Ctx c = ep_source_ctx(S, ctx, ws, P.base[rank]);
  int* status = c.hdr + HDR_STATUS;
  MOE_TRY(launch_ep_wait(P, R, rank, true, S.B.flags, EPF_DONE + R, epoch, status, st));
  if (L.T == 0) {
    MOE_TRY(cudaMemsetAsync(dW_r, 0, static_cast<size_t>(L.d) * L.E * 4, st));
    return MOE_OK;
  }
  // router backward over this rank's tokens (dg pushed back by the owners, one value per
  // assignment), its part of dW_r, and dX = the pushed dX rows in slot order + the router term
  MOE_TRY(timed(K_ROUTER_BWD, st, [&] { return launch_router_bwd(L, c, st, 1); }));
  MOE_TRY(timed(K_ROUTER_WGRAD, st, [&] { return launch_router_wgrad(L, c, X, dW_r, status, st); }));
  MOE_TRY(timed(K_TRANSPOSE_WR, st, [&] {
    return launch_transpose_wr(L, static_cast<const __nv_bfloat16*>(W_r), c.wrt, st);
  }));
  MOE_TRY(timed(K_REV_DISPATCH, st, [&] { return launch_rev_dispatch(L, c, static_cast<__nv_bfloat16*>(dX), st); }));
  return MOE_OK;
}

moe_status moe_ep_debug_plan(const moe_shape* s, int32_t R, int32_t rank, const void* ctx, int32_t* counts,
                             int32_t* padded_offsets, int32_t* row_src, void* stream) {
  EpSetup S;
  const moe_status e = ep_setup(s, R, rank, &S);
  if (e != MOE_OK) return e;
  if (!ctx) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ctx c = make_ctx(S.Lo, const_cast<char*>(static_cast<const char*>(ctx)) + S.ctx_o, nullptr);
  if (counts) MOE_TRY(cudaMemcpyAsync(counts, c.counts + S.first, S.El * 4, cudaMemcpyDeviceToDevice, st));
  if (padded_offsets)
    MOE_TRY(cudaMemcpyAsync(padded_offsets, c.poff, (S.El + 1) * 4, cudaMemcpyDeviceToDevice, st));
  if (row_src)
    MOE_TRY(cudaMemcpyAsync(row_src, c.row_asg, static_cast<size_t>(S.Lo.RP) * 4, cudaMemcpyDeviceToDevice, st));
  return MOE_OK;
}

}  // extern "C"
