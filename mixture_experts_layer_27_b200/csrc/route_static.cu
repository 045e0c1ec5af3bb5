// Router GEMM + top-k gating with no allocation: the scratch the step needs
// (W_r transposed, the router GEMM's split-K partial sums, the logits and the
// per-block expert histograms) lives in one file-scope device array instead of
// a caller-provided workspace.
//
// Who needs this: callers that must not allocate device memory once they are
// running -- for example code that runs inside a memory planner or allocator
// callback (where calling cudaMalloc would re-enter the allocator), or a
// long-running service whose device memory has all been handed out by its
// own pool at start-up.  They pass inputs and outputs only.
//
// The array is MOE_STATIC_SCRATCH_BYTES long and every GPU that loads this
// library holds it until the process exits.  All calls share it: calls that
// overlap on the GPU (different streams, or different host threads on one
// device) race on it, so serialise them.  It keeps the last call's contents;
// every region a call reads is written earlier in that same call, so nothing
// needs clearing between calls.
//
// Set-up: the library's kernels and this array are loaded lazily by CUDA (on
// first use, unless CUDA_MODULE_LOADING=EAGER), and loading commits device
// memory.  So the first call on each device does the set-up, with that device
// current: it looks up the array's device address and loads every kernel the
// call launches.  That first call therefore allocates; later calls do not.
// Make it before entering the region that must not allocate, and before any
// stream capture.  The device address is kept for the life of the process: it
// does not survive cudaDeviceReset (or anything else that destroys the
// device's primary context), after which this entry point must not be called
// again in that process.
#include <cstdint>
#include <mutex>

#include "moe_internal.cuh"

#define MOE_STATIC_SCRATCH_BYTES (32u << 20)

namespace moe {

static __device__ __align__(256) unsigned char g_route_scratch[MOE_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void* g_scratch_dev[kMaxDevices] = {};  // device address of g_route_scratch, per device

// In host code `g_route_scratch` names a host-side stand-in, not device memory:
// the device address comes from cudaGetSymbolAddress, once per device, with
// that device current.  The same set-up loads the kernels the call launches.
cudaError_t setup_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_setup_mu);
  if (!g_scratch_dev[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess) return e;
    e = preload_router_kernels();
    if (e != cudaSuccess) return e;
    e = preload_gemm(G_ROUTER);
    if (e != cudaSuccess) return e;
    g_scratch_dev[dev] = p;
  }
  *out = g_scratch_dev[dev];
  return cudaSuccess;
}

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_route_static(const moe_shape* shape, const void* X, const void* W_r, const float* bias,
                                       int32_t* ids, float* gates, int32_t* status, void* stream) {
  if (!shape || shape->prec != MOE_BF16) return shape ? MOE_ERR_UNSUPPORTED : MOE_ERR_INVALID_ARG;
  Layout L;
  if (!make_layout(*shape, &L)) return MOE_ERR_UNSUPPORTED;
  const bool tok = L.T > 0;
  if (!W_r || (tok && (!X || !ids || !gates))) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(X) | reinterpret_cast<uintptr_t>(W_r)) & 15u) return MOE_ERR_INVALID_ARG;

  // scratch regions, each 256-byte aligned: W_r^T | split partials | logits | histograms
  const int splits = router_splits(L.T, L.E, L.d);
  const size_t T = static_cast<size_t>(L.T), E = static_cast<size_t>(L.E);
  const size_t o_wrt = 0;
  const size_t o_part = o_wrt + up256(E * L.d * 2);
  const size_t o_logits = o_part + up256(static_cast<size_t>(splits) * T * E * 4);
  const size_t o_hist = o_logits + up256(T * E * 4);
  const size_t need = o_hist + up256(static_cast<size_t>(L.nblk) * E * 4);
  if (need > MOE_STATIC_SCRATCH_BYTES) return MOE_ERR_WORKSPACE_TOO_SMALL;

  void* base = nullptr;
  if (setup_device(&base) != cudaSuccess) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (status && cudaMemsetAsync(status, 0, sizeof(int32_t), st) != cudaSuccess) return MOE_ERR_CUDA;
  if (!tok) return MOE_OK;
  char* s = static_cast<char*>(base);
  auto* wrt = reinterpret_cast<__nv_bfloat16*>(s + o_wrt);

  Ctx c = {};
  c.hdr = status;  // HDR_STATUS is word 0: device errors land in the caller's status word
  c.ids = ids;
  c.gates = gates;
  c.rpart = reinterpret_cast<float*>(s + o_part);
  c.logits = reinterpret_cast<float*>(s + o_logits);
  c.hist = reinterpret_cast<int*>(s + o_hist);

  if (launch_transpose_wr(L, static_cast<const __nv_bfloat16*>(W_r), wrt, st) != cudaSuccess) return MOE_ERR_CUDA;
  if (launch_router_logits(L, X, wrt, c.rpart, status, st) != cudaSuccess) return MOE_ERR_CUDA;
  if (launch_topk(L, c, bias, splits, st) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}
