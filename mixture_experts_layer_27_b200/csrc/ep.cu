// Expert parallelism across ranks: the exchange kernels.
//
// The MoK pages ("Cursor open-sources Mixture-of-Kittens (MoK)...", page 1, "Three design
// decisions that matter", bullet 1) dispatch tokens by pulling: the rank that owns an expert
// reads the tokens it needs straight from the senders' memory, so no sender has to signal that
// its rows have arrived; the combine pushes each expert output back to the token's rank; one
// schedule table serves the forward and the mirrored backward.  Here every rank keeps an
// exchange buffer (ep_internal.cuh) in memory its peers can address (peer pointers over
// NVLink, or, with all ranks on one device, plain device memory); these kernels read the
// sources' routing tables and token rows from it, and write outputs into it, with ordinary
// vector loads and stores.  The only signals are one ready flag per rank (its table and rows
// are published) and one done flag per (owner, source) pair (the owner's pushes into that
// source are complete); every wait on them is bounded.
//
// Row order on an owner: per local expert, the sources in rank order, each source's tokens in
// ascending order -- the order the one-device layer gives the rank-major concatenation of the
// ranks' tokens, so the grouped GEMMs (and their fixed K order in the weight gradients) see
// the same rows in the same order.
#include "ep_internal.cuh"
#include "moe_internal.cuh"
#include "ptx.cuh"

namespace moe {

static size_t ep_align(size_t x) { return (x + 255) / 256 * 256; }

EpBuf ep_buffer_layout(int64_t T, int k, int E, int d, int R) {
  EpBuf b;
  const size_t TK = static_cast<size_t>(T) * k;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = ep_align(o + bytes);
    return at;
  };
  b.flags = take(static_cast<size_t>(2 + 2 * R) * 4);
  b.counts = take(static_cast<size_t>(E) * 4);
  b.offsets = take(static_cast<size_t>(E + 1) * 4);
  b.perm_asg = take(TK * 4);
  b.gates = take(TK * 4);
  b.x = take(static_cast<size_t>(T) * d * 2);
  b.dy = take(static_cast<size_t>(T) * d * 2);
  b.recv_o = take(TK * d * 2);
  b.recv_dx = take(TK * d * 2);
  b.recv_dg = take(TK * 4);
  b.bytes = o;
  return b;
}

__device__ __forceinline__ int* ep_flag(const EpPeers& P, int r, size_t flags_off, int idx) {
  return reinterpret_cast<int*>(P.base[r] + flags_off) + idx;
}

__global__ void k_ep_signal(const __grid_constant__ EpPeers P, int R, int self, int all, size_t flags_off, int idx,
                            int epoch) {
  const int r = threadIdx.x;
  if (r >= R || (!all && r != self)) return;
  __threadfence_system();  // this stream's earlier writes into the buffers before the flag
  atomicExch_system(ep_flag(P, r, flags_off, idx), epoch);
}

__global__ void k_ep_wait(const __grid_constant__ EpPeers P, int R, int self, int own, size_t flags_off, int idx,
                          int epoch, int* status) {
  const int i = threadIdx.x;
  if (i < R) {
    const volatile int* f = own ? ep_flag(P, self, flags_off, idx + i) : ep_flag(P, i, flags_off, idx);
    const long long t0 = clock64();
    while (*f != epoch) {
      if (status_set(status)) break;
      if (clock64() - t0 > MOE_SPIN_CYCLES) {
        raise_status(status, MOE_ERR_DEVICE_TIMEOUT);
        break;
      }
      __nanosleep(128);
    }
    __threadfence_system();  // the flag before the data it guards
  }
}

// exclusive scan of one value per thread over a block of 512 threads
__device__ __forceinline__ int ep_block_scan(int v, int* wsum, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nw) wsum[lane] = w;
  }
  __syncthreads();
  const int r = (warp > 0 ? wsum[warp - 1] : 0) + x - v;
  *total = wsum[nw - 1];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(512) k_ep_plan(const __grid_constant__ EpPeers P, int R, size_t counts_off,
                                                 int first, int El, int64_t max_rows, int* counts, int* poff,
                                                 int* base, int* hdr, int* status) {
  __shared__ int wsum[32];
  __shared__ int bad;
  if (threadIdx.x == 0) bad = status_set(status) ? 1 : 0;
  __syncthreads();
  if (bad) return;
  const int el = threadIdx.x;
  int run = 0;
  if (el < El) {
    for (int r = 0; r < R; ++r) {
      base[el * (R + 1) + r] = run;
      run += reinterpret_cast<const int*>(P.base[r] + counts_off)[first + el];
    }
    base[el * (R + 1) + R] = run;
  }
  const int padded = el < El ? (run + kPad - 1) / kPad * kPad : 0;
  int total = 0;
  const int p = ep_block_scan(padded, wsum, &total);
  const bool ok = run >= 0 && static_cast<int64_t>(total) <= max_rows;
  if (!__syncthreads_and(ok)) {  // counts no layout can hold: no rows at all, and an error
    if (el < El) {
      counts[first + el] = 0;
      poff[el] = 0;
    }
    if (el == 0) {
      raise_status(status, MOE_ERR_EXCHANGE);
      poff[El] = 0;
      hdr[HDR_ROWS_P] = hdr[HDR_MTILES] = 0;
    }
    return;
  }
  if (el < El) {
    counts[first + el] = run;
    poff[el] = p;
  }
  if (el == 0) {
    poff[El] = total;
    hdr[HDR_ROWS_P] = total;
    hdr[HDR_MTILES] = total / kPad;
  }
}

__global__ void __launch_bounds__(256) k_ep_table(const __grid_constant__ EpPeers P, int R, size_t offsets_off,
                                                  size_t perm_off, size_t gates_off, int first, int El, int TK,
                                                  const int* __restrict__ poff, const int* __restrict__ base,
                                                  int* __restrict__ row_asg, float* __restrict__ row_gate,
                                                  int* status) {
  if (status_set(status)) return;
  const int el = blockIdx.y;
  const int* b = base + el * (R + 1);
  const int n = b[R], p0 = poff[el];
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    int r = 0;
    while (r + 1 < R && b[r + 1] <= i) ++r;
    const int li = i - b[r];
    const int pos = reinterpret_cast<const int*>(P.base[r] + offsets_off)[first + el] + li;
    const int a = pos >= 0 && pos < TK ? reinterpret_cast<const int*>(P.base[r] + perm_off)[pos] : -1;
    if (a < 0 || a >= TK) {  // tables that do not match: leave the row as padding
      raise_status(status, MOE_ERR_EXCHANGE);
      continue;
    }
    row_asg[p0 + i] = r * TK + a;
    row_gate[p0 + i] = reinterpret_cast<const float*>(P.base[r] + gates_off)[a];
  }
}

__global__ void __launch_bounds__(128) k_ep_gather(const __grid_constant__ EpPeers P, size_t src_off, int TK, int k,
                                                   int d, const int* __restrict__ poff, int El,
                                                   const int* __restrict__ row_asg, int64_t max_rows,
                                                   __nv_bfloat16* __restrict__ dst, int* status) {
  if (status_set(status)) return;
  const int64_t r0 = poff[0], r1 = poff[El] < max_rows ? poff[El] : max_rows;
  const int nv = d / 8;
  for (int64_t R = r0 + blockIdx.x; R < r1; R += gridDim.x) {
    const int ae = row_asg[R];
    if (ae == ROW_DEAD) continue;
    uint4* out = reinterpret_cast<uint4*>(dst + R * d);
    const uint4* in = nullptr;
    if (ae >= 0) {
      const int r = ae / TK, a = ae - r * TK;
      in = reinterpret_cast<const uint4*>(P.base[r] + src_off + static_cast<size_t>(a / k) * d * 2);
    }
    for (int i0 = threadIdx.x; i0 < nv; i0 += 4 * blockDim.x) {
      uint4 u[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = i0 + j * blockDim.x;
        u[j] = (in != nullptr && i < nv) ? in[i] : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = i0 + j * blockDim.x;
        if (i < nv) out[i] = u[j];
      }
    }
  }
}

__global__ void __launch_bounds__(128) k_ep_push_rows(const __grid_constant__ EpPeers P, size_t dst_off, int TK,
                                                      int d, const int* __restrict__ poff, int El,
                                                      const int* __restrict__ row_asg, int64_t max_rows,
                                                      const __nv_bfloat16* __restrict__ src, int* status) {
  if (status_set(status)) return;
  const int64_t r0 = poff[0], r1 = poff[El] < max_rows ? poff[El] : max_rows;
  const int nv = d / 8;
  for (int64_t R = r0 + blockIdx.x; R < r1; R += gridDim.x) {
    const int ae = row_asg[R];
    if (ae < 0) continue;
    const int r = ae / TK, a = ae - r * TK;
    uint4* out = reinterpret_cast<uint4*>(P.base[r] + dst_off + static_cast<size_t>(a) * d * 2);
    const uint4* in = reinterpret_cast<const uint4*>(src + R * d);
    for (int i0 = threadIdx.x; i0 < nv; i0 += 4 * blockDim.x) {
      uint4 u[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = i0 + j * blockDim.x;
        u[j] = i < nv ? __ldg(in + i) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = i0 + j * blockDim.x;
        if (i < nv) out[i] = u[j];
      }
    }
  }
  __threadfence_system();  // the pushed rows before the done flag the next kernel writes
}

__global__ void __launch_bounds__(256) k_ep_push_dg(const __grid_constant__ EpPeers P, size_t dst_off, int TK,
                                                    const int* __restrict__ poff, int El,
                                                    const int* __restrict__ row_asg, const float* __restrict__ dgpart,
                                                    int ntn, int64_t max_rows, int* status) {
  if (status_set(status)) return;
  const int64_t r0 = poff[0], r1 = poff[El] < max_rows ? poff[El] : max_rows;
  for (int64_t R = r0 + blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; R < r1;
       R += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int ae = row_asg[R];
    if (ae < 0) continue;
    float dg = 0.f;  // the partials of the dgrad-down GEMM's n-tiles, in order
    for (int q = 0; q < ntn; ++q) dg += dgpart[R * ntn + q];
    const int r = ae / TK, a = ae - r * TK;
    reinterpret_cast<float*>(P.base[r] + dst_off)[a] = dg;
  }
  __threadfence_system();
}

__global__ void k_ep_identity(int* slot_row, int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    slot_row[i] = static_cast<int>(i);
}

static int ep_grid(int64_t rows) { return static_cast<int>(rows < 148 * 8 ? (rows > 0 ? rows : 1) : 148 * 8); }

cudaError_t launch_ep_signal(const EpPeers& P, int R, int self, bool all, size_t flags_off, int idx, int epoch,
                             cudaStream_t st) {
  k_ep_signal<<<1, kEpMaxRanks, 0, st>>>(P, R, self, all ? 1 : 0, flags_off, idx, epoch);
  return cudaGetLastError();
}
cudaError_t launch_ep_wait(const EpPeers& P, int R, int self, bool own, size_t flags_off, int idx, int epoch,
                           int* status, cudaStream_t st) {
  k_ep_wait<<<1, kEpMaxRanks, 0, st>>>(P, R, self, own ? 1 : 0, flags_off, idx, epoch, status);
  return cudaGetLastError();
}
cudaError_t launch_ep_plan(const EpPeers& P, int R, size_t counts_off, int first, int El, int64_t max_rows,
                           int* counts, int* poff, int* base, int* hdr, int* status, cudaStream_t st) {
  k_ep_plan<<<1, 512, 0, st>>>(P, R, counts_off, first, El, max_rows, counts, poff, base, hdr, status);
  return cudaGetLastError();
}
cudaError_t launch_ep_table(const EpPeers& P, int R, const EpBuf& B, int first, int El, int TK, const int* poff,
                            const int* base, int* row_asg, float* row_gate, int* status, cudaStream_t st) {
  k_ep_table<<<dim3(8, El), 256, 0, st>>>(P, R, B.offsets, B.perm_asg, B.gates, first, El, TK, poff, base, row_asg,
                                          row_gate, status);
  return cudaGetLastError();
}
cudaError_t launch_ep_gather(const EpPeers& P, size_t src_off, int TK, int k, int d, const int* poff, int El,
                             const int* row_asg, int64_t max_rows, __nv_bfloat16* dst, int* status, cudaStream_t st) {
  k_ep_gather<<<ep_grid(max_rows), 128, 0, st>>>(P, src_off, TK, k, d, poff, El, row_asg, max_rows, dst, status);
  return cudaGetLastError();
}
cudaError_t launch_ep_push_rows(const EpPeers& P, size_t dst_off, int TK, int d, const int* poff, int El,
                                const int* row_asg, int64_t max_rows, const __nv_bfloat16* src, int* status,
                                cudaStream_t st) {
  k_ep_push_rows<<<ep_grid(max_rows), 128, 0, st>>>(P, dst_off, TK, d, poff, El, row_asg, max_rows, src, status);
  return cudaGetLastError();
}
cudaError_t launch_ep_push_dg(const EpPeers& P, size_t dst_off, int TK, const int* poff, int El, const int* row_asg,
                              const float* dgpart, int ntn, int64_t max_rows, int* status, cudaStream_t st) {
  k_ep_push_dg<<<ep_grid((max_rows + 255) / 256), 256, 0, st>>>(P, dst_off, TK, poff, El, row_asg, dgpart, ntn,
                                                                 max_rows, status);
  return cudaGetLastError();
}
cudaError_t launch_ep_identity(int* slot_row, int64_t n, cudaStream_t st) {
  k_ep_identity<<<ep_grid((n + 255) / 256), 256, 0, st>>>(slot_row, n);
  return cudaGetLastError();
}

}  // namespace moe
