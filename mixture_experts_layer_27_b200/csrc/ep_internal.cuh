// Expert parallelism across ranks (see ep.cu): the per-rank exchange buffer and the
// exchange kernels' launchers.  Internal to libmoe.so.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace moe {

constexpr int kEpMaxRanks = 64;

// Byte offsets of the regions of one rank's exchange buffer (each 256-byte aligned).  Peers
// read the routing table, X and dY of a source rank (pull), and write into its receive
// regions (push).  flags: [0] forward ready, [1] backward ready (written by the rank itself,
// read by its peers), [2 + q] forward done and [2 + R + q] backward done (written by owner q
// once its pushes into this buffer are complete).
struct EpBuf {
  size_t flags, counts, offsets, perm_asg, gates, x, dy, recv_o, recv_dx, recv_dg, bytes;
};
EpBuf ep_buffer_layout(int64_t T, int k, int E, int d, int R);
enum EpFlagIdx { EPF_FWD_READY = 0, EPF_BWD_READY = 1, EPF_DONE = 2 };

// Base addresses of all ranks' exchange buffers (this process's mapping), by value.
struct EpPeers {
  uint8_t* base[kEpMaxRanks];
};

// Sets flag `idx` to `epoch`: in every rank's buffer (all = true) or in rank `self`'s only.
cudaError_t launch_ep_signal(const EpPeers& P, int R, int self, bool all, size_t flags_off, int idx, int epoch,
                             cudaStream_t st);
// Waits (bounded, about 2 s) until flag `idx` of every rank's buffer (own = false) or flags
// idx .. idx + R - 1 of rank `self`'s buffer (own = true) equal `epoch`; on expiry records
// MOE_ERR_DEVICE_TIMEOUT in *status.
cudaError_t launch_ep_wait(const EpPeers& P, int R, int self, bool own, size_t flags_off, int idx, int epoch,
                           int* status, cudaStream_t st);
// Owner: rows per local expert from every source's counts, their prefix over sources
// base[el * (R + 1) + r], counts[first + el], padded offsets poff[El + 1], hdr rows.
cudaError_t launch_ep_plan(const EpPeers& P, int R, size_t counts_off, int first, int El, int64_t max_rows,
                           int* counts, int* poff, int* base, int* hdr, int* status, cudaStream_t st);
// Owner: the assignment (source r, index a of r's T k assignments; encoded r * TK + a) and
// gate of every real row, from the sources' expert-major tables.
cudaError_t launch_ep_table(const EpPeers& P, int R, const EpBuf& B, int first, int El, int TK, const int* poff,
                            const int* base, int* row_asg, float* row_gate, int* status, cudaStream_t st);
// Owner: rows [poff[0], poff[El]) of dst from the sources' token rows at region src_off
// (token a / k of the row's assignment); live pad rows zero, dead pad rows untouched.
cudaError_t launch_ep_gather(const EpPeers& P, size_t src_off, int TK, int k, int d, const int* poff, int El,
                             const int* row_asg, int64_t max_rows, __nv_bfloat16* dst, int* status, cudaStream_t st);
// Owner: every real row of src to its source's receive region dst_off, at its assignment.
cudaError_t launch_ep_push_rows(const EpPeers& P, size_t dst_off, int TK, int d, const int* poff, int El,
                                const int* row_asg, int64_t max_rows, const __nv_bfloat16* src, int* status,
                                cudaStream_t st);
// Owner: each real row's router-gate gradient (its ntn partials summed in order) to its source.
cudaError_t launch_ep_push_dg(const EpPeers& P, size_t dst_off, int TK, const int* poff, int El, const int* row_asg,
                              const float* dgpart, int ntn, int64_t max_rows, int* status, cudaStream_t st);
// slot_row[a] = a (a source's receive regions are indexed by assignment)
cudaError_t launch_ep_identity(int* slot_row, int64_t n, cudaStream_t st);

}  // namespace moe
