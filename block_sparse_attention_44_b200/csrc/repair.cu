// Runtime mask repair, compaction, realised per-head workload and the
// heavy-first work list ("FVAttn: Adaptive Sparse Attention with Runtime Load
// Balancing for Video Generation": abstract — the materialised mask is repaired
// at run time; §2 sequence parallelism — per-head workload W_h as the count of
// kept block pairs; §3.2 — heads are the unit of rebalancing, whose single-GPU
// counterpart here is a longest-processing-time-first order of (b, h, i) items).
//
//   compact_kernel — one warp per (b, h, i) row: kept = Top-p mask | Top-k floor |
//                    diagonal, written as an ascending id list with ballot/popc.
//   lpt_*_kernel   — W_h and the work list: a stable counting sort of the items by
//                    count, descending, in three passes (histograms per head, list
//                    offsets, scatter), without output atomics.
#include "fva_common.cuh"
#include "fva_internal.h"

namespace fva {
namespace {

constexpr int kCompactWarps = 8;

__global__ void __launch_bounds__(kCompactWarps * 32) compact_kernel(const uint8_t* __restrict__ topp_mask,
                                                                     const int32_t* __restrict__ topk_idx,
                                                                     long long rows, int Nb, int kk,
                                                                     int32_t* __restrict__ counts,
                                                                     int32_t* __restrict__ idx, int* dev_err) {
  extern __shared__ unsigned char keep_smem[];
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * kCompactWarps + warp;
  if (row >= rows) return;
  unsigned char* keep = keep_smem + static_cast<size_t>(warp) * Nb;
  const int i = static_cast<int>(row % Nb);
  const uint8_t* mrow = topp_mask + row * Nb;
  for (int t = lane; t < Nb; t += 32) keep[t] = mrow[t] ? 1 : 0;
  __syncwarp();
  const int32_t* krow = topk_idx + row * kk;
  for (int q = lane; q < kk; q += 32) {
    const int j = krow[q];
    if (j >= 0 && j < Nb)
      keep[j] = 1;
    else
      set_device_error(dev_err, kDevErrBadIndex);
  }
  if (lane == 0) keep[i] = 1;
  __syncwarp();
  int32_t* irow = idx + row * Nb;
  int pos = 0;
  for (int base = 0; base < Nb; base += 32) {
    const int t = base + lane;
    const bool in = t < Nb && keep[t];
    const unsigned bal = __ballot_sync(0xffffffffu, in);
    if (in) irow[pos + __popc(bal & ((1u << lane) - 1u))] = t;
    pos += __popc(bal);
  }
  if (lane == 0) counts[row] = pos;
}

constexpr int kLptThreads = 256;
constexpr int kLptScanThreads = 1024;

// Sort key of a count: clamped into [0, Nb] (the attention kernel reads counts the same way).
__device__ __forceinline__ int lpt_key(int c, int Nb) { return c < 0 ? 0 : (c > Nb ? Nb : c); }

// The LPT work list is a stable counting sort of the items u = bh * Nb + i by count,
// descending, in three passes over the B*H heads ("chunks" of Nb items), none with
// output atomics, so the list is deterministic:
//   lpt_hist_kernel    — per chunk: histogram of its counts over [0, Nb], and W_h;
//   lpt_offsets_kernel — one CTA: for every count value v (descending) and chunk c
//                        (ascending), the list position of the first item of chunk c
//                        with count v, written over the histogram;
//   lpt_scatter_kernel — per chunk: one warp walks the chunk's items in order, 32 at a
//                        time; items with equal counts take consecutive positions
//                        (warp match + running per-value cursors in shared memory).
// Work is O(B*H*Nb) plus O(B*H*Nb) for the offsets (histogram entries).

// grid.x = BH; hist: [BH][Nb + 1] int32 output; head_work[bh] = sum of the counts.
__global__ void __launch_bounds__(kLptThreads) lpt_hist_kernel(const int32_t* __restrict__ counts, int Nb,
                                                               int32_t* __restrict__ hist,
                                                               int64_t* __restrict__ head_work) {
  extern __shared__ int h_smem[];
  __shared__ long long part[kLptThreads / 32];
  const long long bh = blockIdx.x;
  for (int v = threadIdx.x; v <= Nb; v += kLptThreads) h_smem[v] = 0;
  __syncthreads();
  long long s = 0;
  for (int i = threadIdx.x; i < Nb; i += kLptThreads) {
    const int c = __ldg(counts + bh * Nb + i);
    s += c;
    atomicAdd(&h_smem[lpt_key(c, Nb)], 1);   // order-free counts: deterministic
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    long long t = 0;
    for (int w = 0; w < kLptThreads / 32; ++w) t += part[w];
    head_work[bh] = t;
  }
  for (int v = threadIdx.x; v <= Nb; v += kLptThreads) hist[bh * (Nb + 1) + v] = h_smem[v];
}

// One CTA.  Thread-owned values v: total[v] = sum over chunks; base[v] = number of items
// with a larger count (block scan over v descending); then hist[c][v] is replaced by
// base[v] + sum of hist[c'][v] over chunks c' < c.  STAGED: the histograms are first
// copied into shared memory in one coalesced pass, so the two passes over the chunks read
// shared memory instead of waiting on dependent rounds of global loads.
template <bool STAGED>
__global__ void __launch_bounds__(kLptScanThreads) lpt_offsets_kernel(int32_t* __restrict__ hist, long long BH,
                                                                      int Nb) {
  constexpr int VPT = (kMaxNb + 1 + kLptScanThreads - 1) / kLptScanThreads;   // values per thread
  __shared__ long long warp_tot[kLptScanThreads / 32];
  extern __shared__ int32_t staged[];
  const int V = Nb + 1;
  const int32_t* src = hist;
  if (STAGED) {
    const long long n = BH * V;
#pragma unroll 8
    for (long long e = threadIdx.x; e < n; e += kLptScanThreads) staged[e] = hist[e];
    __syncthreads();
    src = staged;
  }
  // thread t owns the values v = V - 1 - (t * VPT + e), e < VPT: descending order runs
  // with the thread index, so an exclusive scan over threads gives "larger counts first"
  long long tot[VPT];
  long long mine = 0;
#pragma unroll
  for (int e = 0; e < VPT; ++e) {
    const int r = threadIdx.x * VPT + e;   // rank of the value in descending order
    tot[e] = 0;
    if (r < V) {
      const int v = V - 1 - r;
#pragma unroll 8
      for (long long c = 0; c < BH; ++c) tot[e] += src[c * V + v];
    }
    mine += tot[e];
  }
  // exclusive scan of `mine` over the threads
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  long long incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  long long before = 0;
  for (int w = 0; w < warp; ++w) before += warp_tot[w];
  long long base = before + incl - mine;
#pragma unroll
  for (int e = 0; e < VPT; ++e) {
    const int r = threadIdx.x * VPT + e;
    if (r < V) {
      const int v = V - 1 - r;
      long long run = base;
#pragma unroll 8
      for (long long c = 0; c < BH; ++c) {
        const int n = src[c * V + v];
        hist[c * V + v] = static_cast<int32_t>(run);
        run += n;
      }
    }
    base += tot[e];
  }
}

// grid.x = BH, one warp per CTA.  off: [BH][Nb + 1] first positions from lpt_offsets_kernel.
// The head's counts are staged in shared memory first (one coalesced pass), so the
// sequential 32-item steps touch only shared memory and the list.
__global__ void __launch_bounds__(32) lpt_scatter_kernel(const int32_t* __restrict__ counts, int Nb,
                                                         const int32_t* __restrict__ off,
                                                         int32_t* __restrict__ worklist) {
  extern __shared__ int cursor[];        // [Nb + 1] cursors, then [Nb] counts
  int* cnt = cursor + Nb + 1;
  const long long bh = blockIdx.x;
  const int lane = threadIdx.x;
  for (int v = lane; v <= Nb; v += 32) cursor[v] = off[bh * (Nb + 1) + v];
  for (int i = lane; i < Nb; i += 32) cnt[i] = lpt_key(__ldg(counts + bh * Nb + i), Nb);
  __syncwarp();
  const unsigned lt = (1u << lane) - 1u;
  for (int i0 = 0; i0 < Nb; i0 += 32) {
    const int i = i0 + lane;
    const bool valid = i < Nb;
    const int key = valid ? cnt[i] : -1 - lane;   // invalid lanes match no one
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    if (valid) worklist[cursor[key] + __popc(peers & lt)] = static_cast<int32_t>(bh * Nb + i);
    __syncwarp();
    if (valid && (peers & lt) == 0) cursor[key] += __popc(peers);   // the group's first lane advances
    __syncwarp();
  }
}

}  // namespace

size_t lpt_workspace_bytes(const Dims& D) {
  return (static_cast<size_t>(D.BH()) * (D.Nb + 1) * sizeof(int32_t) + 255) & ~static_cast<size_t>(255);
}

cudaError_t launch_lpt(const int32_t* counts, const Dims& D, int64_t* head_work, int32_t* worklist, void* ws,
                       cudaStream_t s, int* launches) {
  int32_t* hist = static_cast<int32_t*>(ws);
  const unsigned grid = static_cast<unsigned>(D.BH());
  const size_t hsmem = static_cast<size_t>(D.Nb + 1) * sizeof(int);
  lpt_hist_kernel<<<grid, kLptThreads, hsmem, s>>>(counts, D.Nb, hist, head_work);
  ++*launches;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // histograms staged in shared memory when they fit (up to 227 KB less the kernel's static share)
  const size_t staged = static_cast<size_t>(D.BH()) * (D.Nb + 1) * sizeof(int32_t);
  if (staged <= 232448 - 1024) {
    e = cudaFuncSetAttribute(lpt_offsets_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(staged));
    if (e != cudaSuccess) return e;
    lpt_offsets_kernel<true><<<1, kLptScanThreads, staged, s>>>(hist, D.BH(), D.Nb);
  } else {
    lpt_offsets_kernel<false><<<1, kLptScanThreads, 0, s>>>(hist, D.BH(), D.Nb);
  }
  ++*launches;
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  lpt_scatter_kernel<<<grid, 32, hsmem + static_cast<size_t>(D.Nb) * sizeof(int), s>>>(counts, D.Nb, hist, worklist);
  ++*launches;
  return cudaGetLastError();
}

cudaError_t launch_repair(const uint8_t* topp_mask, const int32_t* topk_idx, const Dims& D, int kk, int32_t* counts,
                          int32_t* idx, int64_t* head_work, int32_t* worklist, void* ws, int* dev_err,
                          cudaStream_t s, int* launches) {
  const unsigned cgrid = static_cast<unsigned>((D.rows() + kCompactWarps - 1) / kCompactWarps);
  const size_t csmem = static_cast<size_t>(kCompactWarps) * D.Nb;
  compact_kernel<<<cgrid, kCompactWarps * 32, csmem, s>>>(topp_mask, topk_idx, D.rows(), D.Nb, kk, counts, idx,
                                                          dev_err);
  ++*launches;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_lpt(counts, D, head_work, worklist, ws, s, launches);
}

}  // namespace fva
