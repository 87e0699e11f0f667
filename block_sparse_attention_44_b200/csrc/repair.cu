// Runtime mask repair, compaction, realised per-head workload and the
// heavy-first work list ("FVAttn: Adaptive Sparse Attention with Runtime Load
// Balancing for Video Generation": abstract — the materialised mask is repaired
// at run time; §2 sequence parallelism — per-head workload W_h as the count of
// kept block pairs; §3.2 — heads are the unit of rebalancing, whose single-GPU
// counterpart here is a longest-processing-time-first order of (b, h, i) items).
//
//   compact_kernel — one warp per (b, h, i) row: kept = Top-p mask | Top-k floor |
//                    diagonal, written as an ascending id list with ballot/popc.
//   lpt_kernel     — one CTA per count value (stable counting sort by count,
//                    descending, without atomics) plus one CTA per head for W_h.
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

// Block-wide exclusive prefix sum of v (every thread of a kLptThreads CTA calls it);
// returns the exclusive prefix and the total in *total.
__device__ __forceinline__ unsigned block_exclusive_scan(unsigned v, unsigned* total, unsigned* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sh[warp] = incl;
  __syncthreads();
  unsigned before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kLptThreads / 32; ++w) {
    const unsigned t = sh[w];
    if (w < warp) before += t;
    all += t;
  }
  __syncthreads();   // sh may be reused by the caller
  *total = all;
  return before + incl - v;
}

// grid.x = (Nb + 1) + BH.  CTA c <= Nb places the items whose count is c: they start
// after every item with a larger count (descending order) and keep their item order
// (ties by item id ascending).  Each thread owns a contiguous run of items, counts the
// larger and equal ones in a first pass over the counts, and after a block scan writes
// its equal items in order in a second pass.  The remaining BH CTAs write
// W_h = sum of the counts of head h.  No atomics: the result is deterministic.
__global__ void __launch_bounds__(kLptThreads) lpt_kernel(const int32_t* __restrict__ counts, long long BH, int Nb,
                                                          int64_t* __restrict__ head_work,
                                                          int32_t* __restrict__ worklist) {
  __shared__ unsigned sh[kLptThreads / 32];
  __shared__ long long shs[kLptThreads / 32];
  const long long n = BH * Nb;
  const int c = static_cast<int>(blockIdx.x);
  if (c > Nb) {   // realised per-head workload
    const long long bh = c - (Nb + 1);
    long long s = 0;
    for (int i = threadIdx.x; i < Nb; i += kLptThreads) s += __ldg(counts + bh * Nb + i);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if ((threadIdx.x & 31) == 0) shs[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
      long long t = 0;
      for (int w = 0; w < kLptThreads / 32; ++w) t += shs[w];
      head_work[bh] = t;
    }
    return;
  }
  const long long per = (n + kLptThreads - 1) / kLptThreads;
  const long long lo = threadIdx.x * per;
  const long long hi = min(n, lo + per);
  unsigned gt = 0, eq = 0;
#pragma unroll 8
  for (long long u = lo; u < hi; ++u) {
    const int v = __ldg(counts + u);
    gt += v > c ? 1u : 0u;
    eq += v == c ? 1u : 0u;
  }
  unsigned larger, equal;
  (void)block_exclusive_scan(gt, &larger, sh);
  unsigned pos = block_exclusive_scan(eq, &equal, sh) + larger;
  if (equal == 0 || eq == 0) return;   // nothing of this count in this thread's run
#pragma unroll 8
  for (long long u = lo; u < hi; ++u)
    if (__ldg(counts + u) == c) worklist[pos++] = static_cast<int32_t>(u);
}

}  // namespace

cudaError_t launch_lpt(const int32_t* counts, const Dims& D, int64_t* head_work, int32_t* worklist, cudaStream_t s,
                       int* launches) {
  const unsigned grid = static_cast<unsigned>(D.Nb + 1 + D.BH());
  lpt_kernel<<<grid, kLptThreads, 0, s>>>(counts, D.BH(), D.Nb, head_work, worklist);
  ++*launches;
  return cudaGetLastError();
}

cudaError_t launch_repair(const uint8_t* topp_mask, const int32_t* topk_idx, const Dims& D, int kk, int32_t* counts,
                          int32_t* idx, int64_t* head_work, int32_t* worklist, int* dev_err, cudaStream_t s,
                          int* launches) {
  const unsigned cgrid = static_cast<unsigned>((D.rows() + kCompactWarps - 1) / kCompactWarps);
  const size_t csmem = static_cast<size_t>(kCompactWarps) * D.Nb;
  compact_kernel<<<cgrid, kCompactWarps * 32, csmem, s>>>(topp_mask, topk_idx, D.rows(), D.Nb, kk, counts, idx,
                                                          dev_err);
  ++*launches;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_lpt(counts, D, head_work, worklist, s, launches);
}

}  // namespace fva
