// Runtime mask repair, compaction, realised per-head workload and the
// heavy-first work list ("FVAttn: Adaptive Sparse Attention with Runtime Load
// Balancing for Video Generation": abstract — the materialised mask is repaired
// at run time; §2 sequence parallelism — per-head workload W_h as the count of
// kept block pairs; §3.2 — heads are the unit of rebalancing, whose single-GPU
// counterpart here is a longest-processing-time-first order of (b, h, i) items).
//
//   compact_kernel — one warp per (b, h, i) row: kept = Top-p mask | Top-k floor |
//                    diagonal, written as an ascending id list with ballot/popc.
//   lpt_kernel     — one CTA: per-head sums, then a stable counting sort of all
//                    items by count (descending) with per-warp histograms so it
//                    stays deterministic.
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

constexpr int kLptWarps = 16;

__global__ void __launch_bounds__(kLptWarps * 32) lpt_kernel(const int32_t* __restrict__ counts, long long BH, int Nb,
                                                             int64_t* __restrict__ head_work,
                                                             int32_t* __restrict__ worklist) {
  extern __shared__ unsigned lpt_smem[];
  const int nb1 = Nb + 1;                       // counts are in [1, Nb]
  unsigned* hist = lpt_smem;                    // [kLptWarps][nb1], later the per-warp cursors
  unsigned* start = lpt_smem + kLptWarps * nb1; // [nb1]: first position of each count value
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  const long long n = BH * Nb;
  const long long chunk = (n + kLptWarps - 1) / kLptWarps;
  const long long lo = warp * chunk;
  const long long hi = min(n, lo + chunk);

  for (int e = threadIdx.x; e < kLptWarps * nb1; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  for (long long u = lo + lane; u < hi; u += 32) atomicAdd(&hist[warp * nb1 + counts[u]], 1u);
  // realised per-head workload
  for (long long bh = warp; bh < BH; bh += kLptWarps) {
    long long s = 0;
    for (int i = lane; i < Nb; i += 32) s += counts[bh * Nb + i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) head_work[bh] = s;
  }
  __syncthreads();
  // start[c] = number of items with a larger count (descending order)
  if (warp == 0) {
    const int per = (nb1 + 31) / 32;
    // lane l owns count values c in (Nb - l*per - per, Nb - l*per], scanned high to low
    unsigned tot = 0;
    for (int q = 0; q < per; ++q) {
      const int c = Nb - lane * per - q;
      if (c >= 0)
        for (int w = 0; w < kLptWarps; ++w) tot += hist[w * nb1 + c];
    }
    unsigned incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    unsigned run = incl - tot;
    for (int q = 0; q < per; ++q) {
      const int c = Nb - lane * per - q;
      if (c >= 0) {
        start[c] = run;
        for (int w = 0; w < kLptWarps; ++w) run += hist[w * nb1 + c];
      }
    }
  }
  __syncthreads();
  // per-warp cursors: warp w's items of count c follow those of warps < w
  for (int c = threadIdx.x; c < nb1; c += blockDim.x) {
    unsigned run = start[c];
    for (int w = 0; w < kLptWarps; ++w) {
      const unsigned t = hist[w * nb1 + c];
      hist[w * nb1 + c] = run;
      run += t;
    }
  }
  __syncthreads();
  // stable scatter, 32 items at a time, in item order within each warp's chunk
  for (long long b0 = lo; b0 < hi; b0 += 32) {
    const long long u = b0 + lane;
    const bool valid = u < hi;
    const int c = valid ? counts[u] : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, c);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    const int leader = __ffs(peers) - 1;
    const unsigned basepos = valid ? hist[warp * nb1 + c] : 0u;
    __syncwarp();
    if (valid && lane == leader) hist[warp * nb1 + c] = basepos + __popc(peers);
    __syncwarp();
    if (valid) worklist[basepos + rank] = static_cast<int32_t>(u);
  }
}

}  // namespace

cudaError_t launch_repair(const uint8_t* topp_mask, const int32_t* topk_idx, const Dims& D, int kk, int32_t* counts,
                          int32_t* idx, int64_t* head_work, int32_t* worklist, int* dev_err, cudaStream_t s,
                          int* launches) {
  const unsigned cgrid = static_cast<unsigned>((D.rows() + kCompactWarps - 1) / kCompactWarps);
  const size_t csmem = static_cast<size_t>(kCompactWarps) * D.Nb;
  compact_kernel<<<cgrid, kCompactWarps * 32, csmem, s>>>(topp_mask, topk_idx, D.rows(), D.Nb, kk, counts, idx,
                                                          dev_err);
  ++*launches;
  const size_t lsmem = (static_cast<size_t>(kLptWarps) + 1) * (D.Nb + 1) * sizeof(unsigned);
  cudaError_t e = cudaFuncSetAttribute(lpt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(lsmem));
  if (e != cudaSuccess) return e;
  lpt_kernel<<<1, kLptWarps * 32, lsmem, s>>>(counts, D.BH(), D.Nb, head_work, worklist);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace fva
