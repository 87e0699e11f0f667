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
//                    stays deterministic; the counts are staged in shared memory
//                    when they fit.
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

constexpr int kLptBatch = 8;   // counts loaded per lane before they are used

// One CTA of NW warps.  Items are split into NW contiguous chunks; warp w histograms
// its chunk, so a stable scatter only needs, per count value, the number of items in
// earlier chunks and the running position inside the warp's own chunk.  With `staged`
// the counts are first copied to shared memory (one pass over global memory).
template <int NW>
__global__ void __launch_bounds__(NW * 32) lpt_kernel(const int32_t* __restrict__ counts, long long BH, int Nb,
                                                      int staged, int64_t* __restrict__ head_work,
                                                      int32_t* __restrict__ worklist) {
  extern __shared__ unsigned lpt_smem[];
  const int nb1 = Nb + 1;                       // counts are in [0, Nb]
  unsigned* hist = lpt_smem;                    // [NW][nb1], later the per-warp cursors
  unsigned* start = lpt_smem + NW * nb1;        // [nb1]: items with a larger count (descending order)
  int32_t* sc = reinterpret_cast<int32_t*>(start + nb1);   // [n] when staged
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  const long long n = BH * Nb;
  const long long chunk = (n + NW - 1) / NW;
  const long long lo = warp * chunk;
  const long long hi = min(n, lo + chunk);

  for (int e = threadIdx.x; e < NW * nb1; e += blockDim.x) hist[e] = 0;
  if (staged) {
    for (long long base = 0; base < n; base += static_cast<long long>(blockDim.x) * kLptBatch) {
      int c[kLptBatch];
#pragma unroll
      for (int t = 0; t < kLptBatch; ++t) {
        const long long u = base + threadIdx.x + static_cast<long long>(blockDim.x) * t;
        c[t] = u < n ? __ldg(counts + u) : 0;
      }
#pragma unroll
      for (int t = 0; t < kLptBatch; ++t) {
        const long long u = base + threadIdx.x + static_cast<long long>(blockDim.x) * t;
        if (u < n) sc[u] = c[t];
      }
    }
  }
  __syncthreads();
  const int32_t* cs = staged ? sc : counts;
  for (long long base = lo; base < hi; base += 32 * kLptBatch) {
    int c[kLptBatch];
#pragma unroll
    for (int t = 0; t < kLptBatch; ++t) {
      const long long u = base + lane + 32 * t;
      c[t] = u < hi ? cs[u] : -1;
    }
#pragma unroll
    for (int t = 0; t < kLptBatch; ++t)
      if (c[t] >= 0) atomicAdd(&hist[warp * nb1 + c[t]], 1u);
  }
  // realised per-head workload
  for (long long bh = warp; bh < BH; bh += NW) {
    long long s = 0;
    for (int i0 = 0; i0 < Nb; i0 += 32 * kLptBatch) {
      int c[kLptBatch];
#pragma unroll
      for (int t = 0; t < kLptBatch; ++t) {
        const int i = i0 + lane + 32 * t;
        c[t] = i < Nb ? cs[bh * Nb + i] : 0;
      }
#pragma unroll
      for (int t = 0; t < kLptBatch; ++t) s += c[t];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) head_work[bh] = s;
  }
  __syncthreads();
  // per count value: total over the chunks (kept in start[] for now)
  for (int v = threadIdx.x; v < nb1; v += blockDim.x) {
    unsigned t = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) t += hist[w * nb1 + v];
    start[v] = t;
  }
  __syncthreads();
  // exclusive scan over count values from high to low (warp 0; lane l owns a run)
  if (warp == 0) {
    const int per = (nb1 + 31) / 32;
    unsigned tot = 0;
    for (int q = 0; q < per; ++q) {
      const int v = Nb - lane * per - q;
      if (v >= 0) tot += start[v];
    }
    unsigned incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    unsigned run = incl - tot;
    for (int q = 0; q < per; ++q) {
      const int v = Nb - lane * per - q;
      if (v >= 0) {
        const unsigned t = start[v];
        start[v] = run;
        run += t;
      }
    }
  }
  __syncthreads();
  // per-warp cursors: warp w's items of count v follow those of warps < w
  for (int v = threadIdx.x; v < nb1; v += blockDim.x) {
    unsigned run = start[v];
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const unsigned t = hist[w * nb1 + v];
      hist[w * nb1 + v] = run;
      run += t;
    }
  }
  __syncthreads();
  // stable scatter in item order within each warp's chunk, 32 items per step
  for (long long base = lo; base < hi; base += 32 * kLptBatch) {
    int c[kLptBatch];
#pragma unroll
    for (int t = 0; t < kLptBatch; ++t) {
      const long long u = base + lane + 32 * t;
      c[t] = u < hi ? cs[u] : -1;
    }
#pragma unroll
    for (int t = 0; t < kLptBatch; ++t) {
      const long long u = base + lane + 32 * t;
      const bool valid = c[t] >= 0;
      const unsigned peers = __match_any_sync(0xffffffffu, c[t]);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int leader = __ffs(peers) - 1;
      const unsigned basepos = valid ? hist[warp * nb1 + c[t]] : 0u;
      __syncwarp();
      if (valid && lane == leader) hist[warp * nb1 + c[t]] = basepos + __popc(peers);
      __syncwarp();
      if (valid) worklist[basepos + rank] = static_cast<int32_t>(u);
    }
  }
}

}  // namespace

cudaError_t launch_lpt(const int32_t* counts, const Dims& D, int64_t* head_work, int32_t* worklist, cudaStream_t s,
                       int* launches) {
  // 32 warps with the counts staged in shared memory when everything fits, else 16
  // warps reading the counts from global memory
  constexpr size_t kMaxSmem = 227 * 1024;
  const size_t nb1 = static_cast<size_t>(D.Nb) + 1;
  const size_t n = static_cast<size_t>(D.rows());
  const size_t big = (32 + 1) * nb1 * sizeof(unsigned) + n * sizeof(int32_t);
  cudaError_t e;
  if (big <= kMaxSmem) {
    e = cudaFuncSetAttribute(lpt_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(big));
    if (e != cudaSuccess) return e;
    lpt_kernel<32><<<1, 32 * 32, big, s>>>(counts, D.BH(), D.Nb, 1, head_work, worklist);
  } else {
    const size_t small = (16 + 1) * nb1 * sizeof(unsigned);
    e = cudaFuncSetAttribute(lpt_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(small));
    if (e != cudaSuccess) return e;
    lpt_kernel<16><<<1, 16 * 32, small, s>>>(counts, D.BH(), D.Nb, 0, head_work, worklist);
  }
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
