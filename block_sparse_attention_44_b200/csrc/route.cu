// Routing frontend: pooled Q/K block scores, Top-p CDF cut, Top-k floor, and
// (optionally) the per-row repair and compaction of the kept set
// ("FVAttn: Adaptive Sparse Attention with Runtime Load Balancing for Video
// Generation", §2 background on dynamic block-sparse routing and §3.1 overview;
// abstract: the mask is repaired at run time).
//
// Two kernels:
//   pool_kernel   — one CTA per (b, h, block) of Q and of K: the float64 mean of its S
//                   bf16 rows.  HBM-bound: every Q/K byte is read once here.
//   select_kernel — one CTA per R query blocks (rows i) of one (b, h): their float64
//                   logits L_ij = Qbar_i . Kbar_j / sqrt(d) against every key block on
//                   the FP64 tensor path (mma.sync m8n8k4), then one warp per row:
//                   softmax, Top-p boundary, Top-k floor, outputs (mask, floor ids,
//                   logits, compacted kept list).
// Both run on the caller's stream, one after the other.  (Splitting the heads into
// chunks and selecting chunk c on a second stream while chunk c + 1 is pooled was
// measured slower: the two kernels compete for the same SM registers and issue slots,
// and the per-chunk grids lose their wave tails.)
//
// Selection arithmetic (deterministic, exact integer sums):
//   - softmax weights e_j = 2^((L_ij - max_j L_ij) log2 e) in float32 (the float64
//     difference rounded once, then the hardware base-2 exponential), z = sum_j e_j
//     in float32 (per lane, then across the warp), and the mass
//     m_j = floor(e_j * (2^31 / z)) as an integer;
//   - the Top-p boundary is the first position, in the ranking (logit descending,
//     block id ascending), where the running sum of m reaches ceil(p * 2^31): found
//     by a 14-step bisection over the bucket index q_j = floor((max L - L_ij) * 256)
//     (buckets 1/256 logit wide rank like the logits; warp sums by redux.sync), then
//     inside the boundary bucket by the exact float64 logits;
//   - the Top-k floor by repeated warp argmax over (logit, -block id); argmaxes are
//     three integer warp reductions over an order-preserving key of the float64 logit,
//     so every ranking decision is exact.
// Error of the running mass at any cut against the exact cumulative softmax mass C_n
// (u = 2^-24).  Relative errors eps_j of the weights move the cut's mass by at most
// sum_j mass_j * eps_j (an error common to the kept and the dropped part cancels):
//   - the exponent argument x_j = (L_j - max) log2 e rounded to float32: eps_j <=
//     ln2 |x_j| u, and sum_j mass_j |x_j| <= log2 Nb (an entropy): 4.5e-7 at Nb = 2048;
//   - the hardware exponential, 2^-22 relative: 2.4e-7.
// z is summed in float32, sequentially over a lane's PL slots and then across the warp,
// so at most PL + 4 roundings lie on any path: (PL + 4) u relative, which moves C_n by
// 7.2e-7 (PL = 8, Nb <= 256), 1.4e-6 (PL = 20, Nb <= 640), 2.6e-6 (PL = 40, Nb <= 1280)
// or 4.1e-6 (PL = 64, Nb <= 2048).  The scaling 2^31 / z and the product add 2u
// (1.2e-7); truncating each mass to 2^-31 loses at most Nb * 2^-31 (9.5e-7 at
// Nb = 2048); weights below e^-45 set to 0 lose less than Nb e^-45 < 1e-16.
// In all: below 2.5e-6 for Nb <= 640 (the 128-token tiles of the 480p and 720p layers)
// and below 6e-6 up to Nb = 2048, inside the 1e-5 band of the parity rule's cumulative-
// mass ties.  A kept set can differ from the exact one only where the cumulative mass
// at the cut lies that close to p.
#include <limits.h>
#include <math.h>

#include <algorithm>

#include "fva_common.cuh"
#include "fva_internal.h"

namespace fva {
namespace {

constexpr int kRouteThreads = 256;
constexpr int kRouteWarps = kRouteThreads / 32;
constexpr int kPoolThreads = 256;
constexpr unsigned kQCap = 45u * 256u;  // bucket of blocks whose weight e^(L - max) < e^-45 (mass 0)
constexpr unsigned kQPad = 0xFFFFu;     // bucket of the padding columns past Nb
constexpr unsigned kFull = 0xffffffffu;
constexpr int kTopkArgmaxMax = 16;      // floors up to this size use repeated warp argmax

struct RouteArgs {
  const double* qbar;
  const double* kbar;
  uint8_t* topp_mask;   // nullable
  int32_t* topk_idx;    // nullable
  double* logits_out;   // nullable
  int32_t* counts;      // nullable (no compaction when null)
  int32_t* idx;
  int32_t* prefix_out;  // nullable: per row, max(n_p, floor) = length of the kept ranked prefix
  const int32_t* kk_rows;   // nullable: per-row floor replacing kk (topk_idx must then be null)
  int Nb, kk;
  unsigned target;      // ceil(p * 2^31)
  int keep_all_p;       // p >= 1
};

// ------------------------------------------------------------------ helpers -------
__device__ __forceinline__ void bf16x8_to_f64_add(const uint4& v, double (&acc)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    acc[2 * q] += static_cast<double>(__uint_as_float(w[q] << 16));
    acc[2 * q + 1] += static_cast<double>(__uint_as_float(w[q] & 0xFFFF0000u));
  }
}

typedef unsigned long long u64;

// Order-preserving map of a float64 logit to an unsigned key (larger logit -> larger
// key, -0 and +0 equal); key 0 lies below every finite logit and is used for "none".
__device__ __forceinline__ u64 order_key(double L) {
  if (L == 0.0) L = 0.0;
  const u64 u = static_cast<u64>(__double_as_longlong(L));
  return (u & 0x8000000000000000ull) ? ~u : (u | 0x8000000000000000ull);
}
__device__ __forceinline__ double key_value(u64 k) {
  const u64 u = (k & 0x8000000000000000ull) ? (k & 0x7FFFFFFFFFFFFFFFull) : ~k;
  return __longlong_as_double(static_cast<long long>(u));
}

// Warp-wide best (key descending, t ascending) with three integer warp reductions;
// every lane returns the winning key and t (key 0 if no lane had a candidate).
__device__ __forceinline__ void warp_best(u64 key, unsigned t, u64& bkey, unsigned& bt) {
  const unsigned khi = static_cast<unsigned>(key >> 32), klo = static_cast<unsigned>(key);
  const unsigned hi = __reduce_max_sync(kFull, khi);
  const unsigned lo = __reduce_max_sync(kFull, khi == hi ? klo : 0u);
  bt = __reduce_min_sync(kFull, (khi == hi && klo == lo) ? t : 0xFFFFFFFFu);
  bkey = (static_cast<u64>(hi) << 32) | lo;
}

__device__ __forceinline__ float warp_sum_f32(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

// ------------------------------------------------------------------ pooling -------
// grid.x = 2 * nrows: blocks row0 .. row0 + nrows - 1 of Q, then the same of K, where
// block (b*H + h)*Nb + i holds rows [i*S, (i+1)*S) of (b, h).  Thread (rg, col) sums
// the 16-byte column chunk col over rows rg, rg + RG, ...; the row groups combine in
// shared memory.  Means go to qbar[block] and kbar[block] ([B*H*Nb, D] float64).
template <int D>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(const uint4* __restrict__ qr, const uint4* __restrict__ kr,
                                                            double* __restrict__ qbar, double* __restrict__ kbar,
                                                            long long row0, long long nrows, int S) {
  constexpr int CPR = D / 8;                 // 16-byte chunks per row
  constexpr int RG = kPoolThreads / CPR;     // row groups
  __shared__ double part[RG][D];
  const bool is_k = blockIdx.x >= nrows;
  const long long blk = row0 + (is_k ? blockIdx.x - nrows : blockIdx.x);
  const int col = threadIdx.x % CPR;
  const int rg = threadIdx.x / CPR;
  double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const uint4* p = (is_k ? kr : qr) + blk * S * CPR;
#pragma unroll 8
  for (int r = rg; r < S; r += RG) bf16x8_to_f64_add(__ldg(p + r * CPR + col), acc);
#pragma unroll
  for (int e = 0; e < 8; ++e) part[rg][col * 8 + e] = acc[e];
  __syncthreads();
  double* out = is_k ? kbar : qbar;
  for (int c = threadIdx.x; c < D; c += kPoolThreads) {
    double s = 0.0;
#pragma unroll 8
    for (int g2 = 0; g2 < RG; ++g2) s += part[g2][c];
    out[blk * D + c] = s / static_cast<double>(S);
  }
}

// ------------------------------------------------------------------ selection -----
// Smallest q in [lo, hi] whose bucket-inclusive weight sum reaches T (weight = mass,
// or 1 per block when !BY_MASS).  Requires the weight of bucket hi to reach T.
template <int PL, bool BY_MASS>
__device__ __forceinline__ unsigned bisect(const unsigned (&q)[PL], const unsigned (&m)[PL], unsigned lo, unsigned hi,
                                           unsigned T) {
  while (lo < hi) {
    const unsigned mid = (lo + hi) >> 1;
    unsigned w = 0;
#pragma unroll
    for (int s = 0; s < PL; ++s)
      if (q[s] <= mid) w += BY_MASS ? m[s] : 1u;
    w = __reduce_add_sync(kFull, w);
    if (w >= T)
      hi = mid;
    else
      lo = mid + 1;
  }
  return lo;
}

// Coarse buckets (32 fine buckets each) of the live blocks: kQCap / 32 = 360 of them,
// held as kHistPerLane per lane.
constexpr int kHistPerLane = 12;
constexpr int kHistBins = 32 * kHistPerLane;   // >= kQCap / 32
static_assert(kHistBins * 32 >= static_cast<int>(kQCap), "histogram covers every live bucket");

// Smallest bucket q (over the live buckets) whose bucket-inclusive mass reaches T, and
// the mass of every bucket before it.  Requires the total mass to reach T.  Same answer
// as a bisection over q: the masses are summed per coarse bucket (q >> 5) through a
// per-warp shared-memory histogram, a warp scan finds the coarse bucket where the
// running mass reaches T, then a 32-bin histogram of that coarse bucket finds the fine
// bucket.  `hist` is this warp's kHistBins words of shared memory.
template <int PL>
__device__ __forceinline__ unsigned boundary_bucket(const unsigned (&q)[PL], const unsigned (&m)[PL], unsigned T,
                                                    unsigned* hist, unsigned& above) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int e = 0; e < kHistPerLane; ++e) hist[lane * kHistPerLane + e] = 0u;
  __syncwarp();
#pragma unroll
  for (int s = 0; s < PL; ++s)
    if (q[s] < kQCap && m[s] != 0u) atomicAdd(&hist[q[s] >> 5], m[s]);
  __syncwarp();
  unsigned lane_sum = 0;
#pragma unroll
  for (int e = 0; e < kHistPerLane; ++e) lane_sum += hist[lane * kHistPerLane + e];
  unsigned incl = lane_sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += y;
  }
  const unsigned excl = incl - lane_sum;
  // the one lane whose bins take the running mass from below T to T or more
  const bool mine = excl < T && incl >= T;
  unsigned bc = 0, before = 0;
  if (mine) {
    unsigned pre = excl;
    for (int e = 0; e < kHistPerLane; ++e) {
      const unsigned v = hist[lane * kHistPerLane + e];
      if (pre + v >= T) {
        bc = static_cast<unsigned>(lane * kHistPerLane + e);
        before = pre;
        break;
      }
      pre += v;
    }
  }
  const unsigned src = __ffs(__ballot_sync(kFull, mine)) - 1;
  bc = __shfl_sync(kFull, bc, src);
  before = __shfl_sync(kFull, before, src);
  // fine buckets of coarse bucket bc
  __syncwarp();
  hist[lane] = 0u;
  __syncwarp();
#pragma unroll
  for (int s = 0; s < PL; ++s)
    if (q[s] < kQCap && (q[s] >> 5) == bc && m[s] != 0u) atomicAdd(&hist[q[s] & 31u], m[s]);
  __syncwarp();
  const unsigned fm = hist[lane];
  unsigned finc = fm;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_up_sync(kFull, finc, o);
    if (lane >= o) finc += y;
  }
  const unsigned fexc = before + finc - fm;
  const bool hit = fexc < T && fexc + fm >= T;
  const unsigned fsrc = __ffs(__ballot_sync(kFull, hit)) - 1;
  above = __shfl_sync(kFull, fexc, fsrc);
  __syncwarp();   // hist is reused by this warp's next row
  return bc * 32u + fsrc;
}

// Walks bucket qs in ranking order from weight `acc` (the weight of every better
// bucket) until the running weight reaches T; returns that block's (key, id).
// Kr = the row's order keys in shared memory.
template <int PL, bool BY_MASS>
__device__ __forceinline__ void walk_bucket(const u64* Kr, const unsigned (&q)[PL], const unsigned (&m)[PL],
                                            unsigned qs, unsigned acc, unsigned T, u64& kb, int& jb) {
  const int lane = threadIdx.x & 31;
  u64 pkey = ~0ull;          // the last block taken, as (key, id); none yet
  unsigned pt = 0;
  for (int guard = 0; guard < 32 * PL; ++guard) {
    u64 bk = 0;
    unsigned bt = 0xFFFFFFFFu, bw = 0;
#pragma unroll
    for (int s = 0; s < PL; ++s) {
      if (q[s] != qs) continue;
      const unsigned t = lane + 32 * s;
      const u64 k = Kr[t];
      const bool after = k < pkey || (k == pkey && t > pt);
      if (after && k > bk) {   // t ascends with s: the first of equal keys is kept
        bk = k;
        bt = t;
        bw = BY_MASS ? m[s] : 1u;
      }
    }
    u64 wk;
    unsigned wt;
    warp_best(bk, bt, wk, wt);
    if (wk == 0) break;        // bucket exhausted: cannot happen when the bucket reaches T
    acc += __shfl_sync(kFull, bw, wt & 31);
    if (acc >= T) {
      kb = wk;
      jb = static_cast<int>(wt);
      return;
    }
    pkey = wk;
    pt = wt;
  }
  kb = 0;   // keep everything
  jb = INT_MAX;
}

// Block (key k, id t) ranks at or before the boundary (kb, jb).
__device__ __forceinline__ bool at_or_before(u64 k, int t, u64 kb, int jb) {
  return k > kb || (k == kb && t <= jb);
}

// Row i of (b, h) = bh; Lr = its logits in shared memory (32*PL entries, -inf past Nb),
// replaced in place by their order keys once the weights are taken.
template <int PL>
__device__ __forceinline__ void select_row(const RouteArgs& a, long long bh, int i, double* Lr, unsigned* hist) {
  const int lane = threadIdx.x & 31;
  const int Nb = a.Nb;
  const long long row = bh * Nb + i;

  double lmax = -INFINITY;
#pragma unroll
  for (int s = 0; s < PL; ++s) lmax = fmax(lmax, Lr[lane + 32 * s]);
  u64 mk;
  unsigned mt;
  warp_best(order_key(lmax), 0u, mk, mt);
  const double mx = key_value(mk);

  // weights 2^((L - max) log2 e) on the MUFU unit, summed in float32 per lane then across the warp; blocks
  // more than 45 below the max (weight < e^-45, mass 0) go to bucket kQCap
  unsigned q[PL], m[PL];
  float zl = 0.0f;
  u64* Kr = reinterpret_cast<u64*>(Lr);
#pragma unroll
  for (int s = 0; s < PL; ++s) {
    const int t = lane + 32 * s;
    const double L = Lr[t];
    const double d = L - mx;
    const bool live = d > -45.0;
    const float e = live ? ex2_approx(__double2float_rn(d * 1.4426950408889634)) : 0.0f;
    zl += e;
    m[s] = __float_as_uint(e);
    q[s] = live ? static_cast<unsigned>(-d * 256.0) : (t < Nb ? kQCap : kQPad);
    Kr[t] = order_key(L);    // this lane's own slot: no other lane reads it before the swap
  }
  const float z = warp_sum_f32(zl);
  const float scale = __fdiv_rn(0x1p31f, z);
  unsigned part = 0;
#pragma unroll
  for (int s = 0; s < PL; ++s) {
    m[s] = __float2uint_rz(__uint_as_float(m[s]) * scale);
    part += m[s];
  }
  const unsigned tot = __reduce_add_sync(kFull, part);

  // Top-p boundary (kpb, jpb): the kept set is every block ranking at or before it
  const bool all_p = a.keep_all_p || tot < a.target;
  unsigned qp = 0;
  u64 kpb = 0;
  int jpb = INT_MAX;
  if (!all_p) {
    unsigned above = 0;
    qp = boundary_bucket<PL>(q, m, a.target, hist, above);
    walk_bucket<PL, true>(Kr, q, m, qp, above, a.target, kpb, jpb);
  }

  // Top-p membership bits of this lane's blocks and the set's size n_p
  unsigned long long inp = 0;
#pragma unroll
  for (int s = 0; s < PL; ++s) {
    const int t = lane + 32 * s;
    bool in = all_p || q[s] < qp;
    if (!all_p && q[s] == qp) in = at_or_before(Kr[t], t, kpb, jpb);
    if (in && t < Nb) inp |= 1ull << s;
  }
  unsigned np_lane = 0;
#pragma unroll
  for (int s = 0; s < PL; ++s) np_lane += static_cast<unsigned>((inp >> s) & 1ull);
  const int n_p = static_cast<int>(__reduce_add_sync(kFull, np_lane));

  // Top-k floor: bit s of `taken` marks block lane + 32 s (kk <= kTopkArgmaxMax).  Both the
  // floor and the Top-p set are prefixes of the same ranking, so when the Top-p set holds
  // at least kk blocks the floor adds nothing to the kept set and is skipped unless its
  // ids are an output.
  const int kk = a.kk_rows ? a.kk_rows[row] : a.kk;
  int32_t* krow = a.topk_idx ? a.topk_idx + row * kk : nullptr;
  const bool need_floor = krow != nullptr || n_p < kk;
  unsigned long long taken = 0;
  unsigned qk = 0;
  u64 kkb = 0;
  int jkb = INT_MAX;
  unsigned mine = 0xFFFFFFFFu;   // lane c holds the c-th chosen id
  const bool big_k = kk > kTopkArgmaxMax;
  if (!need_floor) {
    // kept set = Top-p set (plus the diagonal)
  } else if (kk <= 4) {
    // each lane's four best (key descending, id ascending) in one pass, then four
    // warp-wide picks among the lane heads
    u64 k4[4] = {0, 0, 0, 0};
    unsigned s4[4] = {0, 0, 0, 0};
#pragma unroll
    for (int s = 0; s < PL; ++s) {
      const u64 k = lane + 32 * s < Nb ? Kr[lane + 32 * s] : 0ull;
      const bool c0 = k > k4[0], c1 = k > k4[1], c2 = k > k4[2], c3 = k > k4[3];
      k4[3] = c2 ? k4[2] : (c3 ? k : k4[3]);
      s4[3] = c2 ? s4[2] : (c3 ? s : s4[3]);
      k4[2] = c1 ? k4[1] : (c2 ? k : k4[2]);
      s4[2] = c1 ? s4[1] : (c2 ? s : s4[2]);
      k4[1] = c0 ? k4[0] : (c1 ? k : k4[1]);
      s4[1] = c0 ? s4[0] : (c1 ? s : s4[1]);
      k4[0] = c0 ? k : k4[0];
      s4[0] = c0 ? s : s4[0];
    }
    for (int c = 0; c < kk; ++c) {
      u64 wk;
      unsigned wt;
      warp_best(k4[0], static_cast<unsigned>(lane) + 32u * s4[0], wk, wt);
      if ((wt & 31u) == static_cast<unsigned>(lane)) {   // the winner lane pops its head
        taken |= 1ull << s4[0];
        k4[0] = k4[1];
        s4[0] = s4[1];
        k4[1] = k4[2];
        s4[1] = s4[2];
        k4[2] = k4[3];
        s4[2] = s4[3];
        k4[3] = 0;
      }
      if (lane == c) mine = wt;
    }
  } else if (!big_k) {
    for (int c = 0; c < kk; ++c) {
      u64 bk = 0;
      unsigned bt = 0xFFFFFFFFu;
#pragma unroll
      for (int s = 0; s < PL; ++s) {
        const int t = lane + 32 * s;
        if (((taken >> s) & 1ull) || t >= Nb) continue;
        const u64 k = Kr[t];
        if (k > bk) {
          bk = k;
          bt = t;
        }
      }
      u64 wk;
      unsigned wt;
      warp_best(bk, bt, wk, wt);
      if ((wt & 31u) == static_cast<unsigned>(lane)) taken |= 1ull << (wt >> 5);
      if (lane == c) mine = wt;
    }
  } else {
    qk = bisect<PL, false>(q, m, 0u, kQCap, static_cast<unsigned>(kk));
    unsigned above = 0;
#pragma unroll
    for (int s = 0; s < PL; ++s)
      if (q[s] < qk) ++above;
    above = __reduce_add_sync(kFull, above);
    walk_bucket<PL, false>(Kr, q, m, qk, above, static_cast<unsigned>(kk), kkb, jkb);
  }
  if (krow && !big_k) {   // ascending block id: lane c writes its id at its rank
    int rank = 0;
    for (int c = 0; c < kk; ++c) rank += __shfl_sync(kFull, mine, c) < mine ? 1 : 0;
    if (lane < kk) krow[rank] = static_cast<int32_t>(mine);
  }

  // floor membership bits (large floors)
  unsigned long long ink = taken;
  if (need_floor && big_k) {
#pragma unroll
    for (int s = 0; s < PL; ++s) {
      const int t = lane + 32 * s;
      if (t < Nb && (q[s] < qk || (q[s] == qk && at_or_before(Kr[t], t, kkb, jkb)))) ink |= 1ull << s;
    }
  }

  if (a.prefix_out && lane == 0) a.prefix_out[row] = n_p > kk ? n_p : kk;   // length of the kept ranked prefix

  // outputs: compacted kept list, Top-p mask, floor ids (large floors), logits
  const int nsl = (Nb + 31) / 32;   // slots holding blocks
  int32_t* irow = a.counts ? a.idx + row * Nb : nullptr;
  int pos = 0;
  if (irow) {
    const unsigned long long keep = inp | ink | ((i & 31) == lane ? 1ull << (i >> 5) : 0ull);
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll
    for (int s = 0; s < PL; ++s) {
      if (s >= nsl) break;
      const bool kp = (keep >> s) & 1ull;
      const unsigned bal = __ballot_sync(kFull, kp);
      if (kp) irow[pos + __popc(bal & lt)] = lane + 32 * s;
      pos += __popc(bal);
    }
  }
  if (a.topp_mask) {
    uint8_t* mrow = a.topp_mask + row * Nb;
#pragma unroll
    for (int s = 0; s < PL; ++s)
      if (lane + 32 * s < Nb) mrow[lane + 32 * s] = static_cast<uint8_t>((inp >> s) & 1ull);
  }
  if (big_k && krow) {
    int kpos = 0;
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll
    for (int s = 0; s < PL; ++s) {
      if (s >= nsl) break;
      const bool kp = (ink >> s) & 1ull;
      const unsigned bal = __ballot_sync(kFull, kp);
      if (kp) krow[kpos + __popc(bal & lt)] = lane + 32 * s;
      kpos += __popc(bal);
    }
  }
  if (a.logits_out) {
    double* lrow = a.logits_out + row * Nb;
#pragma unroll
    for (int s = 0; s < PL; ++s)
      if (lane + 32 * s < Nb) lrow[lane + 32 * s] = key_value(Kr[lane + 32 * s]);
  }
  if (irow && lane == 0) a.counts[row] = pos;
}

// R query blocks [i0, i0 + R) of bh: logits into shared memory, then one warp per row.
template <int D, int PL, int R, int KU>
__device__ __forceinline__ void select_item(const RouteArgs& a, long long bh, int i0, unsigned char* smem) {
  constexpr int LDQ = D + 4;             // padded rows (8-byte words)
  constexpr int LDL = 32 * PL + 2;
  constexpr int NT = 4 * PL;             // 8-column tiles covering 32 * PL columns
  double* Qs = reinterpret_cast<double*>(smem);
  double* Ls = Qs + R * LDQ;
  unsigned* Hs = reinterpret_cast<unsigned*>(Ls + R * LDL);   // per-warp histograms
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Nb = a.Nb;

  const double* qb = a.qbar + bh * Nb * D;
  const double* kb = a.kbar + bh * Nb * D;
  for (int e = tid; e < R * D; e += kRouteThreads) {
    const int r = e / D, c = e - r * D;
    Qs[r * LDQ + c] = i0 + r < Nb ? __ldcg(qb + static_cast<long long>(i0 + r) * D + c) : 0.0;
  }
  __syncthreads();

  // L = Qbar Kbar^T / sqrt(D): warp w takes column tiles w, w + 8, w + 16, ... NG at a
  // time for all MT row tiles, so every loaded fragment feeds MT (A: NG) products and
  // the warp runs MT * NG independent accumulation chains.  Fragment coordinates of
  // m8n8k4 (row.col): A[gid][kq], B[kq][gid], C[gid][2 tq + e], where the four k of
  // one product are taken as 8 c + 2 tq + h (h = 0 for the first product of a pair,
  // 1 for the second), so each thread loads its two k of a pair as one 16-byte word.
  // The product covers every k exactly once, in a different grouping (float64 sums).
  // Columns past Nb read block 0 and are overwritten by -inf below.
  constexpr int MT = R / 8;                      // 8-row tiles
  constexpr int NG = 4 / MT;                     // column tiles per group
  constexpr int NTW = NT / kRouteWarps;          // column tiles per warp
  static_assert(R % 8 == 0 && MT * NG == 4, "8 or 16 rows per item");
  const int gid = lane >> 2, tq = lane & 3;
  const int ntv = (Nb + 7) / 8;
  const double inv_rs = 1.0 / sqrt(static_cast<double>(D));
  const double* qa = Qs + gid * LDQ + 2 * tq;
#pragma unroll 1
  for (int j0 = 0; j0 < NTW; j0 += NG) {
    double acc[NG][MT][2];
    const double2* kp[NG];
#pragma unroll
    for (int u = 0; u < NG; ++u) {
      const int nt = warp + kRouteWarps * (j0 + u);
      const int j = nt * 8 + gid;
      const bool jv = j0 + u < NTW && nt < ntv && j < Nb;
      kp[u] = reinterpret_cast<const double2*>(kb + static_cast<long long>(jv ? j : 0) * D + 2 * tq);
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) acc[u][mt][0] = acc[u][mt][1] = 0.0;
    }
#pragma unroll KU
    for (int c = 0; c < D / 8; ++c) {
      double2 av[MT];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) av[mt] = *reinterpret_cast<const double2*>(qa + mt * 8 * LDQ + 8 * c);
#pragma unroll
      for (int u = 0; u < NG; ++u) {
        const double2 b = __ldcg(kp[u] + 4 * c);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                       : "+d"(acc[u][mt][0]), "+d"(acc[u][mt][1])
                       : "d"(av[mt].x), "d"(b.x));
          asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                       : "+d"(acc[u][mt][0]), "+d"(acc[u][mt][1])
                       : "d"(av[mt].y), "d"(b.y));
        }
      }
    }
#pragma unroll
    for (int u = 0; u < NG; ++u) {
      if (j0 + u >= NTW) break;
      const int nt = warp + kRouteWarps * (j0 + u);
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int cc = nt * 8 + 2 * tq + e;
          Ls[(mt * 8 + gid) * LDL + cc] = cc < Nb ? acc[u][mt][e] * inv_rs : -INFINITY;
        }
    }
  }
  __syncthreads();

  for (int r = warp; r < R; r += kRouteWarps)
    if (i0 + r < Nb) select_row<PL>(a, bh, i0 + r, Ls + r * LDL, Hs + warp * kHistBins);
}

template <int D, int PL, int R>
constexpr size_t select_smem_bytes() {
  return (static_cast<size_t>(R) * (D + 4) + static_cast<size_t>(R) * (32 * PL + 2)) * sizeof(double) +
         static_cast<size_t>(kRouteWarps) * kHistBins * sizeof(unsigned);
}

// grid = (ceil(Nb / R), heads): CTA (x, y) selects rows [x*R, x*R + R) of (b, h) = bh0 + y.
// MINB CTAs per SM; KU = unrolled k-steps of the logits loop for that register budget.
template <int D, int PL, int R, int MINB>
__global__ void __launch_bounds__(kRouteThreads, MINB) select_kernel(const RouteArgs a, long long bh0) {
  constexpr int KU = MINB >= 4 ? 4 : (MINB == 3 ? 4 : 8);
  extern __shared__ __align__(16) unsigned char sel_smem[];
  select_item<D, PL, R, KU>(a, bh0 + blockIdx.y, static_cast<int>(blockIdx.x) * R, sel_smem);
}

size_t align_up(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct Carve {
  double* qbar;
  double* kbar;
};

Carve carve(const Dims& D, void* ws) {
  const size_t pooled = align_up(static_cast<size_t>(D.rows()) * D.d * sizeof(double));
  unsigned char* w = static_cast<unsigned char*>(ws);
  return Carve{reinterpret_cast<double*>(w), reinterpret_cast<double*>(w + pooled)};
}

template <int D, int PL, int R, int MINB>
cudaError_t launch_select_variant(const RouteArgs& a, long long bh0, long long nbh, cudaStream_t s) {
  auto kern = select_kernel<D, PL, R, MINB>;
  constexpr size_t smem = select_smem_bytes<D, PL, R>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>((a.Nb + R - 1) / R), static_cast<unsigned>(nbh));
  kern<<<grid, kRouteThreads, smem, s>>>(a, bh0);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_select(const RouteArgs& a, long long bh0, long long nbh, cudaStream_t s) {
  if (a.Nb <= 256) return launch_select_variant<D, 8, 8, 4>(a, bh0, nbh, s);
  if (a.Nb <= 640) return launch_select_variant<D, 20, 16, 2>(a, bh0, nbh, s);
  if (a.Nb <= 1280) return launch_select_variant<D, 40, 16, 1>(a, bh0, nbh, s);
  return launch_select_variant<D, 64, 8, 1>(a, bh0, nbh, s);
}

}  // namespace

size_t route_workspace_bytes(const Dims& D) {
  const size_t pooled = static_cast<size_t>(D.rows()) * D.d * sizeof(double);
  return 2 * align_up(pooled);
}

namespace {
RouteArgs make_args(const double* qbar, const double* kbar, const Dims& D, double p, int kk, uint8_t* topp_mask,
                    int32_t* topk_idx, double* logits_out, int32_t* counts, int32_t* idx) {
  RouteArgs a;
  a.qbar = qbar;
  a.kbar = kbar;
  a.topp_mask = topp_mask;
  a.topk_idx = topk_idx;
  a.logits_out = logits_out;
  a.counts = counts;
  a.idx = idx;
  a.prefix_out = nullptr;
  a.kk_rows = nullptr;
  a.Nb = D.Nb;
  a.kk = kk;
  a.keep_all_p = p >= 1.0 ? 1 : 0;
  const double tp = ceil(p * 0x1p31);
  a.target = a.keep_all_p ? 0u : static_cast<unsigned>(tp < 1.0 ? 1.0 : tp);
  return a;
}

// Slack-aware augmentation, single-GPU reading (§3.3 SASA): the heads form num_ranks
// virtual ranks of H / num_ranks consecutive heads; W_r = kept block pairs of the rank
// (from the counts); rank r gets B_r = floor(alpha * (W* - W_r)) more pairs, W* the
// largest W_r, spread round-robin over its rows in item order; a row's floor becomes
// min(Nb, prefix + share), i.e. its ranked prefix grows by its share.
constexpr int kSasaThreads = 256;
constexpr int kSasaMaxRanks = 1024;

__global__ void __launch_bounds__(kSasaThreads) sasa_kernel(const int32_t* __restrict__ counts,
                                                            const int32_t* __restrict__ prefix, int B, int H, int Nb,
                                                            int num_ranks, double alpha, int32_t* __restrict__ kk_rows,
                                                            int32_t* __restrict__ extra) {
  __shared__ unsigned long long W[kSasaMaxRanks];
  __shared__ long long budget[kSasaMaxRanks];
  const int hpr = H / num_ranks;
  for (int r = threadIdx.x; r < num_ranks; r += kSasaThreads) W[r] = 0;
  __syncthreads();
  const long long n = static_cast<long long>(B) * H * Nb;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (long long bh = warp; bh < static_cast<long long>(B) * H; bh += kSasaThreads / 32) {   // W_h, a warp each
    unsigned long long w = 0;
    for (int i = lane; i < Nb; i += 32) w += static_cast<unsigned long long>(counts[bh * Nb + i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) w += __shfl_xor_sync(kFull, w, o);
    if (lane == 0) atomicAdd(&W[static_cast<int>(bh % H) / hpr], w);
  }
  __syncthreads();
  unsigned long long wmax = 0;
  for (int r = 0; r < num_ranks; ++r) wmax = W[r] > wmax ? W[r] : wmax;
  for (int r = threadIdx.x; r < num_ranks; r += kSasaThreads)
    budget[r] = static_cast<long long>(floor(alpha * static_cast<double>(wmax - W[r])));
  __syncthreads();
  const long long n_rows = static_cast<long long>(B) * hpr * Nb;   // rows per rank
  for (long long u = static_cast<long long>(blockIdx.x) * kSasaThreads + threadIdx.x; u < n;
       u += static_cast<long long>(gridDim.x) * kSasaThreads) {
    const int i = static_cast<int>(u % Nb);
    const int h = static_cast<int>((u / Nb) % H);
    const long long b = u / (static_cast<long long>(H) * Nb);
    const int r = h / hpr;
    const long long pos = (b * hpr + (h - r * hpr)) * Nb + i;        // rank of the row in item order
    const long long share = budget[r] / n_rows + (pos < budget[r] % n_rows ? 1 : 0);
    const long long len = prefix[u] + share;
    const int32_t v = static_cast<int32_t>(len < Nb ? len : Nb);
    kk_rows[u] = v;
    if (extra) extra[u] = v - prefix[u];
  }
}
}  // namespace

cudaError_t launch_select_pooled(const double* qbar, const double* kbar, const Dims& D, double p, int kk,
                                 uint8_t* topp_mask, int32_t* topk_idx, double* logits_out, int32_t* counts,
                                 int32_t* idx, cudaStream_t s, int* launches) {
  const RouteArgs a = make_args(qbar, kbar, D, p, kk, topp_mask, topk_idx, logits_out, counts, idx);
  cudaError_t e = D.d == 128 ? launch_select<128>(a, 0, D.BH(), s) : launch_select<64>(a, 0, D.BH(), s);
  ++*launches;
  return e;
}

cudaError_t launch_sasa(const double* qbar, const double* kbar, const Dims& D, double p, int kk, int num_ranks,
                        double alpha, int32_t* counts, int32_t* idx, int32_t* extra, void* ws, cudaStream_t s,
                        int* launches) {
  int32_t* prefix = static_cast<int32_t*>(ws);
  int32_t* kk_rows = prefix + ((D.rows() + 63) / 64) * 64;
  RouteArgs a = make_args(qbar, kbar, D, p, kk, nullptr, nullptr, nullptr, counts, idx);
  a.prefix_out = prefix;
  cudaError_t e = D.d == 128 ? launch_select<128>(a, 0, D.BH(), s) : launch_select<64>(a, 0, D.BH(), s);
  ++*launches;
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(std::min<long long>((D.rows() + kSasaThreads - 1) / kSasaThreads, 148));
  sasa_kernel<<<grid, kSasaThreads, 0, s>>>(counts, prefix, D.B, D.H, D.Nb, num_ranks, alpha, kk_rows, extra);
  ++*launches;
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  RouteArgs a2 = make_args(qbar, kbar, D, p, kk, nullptr, nullptr, nullptr, counts, idx);
  a2.kk_rows = kk_rows;
  e = D.d == 128 ? launch_select<128>(a2, 0, D.BH(), s) : launch_select<64>(a2, 0, D.BH(), s);
  ++*launches;
  return e;
}

size_t sasa_workspace_bytes(const Dims& D) { return 2 * static_cast<size_t>((D.rows() + 63) / 64) * 64 * sizeof(int32_t); }

cudaError_t launch_route(const void* qr, const void* kr, const Dims& D, double p, int kk, uint8_t* topp_mask,
                         int32_t* topk_idx, double* logits_out, int32_t* counts, int32_t* idx, void* ws,
                         cudaStream_t s, int* launches) {
  const Carve c = carve(D, ws);
  const RouteArgs a = make_args(c.qbar, c.kbar, D, p, kk, topp_mask, topk_idx, logits_out, counts, idx);
  const long long rows = D.rows();
  const dim3 pgrid(static_cast<unsigned>(2 * rows));
  if (D.d == 128)
    pool_kernel<128><<<pgrid, kPoolThreads, 0, s>>>(static_cast<const uint4*>(qr), static_cast<const uint4*>(kr),
                                                    c.qbar, c.kbar, 0, rows, D.S);
  else
    pool_kernel<64><<<pgrid, kPoolThreads, 0, s>>>(static_cast<const uint4*>(qr), static_cast<const uint4*>(kr),
                                                   c.qbar, c.kbar, 0, rows, D.S);
  ++*launches;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = D.d == 128 ? launch_select<128>(a, 0, D.BH(), s) : launch_select<64>(a, 0, D.BH(), s);
  ++*launches;
  return e;
}

}  // namespace fva
