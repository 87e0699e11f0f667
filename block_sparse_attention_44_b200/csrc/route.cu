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
// The heads are split into chunks: chunk c is pooled on the caller's stream while a
// second stream scores and selects chunk c - 1, so selection runs under the memory
// stream instead of after it.  The two streams meet through events only.
//
// Selection arithmetic (deterministic, exact integer sums):
//   - softmax weights e_j = exp(L_ij - max_j L_ij) in float64, then the mass
//     m_j = floor(e_j / z * 2^31) (z = sum_j e_j) as an unsigned integer;
//   - the Top-p boundary is the first position, in the ranking (logit descending,
//     block id ascending), where the running sum of m reaches ceil(p * 2^31): found
//     by a 14-step bisection over the bucket index q_j = floor((max L - L_ij) * 256)
//     (buckets 1/256 logit wide rank like the logits; warp sums by redux.sync), then
//     inside the boundary bucket by the exact float64 logits;
//   - the Top-k floor by repeated warp argmax over (logit, -block id).
// Every mass carries a relative error below 2e-7 and is truncated by less than 2^-31,
// so the running sum at any cut is within 1.2e-6 of the exact cumulative softmax
// mass: a kept set can differ from the exact one only where the cumulative mass at
// the cut lies within that distance of p.
#include <limits.h>
#include <math.h>

#include "fva_common.cuh"
#include "fva_internal.h"

namespace fva {
namespace {

constexpr int kRouteThreads = 256;
constexpr int kRouteWarps = kRouteThreads / 32;
constexpr int kPoolThreads = 256;
constexpr int kMaxChunks = 4;           // head chunks overlapped across the two streams
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

__device__ __forceinline__ double warp_max_f64(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(kFull, v, o));
  return v;
}
__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

// (L, t) ranks before (L2, t2): logit descending, block id ascending.
__device__ __forceinline__ bool ranks_before(double L, int t, double L2, int t2) {
  return L > L2 || (L == L2 && t < t2);
}

// Warp argmax of (L, t) in ranking order, carrying a payload word.
__device__ __forceinline__ void warp_argmax(double& L, int& t, unsigned& w) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double oL = __shfl_xor_sync(kFull, L, o);
    const int ot = __shfl_xor_sync(kFull, t, o);
    const unsigned ow = __shfl_xor_sync(kFull, w, o);
    if (ranks_before(oL, ot, L, t)) {
      L = oL;
      t = ot;
      w = ow;
    }
  }
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

// Walks bucket qs in ranking order from weight `acc` (the weight of every better
// bucket) until the running weight reaches T; returns that block's (logit, id).
template <int PL, bool BY_MASS>
__device__ __forceinline__ void walk_bucket(const double* Lr, const unsigned (&q)[PL], const unsigned (&m)[PL], unsigned qs,
                            unsigned acc, unsigned T, double& Lb, int& jb) {
  const int lane = threadIdx.x & 31;
  double Lp = INFINITY;
  int jp = -1;
  for (int guard = 0; guard < 32 * PL; ++guard) {
    double bL = -INFINITY;
    int bt = INT_MAX;
    unsigned bw = 0;
#pragma unroll
    for (int s = 0; s < PL; ++s) {
      if (q[s] != qs) continue;
      const int t = lane + 32 * s;
      const double L = Lr[t];
      if (ranks_before(Lp, jp, L, t) && ranks_before(L, t, bL, bt)) {
        bL = L;
        bt = t;
        bw = BY_MASS ? m[s] : 1u;
      }
    }
    warp_argmax(bL, bt, bw);
    if (bt == INT_MAX) break;   // bucket exhausted: cannot happen when the bucket reaches T
    acc += bw;
    if (acc >= T) {
      Lb = bL;
      jb = bt;
      return;
    }
    Lp = bL;
    jp = bt;
  }
  Lb = -INFINITY;   // keep everything
  jb = INT_MAX;
}

// Row i of (b, h) = bh; Lr = its logits in shared memory (32*PL entries, -inf past Nb).
template <int PL>
__device__ __forceinline__ void select_row(const RouteArgs& a, long long bh, int i, const double* Lr) {
  const int lane = threadIdx.x & 31;
  const int Nb = a.Nb;
  const long long row = bh * Nb + i;

  double mx = -INFINITY;
#pragma unroll
  for (int s = 0; s < PL; ++s) mx = fmax(mx, Lr[lane + 32 * s]);
  mx = warp_max_f64(mx);

  // weights, bucket indices; e^-45 < 2^-64: those blocks carry mass 0 and go to kQCap
  unsigned q[PL], m[PL];
  double z = 0.0;
#pragma unroll
  for (int s = 0; s < PL; ++s) {
    const int t = lane + 32 * s;
    const double d = Lr[t] - mx;
    const bool live = d > -45.0;
    const double e = live ? exp(d) : 0.0;
    z += e;
    m[s] = __float_as_uint(__double2float_rn(e));
    q[s] = live ? static_cast<unsigned>(-d * 256.0) : (t < Nb ? kQCap : kQPad);
  }
  z = warp_sum_f64(z);
  const float scale = __double2float_rn(0x1p31 / z);
  unsigned part = 0;
#pragma unroll
  for (int s = 0; s < PL; ++s) {
    m[s] = __float2uint_rz(__uint_as_float(m[s]) * scale);
    part += m[s];
  }
  const unsigned tot = __reduce_add_sync(kFull, part);

  // Top-p boundary (Lp_b, jp_b): the kept set is every block ranking at or before it
  const bool all_p = a.keep_all_p || tot < a.target;
  unsigned qp = 0;
  double Lpb = -INFINITY;
  int jpb = INT_MAX;
  if (!all_p) {
    qp = bisect<PL, true>(q, m, 0u, kQCap - 1u, a.target);
    unsigned above = 0;
#pragma unroll
    for (int s = 0; s < PL; ++s)
      if (q[s] < qp) above += m[s];
    above = __reduce_add_sync(kFull, above);
    walk_bucket<PL, true>(Lr, q, m, qp, above, a.target, Lpb, jpb);
  }

  // Top-k floor
  const int kk = a.kk;
  unsigned long long taken = 0;   // bit s: block lane + 32 s is in the floor (kk <= kTopkArgmaxMax)
  unsigned qk = 0;
  double Lkb = -INFINITY;
  int jkb = INT_MAX;
  int32_t* krow = a.topk_idx ? a.topk_idx + row * kk : nullptr;
  if (kk <= kTopkArgmaxMax) {
    int mine = INT_MAX;   // lane c holds the c-th chosen id
    for (int c = 0; c < kk; ++c) {
      double bL = -INFINITY;
      int bt = INT_MAX;
      unsigned bs = 0;
#pragma unroll
      for (int s = 0; s < PL; ++s) {
        const int t = lane + 32 * s;
        if (((taken >> s) & 1ull) || t >= Nb) continue;
        const double L = Lr[t];
        if (ranks_before(L, t, bL, bt)) {
          bL = L;
          bt = t;
          bs = static_cast<unsigned>(s);
        }
      }
      warp_argmax(bL, bt, bs);
      if ((bt & 31) == lane) taken |= 1ull << bs;
      if (lane == c) mine = bt;
    }
    if (krow) {   // ascending block id: lane c writes its id at its rank
      int rank = 0;
      for (int c = 0; c < kk; ++c) rank += __shfl_sync(kFull, mine, c) < mine ? 1 : 0;
      if (lane < kk) krow[rank] = mine;
    }
  } else {
    qk = bisect<PL, false>(q, m, 0u, kQCap, static_cast<unsigned>(kk));
    unsigned above = 0;
#pragma unroll
    for (int s = 0; s < PL; ++s)
      if (q[s] < qk) ++above;
    above = __reduce_add_sync(kFull, above);
    walk_bucket<PL, false>(Lr, q, m, qk, above, static_cast<unsigned>(kk), Lkb, jkb);
  }

  // outputs: Top-p mask, floor ids (large floors), logits, compacted kept list
  uint8_t* mrow = a.topp_mask ? a.topp_mask + row * Nb : nullptr;
  double* lrow = a.logits_out ? a.logits_out + row * Nb : nullptr;
  int32_t* irow = a.counts ? a.idx + row * Nb : nullptr;
  const bool big_k = kk > kTopkArgmaxMax;
  int kpos = 0, pos = 0;
#pragma unroll
  for (int s = 0; s < PL; ++s) {
    if (32 * s >= Nb) break;
    const int t = lane + 32 * s;
    const bool valid = t < Nb;
    const double L = Lr[t];
    const bool in_p = valid && (all_p || q[s] < qp || (q[s] == qp && !ranks_before(Lpb, jpb, L, t)));
    const bool in_k = big_k ? valid && (q[s] < qk || (q[s] == qk && !ranks_before(Lkb, jkb, L, t)))
                            : ((taken >> s) & 1ull) != 0;
    if (valid && mrow) mrow[t] = in_p ? 1 : 0;
    if (valid && lrow) lrow[t] = L;
    if (big_k) {
      const unsigned bal = __ballot_sync(kFull, in_k);
      if (in_k && krow) krow[kpos + __popc(bal & ((1u << lane) - 1u))] = t;
      kpos += __popc(bal);
    }
    if (irow) {
      const bool keep = in_p || in_k || t == i;
      const unsigned bal = __ballot_sync(kFull, valid && keep);
      if (valid && keep) irow[pos + __popc(bal & ((1u << lane) - 1u))] = t;
      pos += __popc(bal);
    }
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
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Nb = a.Nb;

  const double* qb = a.qbar + bh * Nb * D;
  const double* kb = a.kbar + bh * Nb * D;
  for (int e = tid; e < R * D; e += kRouteThreads) {
    const int r = e / D, c = e - r * D;
    Qs[r * LDQ + c] = i0 + r < Nb ? __ldcg(qb + static_cast<long long>(i0 + r) * D + c) : 0.0;
  }
  __syncthreads();

  // L = Qbar Kbar^T / sqrt(D): warp w takes column tiles w, w + 8, w + 16, ... four at
  // a time, so each A fragment feeds four independent accumulation chains.  Fragment
  // coordinates of m8n8k4 (row.col): A[gid][tq], B[tq][gid], C[gid][2 tq + e].
  static_assert(R == 8, "one 8-row MMA tile per item");
  constexpr int NTW = NT / kRouteWarps;          // column tiles per warp
  const int gid = lane >> 2, tq = lane & 3;
  const int ntv = (Nb + 7) / 8;
  const double rs = sqrt(static_cast<double>(D));
  const double* qa = Qs + gid * LDQ + tq;
#pragma unroll 1
  for (int j0 = 0; j0 < NTW; j0 += 4) {
    double acc[4][2];
    const double* kp[4];
    bool jv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int nt = warp + kRouteWarps * (j0 + u);
      const int j = nt * 8 + gid;
      jv[u] = j0 + u < NTW && nt < ntv && j < Nb;
      kp[u] = kb + static_cast<long long>(jv[u] ? j : 0) * D + tq;
      acc[u][0] = acc[u][1] = 0.0;
    }
#pragma unroll KU
    for (int k = 0; k < D; k += 4) {
      const double av = qa[k];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const double b = jv[u] ? __ldcg(kp[u] + k) : 0.0;
        asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                     : "+d"(acc[u][0]), "+d"(acc[u][1])
                     : "d"(av), "d"(b));
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (j0 + u >= NTW) break;
      const int nt = warp + kRouteWarps * (j0 + u);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int c = nt * 8 + 2 * tq + e;
        Ls[gid * LDL + c] = c < Nb ? acc[u][e] / rs : -INFINITY;
      }
    }
  }
  __syncthreads();

  for (int r = warp; r < R; r += kRouteWarps)
    if (i0 + r < Nb) select_row<PL>(a, bh, i0 + r, Ls + r * LDL);
}

template <int D, int PL, int R>
constexpr size_t select_smem_bytes() {
  return (static_cast<size_t>(R) * (D + 4) + static_cast<size_t>(R) * (32 * PL + 2)) * sizeof(double);
}

// grid = (ceil(Nb / R), heads): CTA (x, y) selects rows [x*R, x*R + R) of (b, h) = bh0 + y.
// MINB CTAs per SM; KU = unrolled k-steps of the logits loop for that register budget.
template <int D, int PL, int R, int MINB>
__global__ void __launch_bounds__(kRouteThreads, MINB) select_kernel(const RouteArgs a, long long bh0) {
  constexpr int KU = MINB >= 4 ? 2 : (MINB == 3 ? 4 : 8);
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

// The second stream and the fork/join events, per host thread and device (a thread
// never shares them, so concurrent callers on other threads cannot interleave).
struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t ev[kMaxChunks + 2] = {};
  bool ready = false;
};

cudaError_t side_stream(SideStream** out) {
  thread_local SideStream ctx[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  SideStream& c = ctx[dev];
  if (!c.ready) {
    int lo = 0, hi = 0;
    e = cudaDeviceGetStreamPriorityRange(&lo, &hi);
    if (e != cudaSuccess) return e;
    e = cudaStreamCreateWithPriority(&c.stream, cudaStreamNonBlocking, hi);   // selection first when both wait
    if (e != cudaSuccess) return e;
    for (auto& ev : c.ev) {
      e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming);
      if (e != cudaSuccess) return e;
    }
    c.ready = true;
  }
  *out = &c;
  return cudaSuccess;
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
  if (a.Nb <= 640) return launch_select_variant<D, 20, 8, 3>(a, bh0, nbh, s);
  if (a.Nb <= 1280) return launch_select_variant<D, 40, 8, 2>(a, bh0, nbh, s);
  return launch_select_variant<D, 64, 8, 1>(a, bh0, nbh, s);
}

}  // namespace

size_t route_workspace_bytes(const Dims& D) {
  const size_t pooled = static_cast<size_t>(D.rows()) * D.d * sizeof(double);
  return 2 * align_up(pooled);
}

cudaError_t launch_route(const void* qr, const void* kr, const Dims& D, double p, int kk, uint8_t* topp_mask,
                         int32_t* topk_idx, double* logits_out, int32_t* counts, int32_t* idx, void* ws,
                         cudaStream_t s, int* launches) {
  const Carve c = carve(D, ws);
  RouteArgs a;
  a.qbar = c.qbar;
  a.kbar = c.kbar;
  a.topp_mask = topp_mask;
  a.topk_idx = topk_idx;
  a.logits_out = logits_out;
  a.counts = counts;
  a.idx = idx;
  a.Nb = D.Nb;
  a.kk = kk;
  a.keep_all_p = p >= 1.0 ? 1 : 0;
  const double tp = ceil(p * 0x1p31);
  a.target = a.keep_all_p ? 0u : static_cast<unsigned>(tp < 1.0 ? 1.0 : tp);

  SideStream* side = nullptr;
  cudaError_t e = side_stream(&side);
  if (e != cudaSuccess) return e;
  const long long BH = D.BH();
  const int nchunks = static_cast<int>(BH < kMaxChunks ? BH : kMaxChunks);
  // fork: the side stream starts after everything already queued on s
  if ((e = cudaEventRecord(side->ev[0], s)) != cudaSuccess) return e;
  if ((e = cudaStreamWaitEvent(side->stream, side->ev[0], 0)) != cudaSuccess) return e;
  for (int ch = 0; ch < nchunks; ++ch) {
    const long long bh0 = BH * ch / nchunks, bh1 = BH * (ch + 1) / nchunks;
    const long long row0 = bh0 * D.Nb, nrows = (bh1 - bh0) * D.Nb;
    const dim3 pgrid(static_cast<unsigned>(2 * nrows));
    if (D.d == 128)
      pool_kernel<128><<<pgrid, kPoolThreads, 0, s>>>(static_cast<const uint4*>(qr), static_cast<const uint4*>(kr),
                                                      c.qbar, c.kbar, row0, nrows, D.S);
    else
      pool_kernel<64><<<pgrid, kPoolThreads, 0, s>>>(static_cast<const uint4*>(qr), static_cast<const uint4*>(kr),
                                                     c.qbar, c.kbar, row0, nrows, D.S);
    ++*launches;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = cudaEventRecord(side->ev[ch + 1], s)) != cudaSuccess) return e;
    if ((e = cudaStreamWaitEvent(side->stream, side->ev[ch + 1], 0)) != cudaSuccess) return e;
    e = D.d == 128 ? launch_select<128>(a, bh0, bh1 - bh0, side->stream)
                   : launch_select<64>(a, bh0, bh1 - bh0, side->stream);
    ++*launches;
    if (e != cudaSuccess) return e;
  }
  // join: later work on s sees every selection
  if ((e = cudaEventRecord(side->ev[kMaxChunks + 1], side->stream)) != cudaSuccess) return e;
  return cudaStreamWaitEvent(s, side->ev[kMaxChunks + 1], 0);
}

}  // namespace fva
