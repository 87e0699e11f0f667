// Routing frontend: pooled Q/K block scores, Top-p CDF cut, Top-k floor
// ("FVAttn: Adaptive Sparse Attention with Runtime Load Balancing for Video
// Generation", §2 background on dynamic block-sparse routing and §3.1 overview).
//
// Three kernels, all float64 so the kept sets agree with an exact computation
// except at genuine ties:
//   pool_kernel    — one CTA per (b, h, block) of Q and of K: mean of S bf16 rows.
//                    HBM-bound, reads every Q/K byte once (S*d*2 bytes per CTA).
//   logits_kernel  — 64x64-tiled float64 GEMM per (b, h) on the FP64 tensor path:
//                    L = Qbar Kbar^T / sqrt(d).
//   select_kernel  — one warp per (b, h, i) row: softmax in float64, masses in 2^-62
//                    fixed point; the row's Top-p boundary by a 16-step bisection
//                    over a 1/256-logit bucket index, resolved inside the boundary
//                    bucket by the exact 64-bit logit key (no sort; integer warp
//                    sums keep it exact and deterministic); the Top-k floor by
//                    repeated warp argmax.
#include <math.h>

#include "fva_common.cuh"
#include "fva_internal.h"

namespace fva {
namespace {

// ------------------------------------------------------------------ pooling -------
constexpr int kPoolThreads = 256;

__device__ __forceinline__ void bf16x8_to_f64_add(const uint4& v, double (&acc)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    acc[2 * q] += static_cast<double>(__uint_as_float(w[q] << 16));
    acc[2 * q + 1] += static_cast<double>(__uint_as_float(w[q] & 0xFFFF0000u));
  }
}

// grid.x = 2 * rows: blocks of Q first, then blocks of K.  Means are written to
// qbar[row] and kbar[row] ([B*H*Nb, D] float64).
template <int D>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(const uint4* __restrict__ qr, const uint4* __restrict__ kr,
                                                            double* __restrict__ qbar, double* __restrict__ kbar,
                                                            long long rows, int S) {
  constexpr int CPR = D / 8;                 // 16-byte chunks per row
  constexpr int RG = kPoolThreads / CPR;     // row groups
  __shared__ double part[RG][D];
  const bool is_k = blockIdx.x >= rows;
  const long long blk = is_k ? blockIdx.x - rows : blockIdx.x;   // (b*H + h)*Nb + i
  const int col = threadIdx.x % CPR;
  const int rg = threadIdx.x / CPR;
  double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const uint4* p = (is_k ? kr : qr) + blk * S * CPR;                // rows of a block are contiguous
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

// ------------------------------------------------------------------ logits --------
constexpr int kLT = 64;       // output tile (rows and columns) per CTA
constexpr int kLK = 32;       // reduction chunk staged in shared memory
constexpr int kLogitThreads = 128;

// L[bh, i, j] = sum_c Qbar[bh, i, c] * Kbar[bh, j, c] / sqrt(D)   (float64)
// FP64 tensor-core products (mma.sync m8n8k4 f64, exact float64 fused multiply-add
// per step): each of the four warps owns a 32 x 32 quarter of the 64 x 64 tile as
// 4 x 4 fragments of 8 x 8; A = Qbar rows, B = Kbar rows (i.e. Kbar^T column-major).
template <int D>
__global__ void __launch_bounds__(kLogitThreads) logits_kernel(const double* __restrict__ qbar,
                                                               const double* __restrict__ kbar,
                                                               double* __restrict__ L, double* __restrict__ L2,
                                                               int Nb) {
  constexpr int LD = kLK + 1;                      // padded row stride (doubles)
  __shared__ double Qs[kLT][LD];
  __shared__ double Ks[kLT][LD];
  const long long bh = blockIdx.z;
  const int i0 = blockIdx.y * kLT;
  const int j0 = blockIdx.x * kLT;
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  const int gid = lane >> 2, tid = lane & 3;       // mma fragment coordinates
  const int wi = (warp >> 1) * 32, wj = (warp & 1) * 32;
  const double* qb = qbar + bh * Nb * D;
  const double* kb = kbar + bh * Nb * D;
  double acc[4][4][2];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[a][c][0] = acc[a][c][1] = 0.0;
  for (int c0 = 0; c0 < D; c0 += kLK) {
    for (int e = threadIdx.x; e < kLT * kLK; e += kLogitThreads) {
      const int r = e / kLK, c = e - r * kLK;
      const int gi = i0 + r, gj = j0 + r;
      Qs[r][c] = gi < Nb ? qb[static_cast<long long>(gi) * D + c0 + c] : 0.0;
      Ks[r][c] = gj < Nb ? kb[static_cast<long long>(gj) * D + c0 + c] : 0.0;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kLK; k += 4) {
      double a[4], bb[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        a[t] = Qs[wi + 8 * t + gid][k + tid];
        bb[t] = Ks[wj + 8 * t + gid][k + tid];
      }
#pragma unroll
      for (int ti = 0; ti < 4; ++ti)
#pragma unroll
        for (int tj = 0; tj < 4; ++tj)
          asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                       : "+d"(acc[ti][tj][0]), "+d"(acc[ti][tj][1])
                       : "d"(a[ti]), "d"(bb[tj]));
    }
    __syncthreads();
  }
  const double rs = sqrt(static_cast<double>(D));
#pragma unroll
  for (int ti = 0; ti < 4; ++ti) {
    const int i = i0 + wi + 8 * ti + gid;
    if (i >= Nb) continue;
#pragma unroll
    for (int tj = 0; tj < 4; ++tj)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int j = j0 + wj + 8 * tj + 2 * tid + e;
        if (j >= Nb) continue;
        const double val = acc[ti][tj][e] / rs;
        const long long o = (bh * Nb + i) * static_cast<long long>(Nb) + j;
        L[o] = val;
        if (L2) L2[o] = val;
      }
  }
}

// ------------------------------------------------------------------ selection -----
constexpr int kSelWarps = 4;
constexpr int kTopkArgmaxMax = 16;   // floors up to this size use repeated warp argmax
typedef unsigned long long u64;

// Order-preserving map of a float64 logit to an unsigned key (larger logit -> larger key).
__device__ __forceinline__ u64 order_key(double L) {
  if (L == 0.0) L = 0.0;  // -0 and +0 rank equal
  const u64 u = static_cast<u64>(__double_as_longlong(L));
  return (u & 0x8000000000000000ull) ? ~u : (u | 0x8000000000000000ull);
}

__device__ __forceinline__ u64 warp_sum_u64(u64 v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Boundary of the ranking (key descending, block id ascending) where the running
// weight first reaches `target` (weight = fixed-point mass, or 1 per block when
// !by_mass).  Requires 0 < target <= total weight.
//   1. Bisection over q = min(65535, floor((Lmax - L) * 256)), which ranks like the
//      logit in steps of 1/256: the boundary bucket q* is the smallest q whose
//      bucket-inclusive weight reaches the target (16 integer-sum steps).
//   2. Inside bucket q* (blocks within 1/256 of each other) the exact order is taken
//      from the 64-bit keys: repeated warp argmax until the weight reaches the target.
// All sums are warp reductions of integers: exact and deterministic.  Outputs the
// boundary's key and block id, and its 1-based rank.
__device__ void warp_select(const u64* key, const u64* mass, const unsigned* qk, int Nb, u64 target, bool by_mass,
                            u64& bkey, int& bj, int& rank) {
  const int lane = threadIdx.x & 31;
  unsigned lo = 0, hi = 65535;
  while (lo < hi) {
    const unsigned mid = (lo + hi) >> 1;
    u64 w = 0;
    for (int t = lane; t < Nb; t += 32)
      if (qk[t] <= mid) w += by_mass ? mass[t] : 1ull;
    w = warp_sum_u64(w);
    if (w >= target)
      hi = mid;
    else
      lo = mid + 1;
  }
  const unsigned qs = lo;
  u64 above_w = 0;
  unsigned above_n = 0;
  for (int t = lane; t < Nb; t += 32)
    if (qk[t] < qs) {
      above_w += by_mass ? mass[t] : 1ull;
      ++above_n;
    }
  above_w = warp_sum_u64(above_w);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) above_n += __shfl_xor_sync(0xffffffffu, above_n, o);
  // walk bucket qs in exact order: key descending, block id ascending
  u64 prev_key = ~0ull;
  int prev_j = -1;
  for (int guard = 0; guard < Nb; ++guard) {
    u64 best = 0;
    int bjx = 0x7fffffff;
    for (int t = lane; t < Nb; t += 32) {
      if (qk[t] != qs) continue;
      const u64 kv = key[t];
      // strictly after (prev_key, prev_j) in the ranking
      const bool after = kv < prev_key || (kv == prev_key && t > prev_j);
      if (after && (kv > best || (kv == best && t < bjx))) {
        best = kv;
        bjx = t;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const u64 ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oj = __shfl_xor_sync(0xffffffffu, bjx, o);
      if (ob > best || (ob == best && oj < bjx)) {
        best = ob;
        bjx = oj;
      }
    }
    if (bjx == 0x7fffffff) break;               // bucket exhausted (cannot happen)
    above_w += by_mass ? mass[bjx] : 1ull;
    ++above_n;
    prev_key = best;
    prev_j = bjx;
    if (above_w >= target) {
      bkey = best;
      bj = bjx;
      rank = static_cast<int>(above_n);
      return;
    }
  }
  // unreachable when 0 < target <= total: keep everything
  bkey = 0;
  bj = Nb;
  rank = Nb;
}

// Per-warp shared memory of select_kernel: keys and masses (8 bytes) and bucket
// indices (4 bytes) per block, rounded up so every warp's 8-byte arrays stay aligned.
__host__ __device__ constexpr size_t sel_bytes_per_warp(int Nb) {
  return ((2 * sizeof(u64) + sizeof(unsigned)) * static_cast<size_t>(Nb) + 15) & ~static_cast<size_t>(15);
}

__global__ void __launch_bounds__(kSelWarps * 32) select_kernel(const double* __restrict__ L, long long rows, int Nb,
                                                                double p, int kk, uint8_t* __restrict__ topp_mask,
                                                                int32_t* __restrict__ topk_idx) {
  extern __shared__ __align__(16) unsigned char sel_smem[];
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * kSelWarps + warp;
  if (row >= rows) return;
  const size_t per_warp = sel_bytes_per_warp(Nb);
  u64* key = reinterpret_cast<u64*>(sel_smem + per_warp * warp);
  u64* mass = key + Nb;
  unsigned* qk = reinterpret_cast<unsigned*>(mass + Nb);
  const double* Lr = L + row * Nb;

  double mx = -INFINITY;
  for (int t = lane; t < Nb; t += 32) mx = fmax(mx, Lr[t]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  // blocks more than 45 below the row max carry a probability below e^-45 < 2^-64,
  // which is exactly zero in the 2^-62 fixed point: their exponential is skipped
  double z = 0.0;
  for (int t = lane; t < Nb; t += 32) {
    const double l = Lr[t];
    key[t] = order_key(l);
    const double d = l - mx;
    const double e = d > -45.0 ? exp(d) : 0.0;
    mass[t] = static_cast<u64>(__double_as_longlong(e));  // raw bits for now
    const double qd = -d * 256.0;
    qk[t] = qd < 65535.0 ? static_cast<unsigned>(qd) : 65535u;
    z += e;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  const double to_fixed = 0x1p62 / z;
  u64 tot = 0;
  for (int t = lane; t < Nb; t += 32) {
    const double e = __longlong_as_double(static_cast<long long>(mass[t]));
    const u64 m = static_cast<u64>(e * to_fixed);
    mass[t] = m;
    tot += m;
  }
  tot = warp_sum_u64(tot);
  __syncwarp();

  // Top-p boundary
  bool keep_all = p >= 1.0;
  u64 bkey_p = 0;
  int bj_p = Nb, n_p = Nb;
  if (!keep_all) {
    u64 target = static_cast<u64>(p * 0x1p62);
    if (target == 0) target = 1;
    if (tot < target) {
      keep_all = true;
    } else {
      warp_select(key, mass, qk, Nb, target, true, bkey_p, bj_p, n_p);
    }
  }

  uint8_t* mrow = topp_mask + row * Nb;
  for (int t = lane; t < Nb; t += 32) {
    const u64 kv = key[t];
    const bool in = keep_all || kv > bkey_p || (kv == bkey_p && t <= bj_p);
    mrow[t] = in ? 1 : 0;
  }

  // Top-k floor: the kk highest-ranked blocks (key descending, block id ascending),
  // by repeated warp argmax for a small floor, by radix select otherwise
  int32_t* krow = topk_idx + row * kk;
  if (kk <= kTopkArgmaxMax) {
    unsigned taken = 0, taken_hi = 0;   // bit s: element lane + 32*s already chosen (s < 64 as Nb <= 2048)
    int chosen[kTopkArgmaxMax];
    for (int q = 0; q < kk; ++q) {
      u64 best = 0;
      int bjx = 0x7fffffff;
      for (int t = lane, sidx = 0; t < Nb; t += 32, ++sidx) {
        const bool tk = sidx < 32 ? ((taken >> sidx) & 1u) : ((taken_hi >> (sidx - 32)) & 1u);
        const u64 kv = key[t];
        if (!tk && (kv > best || (kv == best && t < bjx))) {
          best = kv;
          bjx = t;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const u64 ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int oj = __shfl_xor_sync(0xffffffffu, bjx, o);
        if (ob > best || (ob == best && oj < bjx)) {
          best = ob;
          bjx = oj;
        }
      }
      chosen[q] = bjx;
      if ((bjx & 31) == lane) {
        const int sidx = bjx >> 5;
        if (sidx < 32)
          taken |= 1u << sidx;
        else
          taken_hi |= 1u << (sidx - 32);
      }
    }
    // write in ascending block id (chosen[] is identical in every lane)
    if (lane == 0) {
      for (int a = 1; a < kk; ++a) {
        const int v = chosen[a];
        int b2 = a - 1;
        while (b2 >= 0 && chosen[b2] > v) {
          chosen[b2 + 1] = chosen[b2];
          --b2;
        }
        chosen[b2 + 1] = v;
      }
      for (int a = 0; a < kk; ++a) krow[a] = chosen[a];
    }
  } else {
    u64 bkey_k;
    int bj_k, n_k;
    warp_select(key, mass, qk, Nb, static_cast<u64>(kk), false, bkey_k, bj_k, n_k);
    int pos = 0;
    for (int base = 0; base < Nb; base += 32) {
      const int t = base + lane;
      bool in = false;
      if (t < Nb) {
        const u64 kv = key[t];
        in = kv > bkey_k || (kv == bkey_k && t <= bj_k);
      }
      const unsigned bal = __ballot_sync(0xffffffffu, in);
      if (in) krow[pos + __popc(bal & ((1u << lane) - 1u))] = t;
      pos += __popc(bal);
    }
  }
}

size_t align_up(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

}  // namespace

size_t route_workspace_bytes(const Dims& D) {
  const size_t pooled = static_cast<size_t>(D.rows()) * D.d * sizeof(double);
  const size_t logits = static_cast<size_t>(D.rows()) * D.Nb * sizeof(double);
  return 2 * align_up(pooled) + align_up(logits);
}

cudaError_t launch_route(const void* qr, const void* kr, const Dims& D, double p, int kk, uint8_t* topp_mask,
                         int32_t* topk_idx, double* logits_out, void* ws, cudaStream_t s, int* launches) {
  const size_t pooled = align_up(static_cast<size_t>(D.rows()) * D.d * sizeof(double));
  unsigned char* w = static_cast<unsigned char*>(ws);
  double* qbar = reinterpret_cast<double*>(w);
  double* kbar = reinterpret_cast<double*>(w + pooled);
  double* L = reinterpret_cast<double*>(w + 2 * pooled);
  const dim3 pgrid(static_cast<unsigned>(2 * D.rows()));
  if (D.d == 128)
    pool_kernel<128><<<pgrid, kPoolThreads, 0, s>>>(static_cast<const uint4*>(qr), static_cast<const uint4*>(kr), qbar,
                                                    kbar, D.rows(), D.S);
  else
    pool_kernel<64><<<pgrid, kPoolThreads, 0, s>>>(static_cast<const uint4*>(qr), static_cast<const uint4*>(kr), qbar,
                                                   kbar, D.rows(), D.S);
  ++*launches;
  const int nt = (D.Nb + kLT - 1) / kLT;
  const dim3 lgrid(nt, nt, static_cast<unsigned>(D.BH()));
  if (D.d == 128)
    logits_kernel<128><<<lgrid, kLogitThreads, 0, s>>>(qbar, kbar, L, logits_out, D.Nb);
  else
    logits_kernel<64><<<lgrid, kLogitThreads, 0, s>>>(qbar, kbar, L, logits_out, D.Nb);
  ++*launches;
  const size_t smem = kSelWarps * sel_bytes_per_warp(D.Nb);
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const unsigned sgrid = static_cast<unsigned>((D.rows() + kSelWarps - 1) / kSelWarps);
  select_kernel<<<sgrid, kSelWarps * 32, smem, s>>>(L, D.rows(), D.Nb, p, kk, topp_mask, topk_idx);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace fva
