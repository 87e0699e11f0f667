// Routing frontend: pooled Q/K block scores, Top-p CDF cut, Top-k floor
// ("FVAttn: Adaptive Sparse Attention with Runtime Load Balancing for Video
// Generation", §2 background on dynamic block-sparse routing and §3.1 overview).
//
// Three kernels, all float64 so the kept sets agree with an exact computation
// except at genuine ties:
//   pool_kernel    — one CTA per (b, h, block): mean of S bf16 rows.  HBM-bound,
//                    reads every Q/K byte once (S*d*2 bytes per CTA).
//   logits_kernel  — 64x64 register-tiled float64 GEMM per (b, h): L = Qbar Kbar^T / sqrt(d).
//   select_kernel  — one warp per (b, h, i) row: softmax in float64, masses in 2^-62
//                    fixed point, then an MSB-first radix select over the 64-bit
//                    order-preserving logit key finds the row's Top-p boundary and
//                    its Top-k boundary without sorting; integer atomics keep it
//                    deterministic.
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

template <int D>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(const uint4* __restrict__ xr, double* __restrict__ out,
                                                            int S) {
  constexpr int CPR = D / 8;                 // 16-byte chunks per row
  constexpr int RG = kPoolThreads / CPR;     // row groups
  __shared__ double part[RG][D];
  const long long blk = blockIdx.x;          // (b*H + h)*Nb + i ; rows of a block are contiguous
  const int col = threadIdx.x % CPR;
  const int rg = threadIdx.x / CPR;
  double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const uint4* p = xr + blk * S * CPR;
#pragma unroll 4
  for (int r = rg; r < S; r += RG) bf16x8_to_f64_add(__ldg(p + r * CPR + col), acc);
#pragma unroll
  for (int e = 0; e < 8; ++e) part[rg][col * 8 + e] = acc[e];
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += kPoolThreads) {
    double s = 0.0;
#pragma unroll 8
    for (int g2 = 0; g2 < RG; ++g2) s += part[g2][c];
    out[blk * D + c] = s / static_cast<double>(S);
  }
}

// ------------------------------------------------------------------ logits --------
constexpr int kLT = 64;       // output tile (rows and columns)
constexpr int kLK = 32;       // reduction chunk
constexpr int kLogitThreads = 256;

// L[bh, i, j] = sum_c Qbar[bh, i, c] * Kbar[bh, j, c] / sqrt(D)   (float64)
template <int D>
__global__ void __launch_bounds__(kLogitThreads) logits_kernel(const double* __restrict__ qbar,
                                                               const double* __restrict__ kbar,
                                                               double* __restrict__ L, double* __restrict__ L2,
                                                               int Nb) {
  __shared__ __align__(16) double Qs[kLK][kLT + 2];
  __shared__ __align__(16) double Ks[kLK][kLT + 2];
  const long long bh = blockIdx.z;
  const int i0 = blockIdx.y * kLT;
  const int j0 = blockIdx.x * kLT;
  const int tx = threadIdx.x % 16;
  const int ty = threadIdx.x / 16;
  const double* qb = qbar + bh * Nb * D;
  const double* kb = kbar + bh * Nb * D;
  double acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[a][c] = 0.0;

  for (int c0 = 0; c0 < D; c0 += kLK) {
    // stage a 64 x 32 slice of Qbar and Kbar, transposed to [c][row]
    for (int e = threadIdx.x; e < kLT * kLK; e += kLogitThreads) {
      const int r = e / kLK;
      const int c = e - r * kLK;
      const int gi = i0 + r;
      const int gj = j0 + r;
      Qs[c][r] = gi < Nb ? qb[static_cast<long long>(gi) * D + c0 + c] : 0.0;
      Ks[c][r] = gj < Nb ? kb[static_cast<long long>(gj) * D + c0 + c] : 0.0;
    }
    __syncthreads();
#pragma unroll 8
    for (int c = 0; c < kLK; ++c) {
      double a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[u] = Qs[c][ty * 4 + u];
        b[u] = Ks[c][tx * 4 + u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fma(a[u], b[v], acc[u][v]);
    }
    __syncthreads();
  }
  const double rs = sqrt(static_cast<double>(D));
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = i0 + ty * 4 + u;
    if (i >= Nb) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int j = j0 + tx * 4 + v;
      if (j >= Nb) continue;
      const double val = acc[u][v] / rs;
      const long long o = (bh * Nb + i) * static_cast<long long>(Nb) + j;
      L[o] = val;
      if (L2) L2[o] = val;
    }
  }
}

// ------------------------------------------------------------------ selection -----
constexpr int kSelWarps = 4;
typedef unsigned long long u64;

struct WarpHist {
  u64 m[256];
  unsigned int c[256];
};

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
// !by_mass).  Requires 0 < target <= total weight.  Outputs the boundary's key and
// block id, and its 1-based rank.
__device__ void warp_select(const u64* key, const u64* mass, int Nb, u64 target, bool by_mass, WarpHist* h,
                            u64& bkey, int& bj, int& rank) {
  const int lane = threadIdx.x & 31;
  u64 prefix = 0, pmask = 0, above_w = 0;
  int above_n = 0;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) {
      h->m[b] = 0;
      h->c[b] = 0;
    }
    __syncwarp();
    for (int t = lane; t < Nb; t += 32) {
      const u64 kv = key[t];
      if ((kv & pmask) == prefix) {
        const int dg = static_cast<int>((kv >> shift) & 255u);
        if (by_mass) atomicAdd(&h->m[dg], mass[t]);
        atomicAdd(&h->c[dg], 1u);
      }
    }
    __syncwarp();
    // lane l owns bins 255-8l ... 248-8l, i.e. the ranking order
    u64 w[8];
    unsigned cn[8];
    u64 wsum = 0;
    unsigned csum = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int bin = 255 - 8 * lane - q;
      cn[q] = h->c[bin];
      w[q] = by_mass ? h->m[bin] : static_cast<u64>(cn[q]);
      wsum += w[q];
      csum += cn[q];
    }
    u64 incl = wsum;
    unsigned cincl = csum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const u64 y = __shfl_up_sync(0xffffffffu, incl, o);
      const unsigned cy = __shfl_up_sync(0xffffffffu, cincl, o);
      if (lane >= o) {
        incl += y;
        cincl += cy;
      }
    }
    const u64 excl = incl - wsum;
    const unsigned cexcl = cincl - csum;
    const u64 need = target - above_w;
    const unsigned own = __ballot_sync(0xffffffffu, excl < need && need <= incl);
    const int owner = __ffs(own) - 1;
    int dstar = 0, nstar = 0;
    u64 add_w = 0;
    unsigned add_n = 0;
    if (lane == owner) {
      u64 run = excl;
      unsigned crun = cexcl;
      bool found = false;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (!found && run < need && need <= run + w[q]) {
          found = true;
          dstar = 255 - 8 * lane - q;
          nstar = static_cast<int>(cn[q]);
          add_w = run;
          add_n = crun;
        }
        run += w[q];
        crun += cn[q];
      }
    }
    dstar = __shfl_sync(0xffffffffu, dstar, owner);
    nstar = __shfl_sync(0xffffffffu, nstar, owner);
    add_w = __shfl_sync(0xffffffffu, add_w, owner);
    add_n = __shfl_sync(0xffffffffu, add_n, owner);
    prefix |= static_cast<u64>(dstar) << shift;
    pmask |= static_cast<u64>(255u) << shift;
    above_w += add_w;
    above_n += static_cast<int>(add_n);
    if (nstar == 1) {
      int who = 0x7fffffff;
      for (int t = lane; t < Nb; t += 32)
        if ((key[t] & pmask) == prefix) who = t;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) who = min(who, __shfl_xor_sync(0xffffffffu, who, o));
      bkey = key[who];
      bj = who;
      rank = above_n + 1;
      __syncwarp();
      return;
    }
    __syncwarp();
  }
  // Several blocks share the exact same logit: they rank by block id ascending.
  for (int base = 0; base < Nb; base += 32) {
    const int t = base + lane;
    const bool mem = t < Nb && key[t] == prefix;
    const unsigned bal = __ballot_sync(0xffffffffu, mem);
    const u64 wt = mem ? (by_mass ? mass[t] : 1ull) : 0ull;
    // members of one equal-key group have equal weight
    const u64 w_each = __shfl_sync(0xffffffffu, wt, bal ? __ffs(bal) - 1 : 0);
    const int cnt = __popc(bal);
    if (cnt && above_w + w_each * cnt >= target) {
      const u64 r = w_each ? (target - above_w + w_each - 1) / w_each : 1;  // 1-based member index
      unsigned m = bal;
      for (u64 q = 1; q < r; ++q) m &= m - 1;
      const int ln = __ffs(m) - 1;
      bkey = prefix;
      bj = base + ln;
      rank = above_n + static_cast<int>(r);
      return;
    }
    above_w += w_each * cnt;
    above_n += cnt;
  }
  // unreachable when 0 < target <= total: keep everything
  bkey = 0;
  bj = Nb;
  rank = Nb;
}

__global__ void __launch_bounds__(kSelWarps * 32) select_kernel(const double* __restrict__ L, long long rows, int Nb,
                                                                double p, int kk, uint8_t* __restrict__ topp_mask,
                                                                int32_t* __restrict__ topk_idx) {
  extern __shared__ __align__(16) unsigned char sel_smem[];
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * kSelWarps + warp;
  if (row >= rows) return;
  const size_t per_warp = sizeof(WarpHist) + 2 * sizeof(u64) * static_cast<size_t>(Nb);
  unsigned char* mine = sel_smem + per_warp * warp;
  WarpHist* h = reinterpret_cast<WarpHist*>(mine);
  u64* key = reinterpret_cast<u64*>(mine + sizeof(WarpHist));
  u64* mass = key + Nb;
  const double* Lr = L + row * Nb;

  double mx = -INFINITY;
  for (int t = lane; t < Nb; t += 32) mx = fmax(mx, Lr[t]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  double z = 0.0;
  for (int t = lane; t < Nb; t += 32) {
    const double l = Lr[t];
    key[t] = order_key(l);
    const double e = exp(l - mx);
    mass[t] = static_cast<u64>(__double_as_longlong(e));  // raw bits for now
    z += e;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  u64 tot = 0;
  for (int t = lane; t < Nb; t += 32) {
    const double e = __longlong_as_double(static_cast<long long>(mass[t]));
    const u64 m = static_cast<u64>((e / z) * 0x1p62);
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
      warp_select(key, mass, Nb, target, true, h, bkey_p, bj_p, n_p);
    }
  }
  // Top-k floor boundary
  u64 bkey_k;
  int bj_k, n_k;
  warp_select(key, mass, Nb, static_cast<u64>(kk), false, h, bkey_k, bj_k, n_k);

  uint8_t* mrow = topp_mask + row * Nb;
  for (int t = lane; t < Nb; t += 32) {
    const u64 kv = key[t];
    const bool in = keep_all || kv > bkey_p || (kv == bkey_p && t <= bj_p);
    mrow[t] = in ? 1 : 0;
  }
  int32_t* krow = topk_idx + row * kk;
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
  const dim3 pgrid(static_cast<unsigned>(D.rows()));
  if (D.d == 128) {
    pool_kernel<128><<<pgrid, kPoolThreads, 0, s>>>(static_cast<const uint4*>(qr), qbar, D.S);
    pool_kernel<128><<<pgrid, kPoolThreads, 0, s>>>(static_cast<const uint4*>(kr), kbar, D.S);
  } else {
    pool_kernel<64><<<pgrid, kPoolThreads, 0, s>>>(static_cast<const uint4*>(qr), qbar, D.S);
    pool_kernel<64><<<pgrid, kPoolThreads, 0, s>>>(static_cast<const uint4*>(kr), kbar, D.S);
  }
  *launches += 2;
  const int nt = (D.Nb + kLT - 1) / kLT;
  const dim3 lgrid(nt, nt, static_cast<unsigned>(D.BH()));
  if (D.d == 128)
    logits_kernel<128><<<lgrid, kLogitThreads, 0, s>>>(qbar, kbar, L, logits_out, D.Nb);
  else
    logits_kernel<64><<<lgrid, kLogitThreads, 0, s>>>(qbar, kbar, L, logits_out, D.Nb);
  ++*launches;
  const size_t smem = kSelWarps * (sizeof(WarpHist) + 2 * sizeof(u64) * static_cast<size_t>(D.Nb));
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const unsigned sgrid = static_cast<unsigned>((D.rows() + kSelWarps - 1) / kSelWarps);
  select_kernel<<<sgrid, kSelWarps * 32, smem, s>>>(L, D.rows(), D.Nb, p, kk, topp_mask, topk_idx);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace fva
