// Block-sparse flash attention on sm_100a tensor cores ("FVAttn: Adaptive Sparse
// Attention with Runtime Load Balancing for Video Generation", §3.1 overview —
// block-sparse attention over the routed pairs; §2 background — only the selected
// query/key block pairs are evaluated).
//
// Persistent kernel, one CTA per SM, walking a work list of (b, h, query-block)
// items (heavy items first when the caller passes the LPT list).  Per item the CTA
// keeps the 128-row Q tile in shared memory and streams the item's kept K/V blocks
// through an NS-stage TMA ring.  Roles (8 warps):
//   warp 0  : TMA producer (one thread)        — Q once per item, K_j and V_j per block
//   warp 1  : MMA issuer (one thread)          — S_j = Q K_j^T (SS), O += P_j V_j (TS)
//   warp 2  : TMEM allocator
//   warps 4-7: softmax / correction / epilogue — thread r owns query row r (TMEM lane r)
// Tensor memory: two S buffers (double-buffered so S_{j+1} overlaps softmax j; the
// bf16 P_j overwrites the first half of its own S buffer and feeds the TS MMA) and
// the fp32 O accumulator.  Online softmax in base 2 with a lazy running max: O and
// the row sum are rescaled only when the max grows by more than 2^8.
// Every wait is bounded; on expiry the CTA drains its in-flight copies/MMAs, frees
// TMEM and reports kDevErrTimeout through the device error word.
#include <stdio.h>

#include "fva_common.cuh"
#include "fva_internal.h"

namespace fva {
namespace {

constexpr int kAttnThreads = 256;
constexpr int kBM = 128;               // MMA M: query rows per tile (S=64 tiles use the top half)
constexpr float kLazyRescaleLog2 = 8.0f;

template <int D, int BN, int NS>
struct AttnCfg {
  static constexpr int NCH = D / 64;                         // 64-column (128-byte) chunks of a row
  static constexpr int Q_CHUNK = kBM * 128;                  // bytes of one Q chunk (128 rows)
  static constexpr int KV_CHUNK = BN * 128;                  // bytes of one K or V chunk
  static constexpr int Q_BYTES = NCH * Q_CHUNK;
  static constexpr int KV_BYTES = NCH * KV_CHUNK;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NS * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + NS * KV_BYTES;
  // barriers: q_full, q_empty, o_done, o_free, drain, k_full[NS], v_full[NS], kv_empty[NS], s_full[2], p_full[2]
  static constexpr int NBAR = 5 + 3 * NS + 4;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;        // tmem base slot, abort flag
  static constexpr int SMEM = OFF_MISC + 16 + 1024;          // + slack to align the base to 1024
  static constexpr int TMEM_USED = 2 * BN + D;
  static constexpr int TMEM_COLS = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64 : TMEM_USED <= 128 ? 128
                                   : TMEM_USED <= 256 ? 256 : 512;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(kBM, BN, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(kBM, D, true);
  static constexpr uint32_t Q_TX = static_cast<uint32_t>(BN) * D * 2;   // S == BN rows loaded
  static constexpr uint32_t KV_TX = static_cast<uint32_t>(BN) * D * 2;
};

struct AttnParams {
  const int32_t* counts;
  const int32_t* idx;
  const int32_t* worklist;
  uint16_t* out;
  int* dev_err;
  long long n_items;
  int N;
  int Nb;
  float scale_log2;
};

// Work item at list position `it`; -1 (and the device error word set) if the list
// holds an id outside [0, n_items).  Every role calls this on the same data, so all
// roles skip the same entries.
__device__ __forceinline__ int item_at(const AttnParams& prm, long long it) {
  const long long u = prm.worklist ? prm.worklist[it] : it;
  if (u < 0 || u >= prm.n_items) {
    set_device_error(prm.dev_err, kDevErrBadIndex);
    return -1;
  }
  return static_cast<int>(u);
}

// Bounded wait that ignores the abort flag (used only while draining).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles / 4) break;
  }
}

template <int D, int BN, int NS>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const AttnParams prm) {
  using C = AttnCfg<D, BN, NS>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::OFF_Q;
  const uint32_t sK = sbase + C::OFF_K;
  const uint32_t sV = sbase + C::OFF_V;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const uint32_t q_full = bar0 + 0, q_empty = bar0 + 8, o_done = bar0 + 16, o_free = bar0 + 24, drain = bar0 + 32;
  auto k_full = [&](int s) { return bar0 + 40 + 8 * s; };
  auto v_full = [&](int s) { return bar0 + 40 + 8 * (NS + s); };
  auto kv_empty = [&](int s) { return bar0 + 40 + 8 * (2 * NS + s); };
  auto s_full = [&](int b) { return bar0 + 40 + 8 * (3 * NS + b); };
  auto p_full = [&](int b) { return bar0 + 40 + 8 * (3 * NS + 2 + b); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(o_done, 1);
    mbar_init(o_free, 128);
    mbar_init(drain, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(v_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full(b), 1);
      mbar_init(p_full(b), 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (BN < kBM) {
    // rows BN..127 of the Q tile are never loaded: keep them finite (zero)
    for (int ch = 0; ch < C::NCH; ++ch) {
      uint4* z = reinterpret_cast<uint4*>(smem + C::OFF_Q + ch * C::Q_CHUNK + BN * 128);
      for (int e = threadIdx.x; e < (kBM - BN) * 128 / 16; e += kAttnThreads) z[e] = make_uint4(0, 0, 0, 0);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS0 = tmem;              // S buffer b at columns b*BN
  const uint32_t tO = tmem + 2 * BN;      // O accumulator

  const long long n_items = prm.n_items;
  const int Nb = prm.Nb;
  const int S = BN;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      long long g = 0;          // running K/V block counter (ring position)
      long long q_items = 0;    // items whose Q was loaded
      bool ok = true;
      for (long long it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
        const int item = item_at(prm, it);
        const int n = item < 0 ? 0 : min(prm.counts[item], Nb);
        if (n <= 0) continue;
        const long long bh = item / Nb;
        const int i = item - static_cast<int>(bh * Nb);
        const long long row0 = bh * prm.N;
        if (q_items > 0 && !(ok = mbar_wait(q_empty, (q_items - 1) & 1, abort_flag))) break;
        mbar_arrive_expect_tx(q_full, C::Q_TX);
        for (int ch = 0; ch < C::NCH; ++ch)
          tma_load_2d(sQ + ch * C::Q_CHUNK, &tmQ, q_full, ch * 64, static_cast<int>(row0 + static_cast<long long>(i) * S));
        ++q_items;
        const int32_t* irow = prm.idx + static_cast<long long>(item) * Nb;
        for (int jj = 0; jj < n; ++jj, ++g) {
          int j = irow[jj];
          if (j < 0 || j >= Nb) {
            set_device_error(prm.dev_err, kDevErrBadIndex);
            j = i;
          }
          const int st = static_cast<int>(g % NS);
          if (g >= NS && !(ok = mbar_wait(kv_empty(st), ((g / NS) - 1) & 1, abort_flag))) break;
          const int krow = static_cast<int>(row0 + static_cast<long long>(j) * S);
          mbar_arrive_expect_tx(k_full(st), C::KV_TX);
          for (int ch = 0; ch < C::NCH; ++ch)
            tma_load_2d(sK + st * C::KV_BYTES + ch * C::KV_CHUNK, &tmK, k_full(st), ch * 64, krow);
          mbar_arrive_expect_tx(v_full(st), C::KV_TX);
          for (int ch = 0; ch < C::NCH; ++ch)
            tma_load_2d(sV + st * C::KV_BYTES + ch * C::KV_CHUNK, &tmV, v_full(st), ch * 64, krow);
        }
      }
      if (!ok) {
        // let the copies already issued land before the CTA goes away
        set_device_error(prm.dev_err, kDevErrTimeout);
        for (long long q = (g > NS ? g - NS : 0); q < g; ++q) {
          const int st = static_cast<int>(q % NS);
          drain_wait(k_full(st), (q / NS) & 1);
          drain_wait(v_full(st), (q / NS) & 1);
        }
        if (q_items > 0) drain_wait(q_full, (q_items - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      long long g = 0;          // K/V ring position (same sequence as the producer)
      long long sidx = 0;       // S buffer sequence number
      long long q_items = 0, o_items = 0;
      bool ok = true;
      bool issued = false;
      for (long long it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
        const int item = item_at(prm, it);
        const int n = item < 0 ? 0 : min(prm.counts[item], Nb);
        if (n <= 0) continue;
        if (!(ok = mbar_wait(q_full, q_items & 1, abort_flag))) break;
        ++q_items;
        // S_jj = Q K_jj^T into S buffer (sidx + jj) & 1
        auto issue_s = [&](int jj) -> bool {
          const long long gg = g + jj;
          const int st = static_cast<int>(gg % NS);
          if (!mbar_wait(k_full(st), (gg / NS) & 1, abort_flag)) return false;
          tc_fence_after();
          const uint32_t dS = tS0 + static_cast<uint32_t>(((sidx + jj) & 1) * BN);
#pragma unroll
          for (int ch = 0; ch < C::NCH; ++ch)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = sdesc_sw128(sQ + ch * C::Q_CHUNK + kk * 32, 16, 1024);
              const uint64_t bd = sdesc_sw128(sK + st * C::KV_BYTES + ch * C::KV_CHUNK + kk * 32, 16, 1024);
              umma_ss(dS, ad, bd, C::IDESC_S, (ch | kk) != 0);
            }
          umma_commit(s_full(static_cast<int>((sidx + jj) & 1)));
          issued = true;
          if (jj == n - 1) umma_commit(q_empty);   // last reader of this item's Q
          return true;
        };
        if (!(ok = issue_s(0))) break;
        for (int jj = 0; jj < n; ++jj) {
          if (jj + 1 < n && !(ok = issue_s(jj + 1))) break;
          const long long gg = g + jj;
          const int st = static_cast<int>(gg % NS);
          const int sb = static_cast<int>((sidx + jj) & 1);
          if (jj == 0 && o_items > 0 && !(ok = mbar_wait(o_free, (o_items - 1) & 1, abort_flag))) break;
          if (!(ok = mbar_wait(p_full(sb), ((sidx + jj) >> 1) & 1, abort_flag))) break;
          if (!(ok = mbar_wait(v_full(st), (gg / NS) & 1, abort_flag))) break;
          tc_fence_after();
          const uint32_t aP = tS0 + static_cast<uint32_t>(sb * BN);
#pragma unroll
          for (int ks = 0; ks < BN / 16; ++ks) {
            const uint64_t bd = sdesc_sw128(sV + st * C::KV_BYTES + ks * 16 * 128, C::KV_CHUNK, 1024);
            umma_ts(tO, aP + ks * 8, bd, C::IDESC_PV, (jj > 0 || ks > 0) ? 1u : 0u);
          }
          umma_commit(kv_empty(st));
          umma_commit(o_done);
        }
        if (!ok) break;
        g += n;
        sidx += n;
        ++o_items;
      }
      if (!ok) set_device_error(prm.dev_err, kDevErrTimeout);
      if (issued) {
        // every MMA issued by this thread has completed before TMEM is released
        umma_commit(drain);
        drain_wait(drain, 0);
      }
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- softmax
    // (waits are made warp-uniform: the tcgen05.ld/st below are warp-collective)
    const int row = (warp - 4) * 32 + lane;                      // TMEM lane == query row
    const uint32_t lane_off = static_cast<uint32_t>((warp - 4) * 32) << 16;
    const float sl2 = prm.scale_log2;
    long long sidx = 0, o_cnt = 0;
    bool ok = true;
    for (long long it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
      const int item = item_at(prm, it);
      if (item < 0) continue;
      const int n = min(prm.counts[item], Nb);
      const long long bh = item / Nb;
      const int i = item - static_cast<int>(bh * Nb);
      uint16_t* orow = prm.out + (bh * prm.N + static_cast<long long>(i) * S + row) * D;
      if (n <= 0) {
        if (row < S)
          for (int c = 0; c < D; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
        continue;
      }
      float m = -INFINITY;   // running max of the scaled logits (base-2 units)
      float l = 0.0f;        // running row sum at max m
      for (int jj = 0; jj < n; ++jj) {
        const int sb = static_cast<int>((sidx + jj) & 1);
        ok = __all_sync(0xffffffffu, mbar_wait(s_full(sb), ((sidx + jj) >> 1) & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
        uint32_t r[BN];
        const uint32_t tS = tS0 + static_cast<uint32_t>(sb * BN) + lane_off;
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[c * 32]));
        tmem_wait_ld();
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < BN; ++c) mx = fmaxf(mx, __uint_as_float(r[c]));
        const float m_cand = mx * sl2;
        float alpha = 1.0f;
        if (m_cand > m + kLazyRescaleLog2) {
          alpha = ex2_approx(m - m_cand);   // 0 on the first block (m = -inf)
          m = m_cand;
        }
        float rs = 0.0f;
#pragma unroll
        for (int c = 0; c < BN / 2; ++c) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(r[2 * c]), sl2, -m));
          const float p1 = ex2_approx(fmaf(__uint_as_float(r[2 * c + 1]), sl2, -m));
          rs += p0 + p1;
          r[c] = pack_bf16x2(p0, p1);
        }
        l = l * alpha + rs;
#pragma unroll
        for (int c = 0; c < BN / 64; ++c) tmem_st32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[c * 32]));
        if (jj > 0) {
          // O must hold P_{jj-1} V_{jj-1} before it is rescaled and P_jj V_jj is added
          ok = __all_sync(0xffffffffu, mbar_wait(o_done, o_cnt & 1, abort_flag));
          if (!ok) break;
          ++o_cnt;
          tc_fence_after();
          if (__any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(tO + lane_off + c * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st32(tO + lane_off + c * 32, o);
            }
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full(sb));
      }
      if (!ok) break;
      ok = __all_sync(0xffffffffu, mbar_wait(o_done, o_cnt & 1, abort_flag));
      if (!ok) break;
      ++o_cnt;
      tc_fence_after();
      const float inv = 1.0f / l;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + lane_off + c * 32, o);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
        if (row < S) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(o_free);
      sidx += n;
    }
    if (!ok) set_device_error(prm.dev_err, kDevErrTimeout);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, C::TMEM_COLS);
}

// ------------------------------------------------------------------ host side ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2D view [rows, D] of a bf16 [B,H,N,D] tensor; box = 64 columns x box_rows rows, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, long long rows, int D, int box_rows, char* msg, size_t msg_len) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) {
    snprintf(msg, msg_len, "cuTensorMapEncodeTiled entry point unavailable");
    return false;
  }
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(msg, msg_len, "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
    return false;
  }
  return true;
}

int sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 1;
  }
  return n;
}

template <int D, int BN, int NS>
cudaError_t launch_t(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const AttnParams& prm,
                     cudaStream_t s) {
  using C = AttnCfg<D, BN, NS>;
  static_assert(C::SMEM <= 232448, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<D, BN, NS>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const long long grid = prm.n_items < sm_count() ? prm.n_items : sm_count();
  attn_kernel<D, BN, NS><<<static_cast<unsigned>(grid), kAttnThreads, C::SMEM, s>>>(mq, mk, mv, prm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const void* qr, const void* kr, const void* vr, const int32_t* counts, const int32_t* idx,
                             const int32_t* worklist, const Dims& D, float scale, void* out, int* dev_err,
                             cudaStream_t s, int* launches, char* msg, size_t msg_len) {
  const long long rows = D.BH() * D.N;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, qr, rows, D.d, D.S, msg, msg_len) || !make_map(&mk, kr, rows, D.d, D.S, msg, msg_len) ||
      !make_map(&mv, vr, rows, D.d, D.S, msg, msg_len))
    return cudaErrorInvalidValue;
  AttnParams prm;
  prm.counts = counts;
  prm.idx = idx;
  prm.worklist = worklist;
  prm.out = static_cast<uint16_t*>(out);
  prm.dev_err = dev_err;
  prm.n_items = D.rows();
  prm.N = D.N;
  prm.Nb = D.Nb;
  prm.scale_log2 = scale * 1.4426950408889634f;
  cudaError_t e;
  if (D.d == 128 && D.S == 128)
    e = launch_t<128, 128, 2>(mq, mk, mv, prm, s);
  else if (D.d == 128 && D.S == 64)
    e = launch_t<128, 64, 4>(mq, mk, mv, prm, s);
  else if (D.d == 64 && D.S == 128)
    e = launch_t<64, 128, 4>(mq, mk, mv, prm, s);
  else
    e = launch_t<64, 64, 4>(mq, mk, mv, prm, s);
  ++*launches;
  return e;
}

}  // namespace fva
