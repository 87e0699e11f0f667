// Block-sparse flash attention on sm_100a tensor cores ("FVAttn: Adaptive Sparse
// Attention with Runtime Load Balancing for Video Generation", §3.1 overview —
// block-sparse attention over the routed pairs; §2 background — only the selected
// query/key block pairs are evaluated).
//
// Persistent kernel, one CTA per SM, walking a work list of (b, h, query-block)
// items (heavy items first when the caller passes the LPT list): with 128-token tiles at
// a stride of the grid, with 64-token tiles (two query blocks per item) by claiming list
// positions from a counter.  Per item the CTA keeps the 128-row Q tile in shared memory
// and streams the item's kept K and V blocks through two TMA rings; a K stage is released
// as soon as its S product is done, a V stage after its PV product.  Roles (12 warps):
//   warp 0    : TMA producer  — Q once per item, K_j per kept block; with 64-token tiles
//               it also claims each item and publishes it to the other warps
//   warp 3    : TMA producer  — V_j per kept block
//   warp 1    : MMA issuer    — S_j = Q K_j^T (both operands in shared memory)
//   warp 2    : MMA issuer    — O += P_j V_j (P from tensor memory); allocates TMEM
//   warps 4-11: softmax, O correction and epilogue — two warps per TMEM lane
//               quarter, each owning half of the columns of its 32 query rows
// One thread can issue a tcgen05.mma only about as fast as a 128x128x16 product
// runs, so the two kinds of product come from two warps on different SM
// sub-partitions and neither waits for the other's completion.  Tensor memory holds
// two S buffers and two bf16 P buffers besides the fp32 O accumulator (all 512
// columns at d = S = 128): S_{j+2} is issued as soon as the softmax has read S_j out,
// and the softmax writes P_j while P_{j-1} V_{j-1} may still run, so it never waits
// for a PV product except to rescale O.  Online softmax in base 2 with a lazy running
// max: O and the row sums are rescaled only when the max grows by more than 2^8; a
// quarter of the exponentials run on the FMA pipe (exp2_poly).
// Every wait is bounded; on expiry the CTA aborts, every role waits for the copies and
// products it issued, TMEM is freed, and kDevErrTimeout goes to the device error word.
#include <stdio.h>

#include <atomic>

#include "fva_common.cuh"
#include "fva_internal.h"

namespace fva {
namespace {

constexpr int kAttnThreads = 384;   // 12 warps: 4 control + 8 softmax
constexpr int kBM = 128;               // MMA M: query rows per tile (S=64 tiles use the top half)
constexpr float kLazyRescaleLog2 = 8.0f;
// Of every 8 probabilities a softmax thread computes, this many use the FMA-pipe
// exp2 (exp2_poly) instead of the MUFU unit, so both units share the work.
constexpr int kPolyPerEight = 2;
// Register split between the control warpgroup (warps 0-3) and the two softmax warpgroups.
constexpr int kCtrlRegs = 80;
constexpr int kSoftmaxRegs = 192;
// Bitmap words of one kept list (one bit per key block, up to kMaxNb blocks).
constexpr int kBmWords = kMaxNb / 32;
// Warps that copy each published work item (all but the K producer, which publishes it).
constexpr int kBmReaders = kAttnThreads / 32 - 1;

template <int D, int BN, int NSK, int NSV>
struct AttnCfg {
  // A "unit" is what one S product covers: KPU kept key blocks of BN rows, KN = 128 key
  // rows (one block of a 128-token tile, two of a 64-token tile).
  static constexpr int KPU = kBM / BN;
  static constexpr int KN = BN * KPU;
  static constexpr int NCH = D / 64;                         // 64-column (128-byte) chunks of a row
  static constexpr int Q_CHUNK = kBM * 128;                  // bytes of one Q chunk (128 rows)
  static constexpr int KV_CHUNK = KN * 128;                  // bytes of one K or V chunk of a unit
  static constexpr int Q_BYTES = NCH * Q_CHUNK;
  static constexpr int KV_BYTES = NCH * KV_CHUNK;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NSK * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + NSV * KV_BYTES;
  // barriers: q_full q_empty s_full[2] s_free[2] p_full[2] o_done[2] o_free drain_s drain_pv wk_full
  // wk_empty; k ring; v ring
  static constexpr int NBAR = 15 + 2 * NSK + 2 * NSV;
  static constexpr int OFF_RED = OFF_BAR + NBAR * 8;         // row maxima / sums [2 parity][2 half][128]
  static constexpr int OFF_MISC = OFF_RED + 2 * 2 * kBM * 4; // tmem base slot, abort flag
  static constexpr int OFF_SLOT = OFF_MISC + 16;             // the work-item slot (Slot)
  static constexpr int SMEM = OFF_SLOT + (16 + 2 * kBmWords * 4);   // base must be 1024-aligned (checked)
  // TMEM columns: S double buffer [0, 2*KN), P double buffer [2*KN, 3*KN) as bf16 pairs
  // (KN/2 columns each), O after it
  static constexpr int T_S = 0, T_P = 2 * KN, T_O = 3 * KN;
  static constexpr int TMEM_USED = T_O + D;
  static constexpr int TMEM_COLS = TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(kBM, KN, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(kBM, D, true);
  static constexpr uint32_t Q_TX = static_cast<uint32_t>(BN) * D * 2;   // S == BN rows loaded
  static constexpr uint32_t KV_TX = static_cast<uint32_t>(KN) * D * 2;
};

struct AttnParams {
  const int32_t* counts;
  const int32_t* idx;
  const int32_t* worklist;
  uint16_t* out;
  int* dev_err;
  long long n_items;
  long long n_iter;       // work positions: list entries, or (b, h, pair) without a list
  unsigned long long* claim;   // position counter, zero at launch; nullptr: positions at a grid stride
  int N;
  int Nb;
  float scale_log2;
  // natural != 0: row r of tile i is written at its natural token position (the inverse
  // reorder fused into the epilogue); grid X, Y and tile tt x ty x tx, nY x nX tiles
  int natural, Y, X, tt, ty, tx, nY, nX;
  const int32_t* order;   // tile numbering table (raster index of tile i), or nullptr
  long long wait_limit;   // cycles one pipeline wait may take before the CTA aborts
};

// Token position of row r of tile i in the output: tile-major i*S + r, or the natural
// raster index of that token when prm.natural is set (-1: bad numbering table entry).
__device__ __forceinline__ long long out_token(const AttnParams& prm, int i, int r, int S) {
  if (!prm.natural) return static_cast<long long>(i) * S + r;
  const int tr = prm.order ? prm.order[i] : i;
  if (tr < 0 || tr >= prm.Nb) return -1;
  const int bt = tr / (prm.nY * prm.nX);
  const int rem = tr - bt * prm.nY * prm.nX;
  const int by = rem / prm.nX;
  const int bx = rem - by * prm.nX;
  const int tyx = prm.ty * prm.tx;
  const int lt = r / tyx;
  const int rr = r - lt * tyx;
  const int ly = rr / prm.tx;
  const int lx = rr - ly * prm.tx;
  return (static_cast<long long>(bt * prm.tt + lt) * prm.Y + by * prm.ty + ly) * prm.X + bx * prm.tx + lx;
}

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
__device__ __forceinline__ int item_count(const AttnParams& prm, int item) {
  return item < 0 ? 0 : min(prm.counts[item], prm.Nb);
}
// One work item of the kernel.  With 128-token tiles: one query block (item).  With 64-token
// tiles: two adjacent query blocks 2p and 2p + 1 of a head share the 128-row query tile (rows
// 0-63 and 64-127) and run over the union of their kept lists, two key blocks per S product;
// each row masks the keys outside its own block's list, so every row's result is that of
// its own list.  The work list's entries for odd blocks carry no work (their pair runs at
// the entry of the even block); without a list the positions are the pairs themselves.
struct Work {
  int item;     // item id of the (first) query block
  int nq;       // query blocks in the tile (2 for a full pair)
  int n0, n1;   // kept-list lengths of the two blocks (n1 = 0 without a second block)
};
template <int KPU>
__device__ __forceinline__ bool work_at(const AttnParams& prm, long long it, Work& w) {
  int item;
  if (KPU == 2 && !prm.worklist) {   // position it = pair p of (b, h): item of block 2p
    const int np = (prm.Nb + 1) / 2;
    const long long bh = it / np;
    item = static_cast<int>(bh * prm.Nb + 2 * (it - bh * np));
  } else {
    item = item_at(prm, it);
  }
  if (item < 0) return false;
  w.item = item;
  w.n0 = item_count(prm, item);
  if (KPU == 1) {
    w.nq = 1;
    w.n1 = 0;
    return true;
  }
  const int i = item % prm.Nb;
  if (i & 1) return false;
  w.nq = i + 1 < prm.Nb ? 2 : 1;
  w.n1 = w.nq == 2 ? item_count(prm, item + 1) : 0;
  return true;
}

// Union of a pair's two kept-list bitmaps held across a warp's lanes (lane l: words l and
// l + 32), walked in ascending block order; every role walks it the same way.
struct Bitmaps {
  uint32_t a0, a1, b0, b1;   // this lane's words of block 2p's and block 2p+1's lists
};
__device__ __forceinline__ Bitmaps load_bitmaps(const uint32_t* bm) {
  const int lane = threadIdx.x & 31;
  return Bitmaps{bm[lane], bm[lane + 32], bm[kBmWords + lane], bm[kBmWords + lane + 32]};
}
__device__ __forceinline__ int union_size(const Bitmaps& b) {
  return static_cast<int>(__reduce_add_sync(0xffffffffu, __popc(b.a0 | b.b0) + __popc(b.a1 | b.b1)));
}
// Next key block of the union (warp-uniform cursor; -1 when exhausted).
struct Cursor {
  int w = -1;
  uint32_t rb = 0;
};
__device__ __forceinline__ int next_key(Cursor& c, const Bitmaps& b, int nwords) {
  while (c.rb == 0) {
    if (++c.w >= nwords) return -1;
    const uint32_t lo = b.a0 | b.b0, hi = b.a1 | b.b1;
    c.rb = __shfl_sync(0xffffffffu, c.w < 32 ? lo : hi, c.w & 31);
  }
  const int j = c.w * 32 + __ffs(c.rb) - 1;
  c.rb &= c.rb - 1;
  return j;
}
// Whether key block j is in the list of the pair's block `which` (0 or 1); warp-uniform.
__device__ __forceinline__ bool in_list(const Bitmaps& b, int which, int j) {
  const int w = j >> 5;
  const uint32_t lo = which ? b.b0 : b.a0, hi = which ? b.b1 : b.a1;
  return (__shfl_sync(0xffffffffu, w < 32 ? lo : hi, w & 31) >> (j & 31)) & 1u;
}
// Kept key block jj of item `item` (row i), replaced by the diagonal if out of range.
__device__ __forceinline__ int block_id(const AttnParams& prm, int item, int i, int jj, bool report) {
  int j = prm.idx[static_cast<long long>(item) * prm.Nb + jj];
  if (j < 0 || j >= prm.Nb) {
    if (report) set_device_error(prm.dev_err, kDevErrBadIndex);
    j = i;
  }
  return j;
}

// The work-item slot in shared memory.  The K producer claims every work item and publishes
// it here (item id, or -1 when no work is left; query blocks; list lengths; with 64-token
// tiles the two lists' bitmaps); each of the other warps waits for it, copies it and releases
// the slot, so all roles take the same items in the same order.
struct Slot {
  int item, nq, n0, n1;
  uint32_t bm[2 * kBmWords];
};
static_assert(sizeof(Slot) == 16 + 2 * kBmWords * 4, "slot layout");
template <int KPU>
__device__ __forceinline__ bool read_work(const Slot* slot, uint32_t full, uint32_t empty, long long k,
                                          volatile int* abort_flag, long long wlim, Work& w, Bitmaps& b) {
  if (!__all_sync(0xffffffffu, mbar_wait(full, k & 1, abort_flag, wlim))) return false;
  w.item = slot->item;
  w.nq = slot->nq;
  w.n0 = slot->n0;
  w.n1 = slot->n1;
  if (KPU == 2 && w.item >= 0) b = load_bitmaps(slot->bm);
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(empty);
  return true;
}
// The next work item of this CTA (whole warp, warp-uniform).  Positions are claimed from the
// launch's counter: every CTA moves through the list with the others (the K and V blocks they
// read at a time overlap in L2), and a CTA that finishes early takes the next item (greedy
// list order).  Without a counter the positions come at a stride of the grid.  Positions that
// carry no work (the odd block of a pair, an id outside the items) are passed over.
template <int KPU>
__device__ __forceinline__ bool next_work(const AttnParams& prm, long long& pos, Work& w) {
  while (true) {
    long long it;
    if (prm.claim) {
      unsigned long long c = 0;
      if ((threadIdx.x & 31) == 0) c = atomicAdd(prm.claim, 1ull);
      it = static_cast<long long>(__shfl_sync(0xffffffffu, c, 0));
    } else {
      it = pos < 0 ? static_cast<long long>(blockIdx.x) : pos + gridDim.x;
      pos = it;
    }
    if (it >= prm.n_iter) return false;
    if (work_at<KPU>(prm, it, w)) return true;
  }
}
// The next work item of a warp other than the K producer: 1 (w and, with 64-token tiles, b
// filled), 0 when no work is left, -1 when the wait expired.  With 128-token tiles every warp
// takes the positions at the grid stride itself (no claims, no slot: measured faster there,
// where every position carries work); with 64-token tiles it reads the published item.
template <int KPU>
__device__ __forceinline__ int take_work(const AttnParams& prm, long long& pos, const Slot* slot, uint32_t full,
                                         uint32_t empty, long long& pubs, volatile int* abort_flag, long long wlim,
                                         Work& w, Bitmaps& b) {
  if (KPU == 1) return next_work<1>(prm, pos, w) ? 1 : 0;
  if (!read_work<KPU>(slot, full, empty, pubs++, abort_flag, wlim, w, b)) return -1;
  return w.item < 0 ? 0 : 1;
}

// One TMA producer warp: one ring stage (K or V, 64-column boxes) per unit of KPU key blocks
// through an ns-stage ring, the blocks at consecutive row offsets.  With 64-token tiles the
// unit's two key blocks are the next two of the pair's union (a unit short of a block repeats
// its block; those rows get probability 0).  The K producer also loads each work item's Q
// rows and, with 64-token tiles, builds the pair's kept-list bitmaps.  The whole warp walks
// the loop and waits (warp-uniform); lane 0 issues.
template <int D, int BN, int NS, bool WITH_Q, typename Cfg>
__device__ void produce(const AttnParams& prm, const CUtensorMap* tm, const CUtensorMap* tmQ, uint32_t ring,
                        uint32_t full0, uint32_t empty0, uint32_t sQ, uint32_t q_full, uint32_t q_empty,
                        Slot* slot, uint32_t wk_full, uint32_t wk_empty, volatile int* abort_flag) {
  const int Nb = prm.Nb;
  const int lane = threadIdx.x & 31;
  const bool leader = lane == 0;
  const int nwords = (Nb + 31) / 32;
  long long g = 0, q_items = 0, pubs = 0, pos = -1;
  bool ok = true;
  while (ok) {
    Work w{-1, 0, 0, 0};
    Bitmaps bmr{0, 0, 0, 0};
    if (WITH_Q && Cfg::KPU == 1) {
      if (!next_work<1>(prm, pos, w)) break;
    } else if (WITH_Q) {
      // claim the next item, then publish it once every reader has copied the previous one
      const bool have = next_work<Cfg::KPU>(prm, pos, w);
      if (pubs > 0 &&
          !(ok = __all_sync(0xffffffffu, mbar_wait(wk_empty, (pubs - 1) & 1, abort_flag, prm.wait_limit))))
        break;
      if (!have) w.item = -1;
      if (Cfg::KPU == 2 && have && w.n0 + w.n1 > 0) {
        const int i = w.item % Nb;
        for (int e = lane; e < 2 * kBmWords; e += 32) slot->bm[e] = 0u;
        __syncwarp();
        for (int x = 0; x < w.nq; ++x) {
          const int n = x ? w.n1 : w.n0;
          for (int c = lane; c < n; c += 32) {
            const int j = block_id(prm, w.item + x, i + x, c, true);
            atomicOr(&slot->bm[x * kBmWords + (j >> 5)], 1u << (j & 31));
          }
        }
      }
      if (leader) {
        slot->item = w.item;
        slot->nq = w.nq;
        slot->n0 = w.n0;
        slot->n1 = w.n1;
      }
      __threadfence_block();
      __syncwarp();
      if (leader) mbar_arrive(wk_full);
      ++pubs;
      if (!have) break;
      if (Cfg::KPU == 2 && w.n0 + w.n1 > 0) bmr = load_bitmaps(slot->bm);
    } else {
      const int t = take_work<Cfg::KPU>(prm, pos, slot, wk_full, wk_empty, pubs, abort_flag, prm.wait_limit, w, bmr);
      if (t <= 0) {
        ok = t == 0;
        break;
      }
    }
    if (w.n0 + w.n1 <= 0) continue;   // an empty list: nothing to load (the softmax writes zeros)
    const long long bh = w.item / Nb;
    const int i = w.item - static_cast<int>(bh * Nb);
    const long long row0 = bh * prm.N;
    const int nu = Cfg::KPU == 2 ? (union_size(bmr) + 1) / 2 : w.n0;
    if (WITH_Q) {
      if (q_items > 0 &&
          !(ok = __all_sync(0xffffffffu, mbar_wait(q_empty, (q_items - 1) & 1, abort_flag, prm.wait_limit))))
        break;
      if (leader) {
        mbar_arrive_expect_tx(q_full, Cfg::Q_TX * static_cast<uint32_t>(w.nq));
        for (int x = 0; x < w.nq; ++x)
          for (int ch = 0; ch < Cfg::NCH; ++ch)
            tma_load_2d(sQ + ch * Cfg::Q_CHUNK + x * BN * 128, tmQ, q_full, ch * 64,
                        static_cast<int>(row0 + static_cast<long long>(i + x) * BN));
      }
      __syncwarp();
      ++q_items;
    }
    Cursor cur;
    for (int u = 0; u < nu; ++u, ++g) {
      int j0 = 0, j1 = 0;
      if (Cfg::KPU == 2) {
        j0 = next_key(cur, bmr, nwords);
        j1 = next_key(cur, bmr, nwords);
        if (j1 < 0) j1 = j0;
      }
      const int st = static_cast<int>(g % NS);
      if (g >= NS && !(ok = __all_sync(0xffffffffu, mbar_wait(empty0 + 8 * st, ((g / NS) - 1) & 1, abort_flag,
                                                              prm.wait_limit))))
        break;
      if (leader) {
        mbar_arrive_expect_tx(full0 + 8 * st, Cfg::KV_TX);
#pragma unroll
        for (int kb = 0; kb < Cfg::KPU; ++kb) {
          const int j = Cfg::KPU == 1 ? block_id(prm, w.item, i, u, WITH_Q) : (kb ? j1 : j0);
          for (int ch = 0; ch < Cfg::NCH; ++ch)
            tma_load_2d(ring + st * Cfg::KV_BYTES + ch * Cfg::KV_CHUNK + kb * BN * 128, tm, full0 + 8 * st, ch * 64,
                        static_cast<int>(row0 + static_cast<long long>(j) * BN));
        }
      }
      __syncwarp();
    }
  }
  if (leader) {
    if (!ok) set_device_error(prm.dev_err, kDevErrTimeout);
    // every copy issued lands before the CTA goes away, whether this role, another one
    // or nobody aborted: the last copy into each stage (earlier ones completed before
    // the stage was refilled) and the last Q.  On a normal exit the consumers already
    // waited for all of them, so these waits return at once.
    for (long long q = (g > NS ? g - NS : 0); q < g; ++q) drain_wait(full0 + 8 * (q % NS), (q / NS) & 1);
    if (WITH_Q && q_items > 0) drain_wait(q_full, (q_items - 1) & 1);
  }
  __syncwarp();
}

template <int D, int BN, int NSK, int NSV>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const AttnParams prm) {
  using C = AttnCfg<D, BN, NSK, NSV>;
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {
    // 128-byte-swizzled TMA tiles and MMA operands need 1024-byte alignment
    if (threadIdx.x == 0) set_device_error(prm.dev_err, kDevErrMisaligned);
    return;
  }
  const uint32_t sQ = sbase + C::OFF_Q;
  const uint32_t sK = sbase + C::OFF_K;
  const uint32_t sV = sbase + C::OFF_V;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const uint32_t q_full = bar0, q_empty = bar0 + 8, s_full0 = bar0 + 16, s_free0 = bar0 + 32;
  const uint32_t p_full0 = bar0 + 48, o_done0 = bar0 + 64, o_free = bar0 + 80, drain_s = bar0 + 88;
  const uint32_t drain_pv = bar0 + 96, wk_full = bar0 + 104, wk_empty = bar0 + 112;
  const uint32_t k_full0 = bar0 + 120;
  const uint32_t k_empty0 = k_full0 + 8 * NSK;
  const uint32_t v_full0 = k_empty0 + 8 * NSK;
  const uint32_t v_empty0 = v_full0 + 8 * NSV;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  Slot* slot = reinterpret_cast<Slot*>(smem + C::OFF_SLOT);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full0 + 8 * b, 1);
      mbar_init(s_free0 + 8 * b, 256);
      mbar_init(p_full0 + 8 * b, 256);
      mbar_init(o_done0 + 8 * b, 1);
    }
    mbar_init(o_free, 256);
    mbar_init(drain_s, 1);
    mbar_init(drain_pv, 1);
    mbar_init(wk_full, 1);
    mbar_init(wk_empty, kBmReaders);
    for (int st = 0; st < NSK; ++st) {
      mbar_init(k_full0 + 8 * st, 1);
      mbar_init(k_empty0 + 8 * st, 1);
    }
    for (int st = 0; st < NSV; ++st) {
      mbar_init(v_full0 + 8 * st, 1);
      mbar_init(v_empty0 + 8 * st, 1);
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

  const int Nb = prm.Nb;
  const int S = BN;
  const bool leader = lane == 0;
  const long long wlim = prm.wait_limit;
  auto wait_all = [&](uint32_t bar, uint32_t parity) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, wlim));
  };

  // Registers: the launch gives every thread 168; the control warpgroup returns what it
  // does not need and the softmax warpgroups take it.  128 x kCtrlRegs + 256 x kSoftmaxRegs
  // stays within the launch's 384 x 168, so the increase always finds its registers.
  static_assert(128 * kCtrlRegs + 256 * kSoftmaxRegs <= kAttnThreads * 168, "register split exceeds the launch");
  if (warp < 4) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCtrlRegs));
  if (warp == 0) {
    // ---------------------------------------------------------------- Q + K producer
    produce<D, BN, NSK, true, C>(prm, &tmK, &tmQ, sK, k_full0, k_empty0, sQ, q_full, q_empty, slot, wk_full, wk_empty,
                                 abort_flag);
  } else if (warp == 3) {
    // ---------------------------------------------------------------- V producer
    produce<D, BN, NSV, false, C>(prm, &tmV, &tmQ, sV, v_full0, v_empty0, sQ, q_full, q_empty, slot, wk_full, wk_empty,
                                  abort_flag);
  } else if (warp == 1) {
    // ---------------------------------------------------------------- S issuer
    // S_j = Q K_j^T into S buffer j % 2 as soon as the softmax has read S_{j-2} out of it.
    // (One thread issues a tcgen05.mma only every ~50 cycles, about the time a
    // 128x128x16 product takes, so S and PV products come from two warps on
    // different SM sub-partitions.)  The whole warp walks the loop and waits; lane 0
    // issues.
    const uint64_t dQ = sdesc_sw128(sQ, 16, 1024);
    const uint64_t dK0 = sdesc_sw128(sK, 16, 1024);
    // (descriptor start addresses are the low 14 bits, address >> 4; operands lie
    //  below 256 KB, so byte offsets add in without carry)
    long long g = 0, q_items = 0, pubs = 0, pos = -1;
    bool ok = true, issued = false;
    while (ok) {
      Work w{-1, 0, 0, 0};
      Bitmaps bmr{0, 0, 0, 0};
      const int t = take_work<C::KPU>(prm, pos, slot, wk_full, wk_empty, pubs, abort_flag, wlim, w, bmr);
      if (t <= 0) {
        ok = t == 0;
        break;
      }
      if (w.n0 + w.n1 <= 0) continue;
      if (!(ok = wait_all(q_full, q_items & 1))) break;
      ++q_items;
      const int nu = C::KPU == 2 ? (union_size(bmr) + 1) / 2 : w.n0;
      for (int jj = 0; jj < nu; ++jj, ++g) {
        const int b = static_cast<int>(g & 1);
        const int st = static_cast<int>(g % NSK);
        // S buffer b is free once the softmax has loaded S_{g-2}; the softmax never waits
        // on a PV product before writing P (P is double-buffered), so running S up to two
        // blocks ahead only keeps the tensor pipe fed
        if (g >= 2 && !(ok = wait_all(s_free0 + 8 * b, ((g >> 1) - 1) & 1))) break;
        if (!(ok = wait_all(k_full0 + 8 * st, (g / NSK) & 1))) break;
        if (leader) {
          tc_fence_after();
          const uint64_t dK = dK0 + static_cast<uint64_t>((st * C::KV_BYTES) >> 4);
          const uint32_t dS = tmem + C::T_S + b * C::KN;
#pragma unroll
          for (int ch = 0; ch < C::NCH; ++ch)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_ss(dS, dQ + ((ch * C::Q_CHUNK + kk * 32) >> 4), dK + ((ch * C::KV_CHUNK + kk * 32) >> 4),
                      C::IDESC_S, (ch | kk) != 0);
          umma_commit(k_empty0 + 8 * st);
          umma_commit(s_full0 + 8 * b);
          if (jj == nu - 1) umma_commit(q_empty);   // last reader of this item's Q
        }
        __syncwarp();
        issued = true;
      }
    }
    if (!ok && leader) set_device_error(prm.dev_err, kDevErrTimeout);
    if (issued) {
      if (leader) umma_commit(drain_s);
      __syncwarp();
      drain_wait(drain_s, 0);
    }
  } else if (warp == 2) {
    // ---------------------------------------------------------------- PV issuer
    // O += P_j V_j once the softmax has written P_j into P buffer j % 2 (p_full); the
    // commit on o_done[j % 2] tells the softmax that buffer and O are free again.
    const uint64_t dV0 = sdesc_sw128(sV, C::KV_CHUNK, 1024);
    long long g = 0, items = 0, pubs = 0, pos = -1;
    bool ok = true, issued = false;
    while (ok) {
      Work w{-1, 0, 0, 0};
      Bitmaps bmr{0, 0, 0, 0};
      const int t = take_work<C::KPU>(prm, pos, slot, wk_full, wk_empty, pubs, abort_flag, wlim, w, bmr);
      if (t <= 0) {
        ok = t == 0;
        break;
      }
      if (w.n0 + w.n1 <= 0) continue;
      const int nu = C::KPU == 2 ? (union_size(bmr) + 1) / 2 : w.n0;
      if (items > 0 && !(ok = wait_all(o_free, (items - 1) & 1))) break;   // epilogue read O
      for (int jj = 0; jj < nu; ++jj, ++g) {
        const int st = static_cast<int>(g % NSV);
        if (!(ok = wait_all(p_full0 + 8 * static_cast<int>(g & 1), (g >> 1) & 1))) break;
        if (!(ok = wait_all(v_full0 + 8 * st, (g / NSV) & 1))) break;
        if (leader) {
          tc_fence_after();
          const uint64_t dV = dV0 + static_cast<uint64_t>((st * C::KV_BYTES) >> 4);
          const uint32_t aP = tmem + C::T_P + static_cast<uint32_t>(g & 1) * (C::KN / 2);
#pragma unroll
          for (int ks = 0; ks < C::KN / 16; ++ks)
            umma_ts(tmem + C::T_O, aP + ks * 8, dV + ((ks * 16 * 128) >> 4), C::IDESC_PV,
                    (jj > 0 || ks > 0) ? 1u : 0u);
          umma_commit(v_empty0 + 8 * st);
          umma_commit(o_done0 + 8 * static_cast<uint32_t>(g & 1));
        }
        __syncwarp();
        issued = true;
      }
      ++items;
    }
    if (!ok && leader) set_device_error(prm.dev_err, kDevErrTimeout);
    if (issued) {
      if (leader) umma_commit(drain_pv);
      __syncwarp();
      drain_wait(drain_pv, 0);
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    // ---------------------------------------------------------------- softmax
    // Eight warps: warp w owns TMEM lane quarter w % 4 (query rows 32*(w%4) ...) and
    // half h = (w - 4) / 4 of the columns of S (and of P and O).  The two warps of a
    // quarter meet at named barrier 1 + quarter once per block to combine their row
    // maxima (and twice per item for the row sums); the barrier also ANDs their
    // "still ok" flags so a bounded-wait failure makes both leave together.  Waits
    // are warp-uniform: the tcgen05.ld/st below are warp-collective.
    constexpr int HB = C::KN / 2;                                 // S columns per half
    constexpr int HD = D / 2;                                     // O columns per half
    const int quarter = warp & 3;
    const int half = (warp - 4) >> 2;
    const int row = quarter * 32 + lane;                          // TMEM lane == query row
    // query block of this warp's rows within the work item: with 64-token tiles lane
    // quarters 0-1 hold block 2p and quarters 2-3 block 2p + 1
    const int which = C::KPU == 2 ? quarter >> 1 : 0;
    const int rloc = row - which * S;                             // row within its query block
    const int nwords = (Nb + 31) / 32;
    const int pair_bar = 1 + quarter;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tP0 = tmem + C::T_P + half * (HB / 2) + lane_off;   // P buffer 0; buffer 1 is KN/2 further
    const uint32_t tO = tmem + C::T_O + half * HD + lane_off;
    float* red_max = reinterpret_cast<float*>(smem + C::OFF_RED);         // [2][2][kBM]
    const float sl2 = prm.scale_log2;
    const uint64_t sl2x2 = f32x2_pack(sl2, sl2);
    long long g = 0, pubs = 0, pos = -1;   // units processed; work items read; list position
    bool ok = true;
    // wait until P_q V_q has completed (its commit on o_done[q % 2] is that barrier's
    // phase q / 2; P_{q+2} V_{q+2} cannot start before this warp writes P_{q+2}, so the
    // barrier is never two phases ahead of the one waited for)
    auto wait_pv = [&](long long q) {
      if (ok && q >= 0)
        ok = __all_sync(0xffffffffu, mbar_wait(o_done0 + 8 * static_cast<uint32_t>(q & 1), (q >> 1) & 1, abort_flag,
                                               wlim));
    };
    while (ok) {
      Work w{-1, 0, 0, 0};
      Bitmaps bmr{0, 0, 0, 0};
      const int t = take_work<C::KPU>(prm, pos, slot, wk_full, wk_empty, pubs, abort_flag, wlim, w, bmr);
      if (C::KPU == 2) {
        // both warps of the quarter leave together or not at all: a warp whose wait expired
        // still meets its partner here, so neither is left waiting at a pair barrier
        ok = bar_and(pair_bar, 64, t >= 0);
        if (!ok) break;
      }
      if (t <= 0) break;
      const long long bh = w.item / Nb;
      const int i = w.item - static_cast<int>(bh * Nb);
      // rows of a query block the tile does not hold (64-token tiles: the odd last block of a
      // head has no partner) skip every load, exponential and store: row r of P V depends on
      // row r of P only, and those rows of O are never written out
      const bool pad = which >= w.nq;
      const int nrow = which ? w.n1 : w.n0;                       // kept blocks of this row's block
      const long long tok = pad ? 0 : out_token(prm, i + which, rloc < S ? rloc : 0, S);
      if (tok < 0) set_device_error(prm.dev_err, kDevErrBadIndex);
      uint16_t* orow = prm.out + (bh * prm.N + (tok < 0 ? 0 : tok)) * D + half * HD;
      const bool wr = !pad && rloc < S && tok >= 0;   // this thread writes its row
      if (w.n0 + w.n1 <= 0) {
        if (wr)
          for (int c = 0; c < HD; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
        continue;
      }
      const int nu = C::KPU == 2 ? (union_size(bmr) + 1) / 2 : w.n0;
      Cursor cur;
      float m = -INFINITY;   // running max of the scaled logits (base-2 units), same in both halves
      float l = 0.0f;        // this half's running row sum at max m
      for (int jj = 0; jj < nu; ++jj, ++g) {
        const int b = static_cast<int>(g & 1);
        const int par = b;
        // this half's key block: the unit's block with 128-token tiles; with 64-token tiles
        // the unit's first or second union block, dead (probability 0) when it is missing or
        // outside this row's own kept list
        bool dead = pad || nrow <= 0;
        if (C::KPU == 2) {
          const int j0 = next_key(cur, bmr, nwords);
          const int j1 = next_key(cur, bmr, nwords);
          const int key = half ? j1 : j0;
          dead = dead || key < 0 || !in_list(bmr, which, key);
        }
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(s_full0 + 8 * b, (g >> 1) & 1, abort_flag, wlim));
        uint32_t r[HB];
        float pm = -INFINITY;
        if (ok) {
          tc_fence_after();
          if (!dead) {
            const uint32_t tS = tmem + C::T_S + b * C::KN + half * HB + lane_off;
#pragma unroll
            for (int c = 0; c < HB / 32; ++c) tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[c * 32]));
            tmem_wait_ld();
          }
          tc_fence_before();
          mbar_arrive(s_free0 + 8 * b);                           // S_j read out: buffer b may be refilled
          if (!dead) {
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < HB; c += 4) {
              mx[0] = fmax3(mx[0], __uint_as_float(r[c]), __uint_as_float(r[c + 1]));
              mx[1] = fmax3(mx[1], __uint_as_float(r[c + 2]), __uint_as_float(r[c + 3]));
            }
            pm = fmaxf(mx[0], mx[1]);
          }
          red_max[(par * 2 + half) * kBM + row] = pm;
        }
        ok = bar_and(pair_bar, 64, ok);                           // both halves' maxima published
        if (!ok) break;
        const float m_cand = fmaxf(pm, red_max[(par * 2 + (half ^ 1)) * kBM + row]) * sl2;
        float alpha = 1.0f;
        if (m_cand > m + kLazyRescaleLog2) {
          alpha = ex2_approx(m - m_cand);   // 0 on the first block (m = -inf)
          m = m_cand;
        }
        const uint64_t negm = f32x2_pack(-m, -m);
        uint64_t rs[4] = {0, 0, 0, 0};      // packed partial row sums
        if (!dead) {
#pragma unroll
          for (int c = 0; c < HB / 2; ++c) {
            // x = s * scale_log2 - m for two columns at once
            const uint64_t x2 =
                ffma2(f32x2_pack(__uint_as_float(r[2 * c]), __uint_as_float(r[2 * c + 1])), sl2x2, negm);
            float x0, x1;
            f32x2_unpack(x2, x0, x1);
            const bool poly = (c % 4) < (kPolyPerEight / 2);
            const float p0 = poly ? exp2_poly(x0) : ex2_approx(x0);
            const float p1 = poly ? exp2_poly(x1) : ex2_approx(x1);
            rs[c & 3] = fadd2(rs[c & 3], f32x2_pack(p0, p1));
            r[c] = pack_bf16x2(p0, p1);
          }
        } else {
#pragma unroll
          for (int c = 0; c < HB / 2; ++c) r[c] = 0u;
        }
        float a0, a1;
        f32x2_unpack(fadd2(fadd2(rs[0], rs[1]), fadd2(rs[2], rs[3])), a0, a1);
        l = l * alpha + (a0 + a1);
        // P buffer b last fed P_{g-2} V_{g-2}; O must hold every earlier product before
        // it is rescaled (rare: only when the max grows by more than 2^8)
        const bool rescale = jj > 0 && __any_sync(0xffffffffu, alpha != 1.0f);
        wait_pv(g - 2);
        if (rescale) wait_pv(g - 1);
        if (ok) {
          tc_fence_after();
          const uint32_t tP = tP0 + static_cast<uint32_t>(b) * (C::KN / 2);
          if (!pad) {
            if constexpr (HB / 2 >= 32) {
#pragma unroll
              for (int c = 0; c < HB / 64; ++c) tmem_st32(tP + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[c * 32]));
            } else {
              tmem_st16(tP, r);
            }
          }
          if (rescale && !pad) {
#pragma unroll
            for (int c = 0; c < HD / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(tO + c * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st32(tO + c * 32, o);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(p_full0 + 8 * b);
        }
      }
      // no early exit before these barriers: the partner warp must meet them too.  The
      // row sums go through the parity region the next block will use; both warps
      // are past their last reads of it, and the second barrier keeps the next
      // block's maxima from overwriting it before both have read it.
      wait_pv(g - 1);                                             // the item's last product is in O
      float* red_l = red_max + (g & 1) * 2 * kBM;
      red_l[half * kBM + row] = l;
      ok = bar_and(pair_bar, 64, ok);
      if (!ok) break;
      const float inv = 1.0f / (red_l[row] + red_l[kBM + row]);
      ok = bar_and(pair_bar, 64, ok);
      if (!ok) break;
      tc_fence_after();
      if (wr && nrow <= 0)   // an empty kept list (its partner's was not): all-zero output
        for (int c = 0; c < HD; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int c = 0; c < (pad || nrow <= 0 ? 0 : HD / 32); ++c) {
        uint32_t o[32];
        tmem_ld32(tO + c * 32, o);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
        if (wr) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(o_free);
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

// Pipeline wait limit of the next launches (0: kWaitLimitCycles); only a test changes it.
std::atomic<long long> g_wait_limit{0};

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

template <int D, int BN, int NSK, int NSV>
cudaError_t launch_t(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const AttnParams& prm,
                     cudaStream_t s) {
  using C = AttnCfg<D, BN, NSK, NSV>;
  static_assert(C::SMEM <= 232448, "shared memory budget");
  static_assert(C::TMEM_USED <= 512, "tensor memory budget");
  cudaError_t e =
      cudaFuncSetAttribute(attn_kernel<D, BN, NSK, NSV>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const long long grid = prm.n_iter < sm_count() ? prm.n_iter : sm_count();
  attn_kernel<D, BN, NSK, NSV><<<static_cast<unsigned>(grid), kAttnThreads, C::SMEM, s>>>(mq, mk, mv, prm);
  return cudaGetLastError();
}

}  // namespace

void set_attn_wait_limit(long long cycles) { g_wait_limit.store(cycles > 0 ? cycles : 0); }

cudaError_t launch_attention(const void* qr, const void* kr, const void* vr, const int32_t* counts, const int32_t* idx,
                             const int32_t* worklist, const Dims& D, const fva_geom* natural, float scale, void* out,
                             int* dev_err, unsigned long long* claim, cudaStream_t s, int* launches, char* msg,
                             size_t msg_len) {
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
  // 64-token tiles run pairs of query blocks: without a work list the positions are the
  // pairs themselves, with one the entries of odd blocks carry no work
  prm.n_iter = (D.S < 128 && !worklist) ? D.BH() * ((D.Nb + 1) / 2) : D.rows();
  prm.claim = D.S < 128 ? claim : nullptr;   // claims only for 64-token pairs
  prm.N = D.N;
  prm.Nb = D.Nb;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.natural = natural ? 1 : 0;
  prm.Y = natural ? natural->Y : 0;
  prm.X = natural ? natural->X : 0;
  prm.tt = natural ? natural->tt : 0;
  prm.ty = natural ? natural->ty : 0;
  prm.tx = natural ? natural->tx : 0;
  prm.nY = D.nY;
  prm.nX = D.nX;
  prm.order = natural ? D.order : nullptr;
  const long long wl = g_wait_limit.load();
  prm.wait_limit = wl > 0 ? wl : kWaitLimitCycles;
  cudaError_t e;
  if (prm.claim && (e = cudaMemsetAsync(prm.claim, 0, sizeof(*prm.claim), s)) != cudaSuccess) return e;
  if (D.d == 128 && D.S == 128)
    e = launch_t<128, 128, 3, 3>(mq, mk, mv, prm, s);
  else if (D.d == 128 && D.S == 64)
    e = launch_t<128, 64, 3, 3>(mq, mk, mv, prm, s);
  else if (D.d == 64 && D.S == 128)
    e = launch_t<64, 128, 5, 5>(mq, mk, mv, prm, s);
  else
    e = launch_t<64, 64, 5, 5>(mq, mk, mv, prm, s);
  ++*launches;
  return e;
}

}  // namespace fva

