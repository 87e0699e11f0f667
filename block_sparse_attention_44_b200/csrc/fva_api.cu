// C ABI entry points: argument validation, workspace carving and kernel launches.
// Nothing here allocates device memory or synchronises (except fva_get_device_error).
#include <math.h>
#include <stdarg.h>
#include <stdio.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <utility>
#include <vector>

#include "fva_common.cuh"
#include "fva_internal.h"

namespace {

thread_local char g_err[512] = "";
std::atomic<long long> g_launches{0};

// Device error words (fva::kDevErr*), one per stream: the first kErrSlots - 1 distinct
// streams a process launches on (per device) each get a word of their own; any further
// stream shares word 0.  A kernel reports into the word of the stream it runs on, and
// fva_get_device_error(stream) reads and clears that word only.
constexpr int kErrSlots = 64;
__device__ int g_dev_err[kErrSlots];
// Work-claim counters of the attention kernel, one per stream slot like the error words; a
// stream on the shared slot 0 gets none (two launches in flight must not share a counter).
__device__ unsigned long long g_claim[kErrSlots];

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_fail(cudaError_t e, const char* where) {
  return fail(FVA_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

// Slot of `stream` on the current device (1 .. kErrSlots - 1 for the first streams seen, 0 for
// any further stream) and the device's base addresses of the error words and claim counters;
// false if the runtime cannot say.
bool stream_slot(void* stream, int** err_base, unsigned long long** claim_base, int* slot_out) {
  constexpr int kMaxDev = 64;
  static std::mutex mu;
  static int* ebase[kMaxDev] = {nullptr};                // the arrays' addresses differ per device
  static unsigned long long* cbase[kMaxDev] = {nullptr};
  static std::vector<std::pair<void*, int>> slots[kMaxDev];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return false;
  std::lock_guard<std::mutex> lock(mu);
  if (!ebase[dev]) {
    void* p = nullptr;
    void* c = nullptr;
    if (cudaGetSymbolAddress(&p, g_dev_err) != cudaSuccess || cudaGetSymbolAddress(&c, g_claim) != cudaSuccess)
      return false;
    ebase[dev] = static_cast<int*>(p);
    cbase[dev] = static_cast<unsigned long long*>(c);
  }
  *err_base = ebase[dev];
  *claim_base = cbase[dev];
  for (const auto& e : slots[dev])
    if (e.first == stream) {
      *slot_out = e.second;
      return true;
    }
  const int slot = static_cast<int>(slots[dev].size()) + 1;
  if (slot >= kErrSlots) {                               // table full: the shared word
    *slot_out = 0;
    return true;
  }
  slots[dev].emplace_back(stream, slot);
  *slot_out = slot;
  return true;
}

// Error word of `stream` on the current device (nullptr if the runtime cannot say).
int* dev_err_ptr(void* stream) {
  int* eb = nullptr;
  unsigned long long* cb = nullptr;
  int slot = 0;
  if (!stream_slot(stream, &eb, &cb, &slot)) return nullptr;
  return eb + slot;
}

// Work-claim counter of `stream` (nullptr on the shared slot or if the runtime cannot say).
unsigned long long* claim_ptr(void* stream) {
  int* eb = nullptr;
  unsigned long long* cb = nullptr;
  int slot = 0;
  if (!stream_slot(stream, &eb, &cb, &slot) || slot == 0) return nullptr;
  return cb + slot;
}

// Validates the geometry; fills D.  Returns FVA_OK or an error code (message set).
int check_geom(const fva_geom& g, fva::Dims& D, bool need_attn_shapes) {
  if (g.B <= 0 || g.H <= 0 || g.T <= 0 || g.Y <= 0 || g.X <= 0 || g.d <= 0 || g.tt <= 0 || g.ty <= 0 || g.tx <= 0)
    return fail(FVA_ERR_INVALID_ARG, "geometry sizes must be positive");
  if (g.T % g.tt || g.Y % g.ty || g.X % g.tx)
    return fail(FVA_ERR_INVALID_ARG, "latent grid %dx%dx%d is not divisible by tile %dx%dx%d", g.T, g.Y, g.X, g.tt,
                g.ty, g.tx);
  const long long N = static_cast<long long>(g.T) * g.Y * g.X;
  const long long S = static_cast<long long>(g.tt) * g.ty * g.tx;
  const long long rows = static_cast<long long>(g.B) * g.H * N;
  if (rows > (1LL << 31) - 1 || N > (1LL << 30))
    return fail(FVA_ERR_INVALID_ARG, "too many tokens (B*H*N must fit in int32)");
  if (g.d != 64 && g.d != 128) return fail(FVA_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", g.d);
  if (S > 4096) return fail(FVA_ERR_UNSUPPORTED, "tile of %lld tokens not supported (<= 4096)", S);
  if (need_attn_shapes && S != 64 && S != 128)
    return fail(FVA_ERR_UNSUPPORTED, "tile of %lld tokens not supported (64 or 128)", S);
  D.B = g.B;
  D.H = g.H;
  D.N = static_cast<int>(N);
  D.d = g.d;
  D.S = static_cast<int>(S);
  D.Nb = static_cast<int>(N / S);
  D.nT = g.T / g.tt;
  D.nY = g.Y / g.ty;
  D.nX = g.X / g.tx;
  D.order = g.tile_order;
  if ((reinterpret_cast<uintptr_t>(g.tile_order) & 3u) != 0)
    return fail(FVA_ERR_INVALID_ARG, "tile_order must be 4-byte aligned");
  return FVA_OK;
}

// Position of cell c (each coordinate < 2^bits) along the 3D Hilbert curve of the
// 2^bits cube, by Skilling's transposed-index construction: from the top bit level
// down, undo the curve's rotations (reflect or exchange the lower bits with the first
// coordinate), Gray-code the coordinates, then read the transposed bits level by
// level, first coordinate first.
unsigned long long hilbert_index_3d(const unsigned (&c)[3], int bits) {
  unsigned x[3] = {c[0], c[1], c[2]};
  const unsigned top = 1u << (bits - 1);
  for (unsigned q = top; q > 1; q >>= 1) {
    const unsigned low = q - 1;
    for (int i = 0; i < 3; ++i) {
      if (x[i] & q) {
        x[0] ^= low;
      } else {
        const unsigned t = (x[0] ^ x[i]) & low;
        x[0] ^= t;
        x[i] ^= t;
      }
    }
  }
  x[1] ^= x[0];
  x[2] ^= x[1];
  unsigned flip = 0;
  for (unsigned q = top; q > 1; q >>= 1)
    if (x[2] & q) flip ^= q - 1;
  for (unsigned& v : x) v ^= flip;
  unsigned long long h = 0;
  for (int j = bits - 1; j >= 0; --j)
    for (int i = 0; i < 3; ++i) h = (h << 1) | ((x[i] >> j) & 1u);
  return h;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int finish(cudaError_t e, int launches, const char* where) {
  g_launches += launches;
  if (e != cudaSuccess) return cuda_fail(e, where);
  g_err[0] = '\0';
  return FVA_OK;
}

}  // namespace

extern "C" {

int32_t fva_version(void) { return 200; }

const char* fva_last_error(void) { return g_err; }

int64_t fva_launch_count(void) { return g_launches.load(); }

int fva_tile_order(fva_geom g, int32_t kind, int32_t* order_out) {
  fva::Dims D;
  int rc = check_geom(g, D, false);
  if (rc) return rc;
  if (!order_out) return fail(FVA_ERR_INVALID_ARG, "null pointer");
  const int n = D.Nb;
  if (kind == FVA_TILES_RASTER) {
    for (int b = 0; b < n; ++b) order_out[b] = b;
    g_err[0] = '\0';
    return FVA_OK;
  }
  if (kind != FVA_TILES_HILBERT) return fail(FVA_ERR_INVALID_ARG, "unknown tile numbering %d", kind);
  int side = 1, bits = 0;
  const int m = D.nT > D.nY ? (D.nT > D.nX ? D.nT : D.nX) : (D.nY > D.nX ? D.nY : D.nX);
  while (side < m) {
    side <<= 1;
    ++bits;
  }
  if (bits == 0) bits = 1;
  std::vector<std::pair<unsigned long long, int>> keys;
  keys.reserve(n);
  for (int bt = 0; bt < D.nT; ++bt)
    for (int by = 0; by < D.nY; ++by)
      for (int bx = 0; bx < D.nX; ++bx) {
        const unsigned c[3] = {static_cast<unsigned>(bt), static_cast<unsigned>(by), static_cast<unsigned>(bx)};
        keys.emplace_back(hilbert_index_3d(c, bits), (bt * D.nY + by) * D.nX + bx);
      }
  std::sort(keys.begin(), keys.end());
  for (int b = 0; b < n; ++b) order_out[b] = keys[b].second;
  g_err[0] = '\0';
  return FVA_OK;
}

static int reorder_common(const void* src, void* dst, fva_geom g, void* stream, bool inverse) {
  fva::Dims D;
  int rc = check_geom(g, D, false);
  if (rc) return rc;
  if (!src || !dst) return fail(FVA_ERR_INVALID_ARG, "null tensor pointer");
  if (src == dst) return fail(FVA_ERR_INVALID_ARG, "in-place reorder is not supported");
  if (!aligned16(src) || !aligned16(dst)) return fail(FVA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  int* de = dev_err_ptr(stream);
  if (!de) return fail(FVA_ERR_CUDA, "reorder: cannot resolve the device error word");
  int launches = 0;
  cudaError_t e = fva::launch_reorder(src, dst, g, D, inverse, de, static_cast<cudaStream_t>(stream), &launches);
  return finish(e, launches, inverse ? "fva_inverse_reorder" : "fva_reorder");
}

int fva_reorder(const void* x, void* xr, fva_geom g, void* stream) { return reorder_common(x, xr, g, stream, false); }

int fva_inverse_reorder(const void* xr, void* x, fva_geom g, void* stream) {
  return reorder_common(xr, x, g, stream, true);
}

int fva_reorder_pool(const void* x, void* xr, double* pooled, fva_geom g, void* stream) {
  fva::Dims D;
  int rc = check_geom(g, D, false);
  if (rc) return rc;
  if (!x || !xr || !pooled) return fail(FVA_ERR_INVALID_ARG, "null pointer");
  if (x == xr) return fail(FVA_ERR_INVALID_ARG, "in-place reorder is not supported");
  if (!aligned16(x) || !aligned16(xr)) return fail(FVA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(pooled) & 7u) != 0) return fail(FVA_ERR_INVALID_ARG, "pooled must be 8-byte aligned");
  int* de = dev_err_ptr(stream);
  if (!de) return fail(FVA_ERR_CUDA, "fva_reorder_pool: cannot resolve the device error word");
  int launches = 0;
  cudaError_t e = fva::launch_reorder_pool(x, xr, pooled, g, D, de, static_cast<cudaStream_t>(stream), &launches);
  return finish(e, launches, "fva_reorder_pool");
}

// Workspace of the routing calls: the float64 block means, then the LPT scratch.
static size_t route_ws_total(const fva::Dims& D) { return fva::route_workspace_bytes(D) + fva::lpt_workspace_bytes(D); }

size_t fva_route_workspace_size(fva_geom g) {
  fva::Dims D;
  if (check_geom(g, D, false)) return 0;
  return route_ws_total(D);
}

// Checks a caller workspace of at least `need` bytes; FVA_OK or an error (message set).
static int check_ws(const void* ws, size_t ws_bytes, size_t need) {
  if (!ws) return fail(FVA_ERR_INVALID_ARG, "null workspace");
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return fail(FVA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (ws_bytes < need)
    return fail(FVA_ERR_INVALID_ARG, "workspace too small: %zu bytes given, %zu needed", ws_bytes, need);
  return FVA_OK;
}

int fva_route(const void* qr, const void* kr, fva_geom g, double p, int32_t k, uint8_t* topp_mask, int32_t* topk_idx,
              double* logits_out, void* workspace, size_t workspace_bytes, void* stream) {
  fva::Dims D;
  int rc = check_geom(g, D, false);
  if (rc) return rc;
  if (!qr || !kr || !topp_mask || !topk_idx) return fail(FVA_ERR_INVALID_ARG, "null pointer");
  if (!(p > 0.0) || !(p <= 1.0)) return fail(FVA_ERR_INVALID_ARG, "p must satisfy 0 < p <= 1 (got %g)", p);
  if (k < 1) return fail(FVA_ERR_INVALID_ARG, "k must be >= 1 (got %d)", k);
  if (D.Nb > fva::kMaxNb) return fail(FVA_ERR_UNSUPPORTED, "Nb = %d blocks exceeds %d", D.Nb, fva::kMaxNb);
  if (!aligned16(qr) || !aligned16(kr)) return fail(FVA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  if ((rc = check_ws(workspace, workspace_bytes, route_ws_total(D)))) return rc;
  const int kk = k < D.Nb ? k : D.Nb;
  int launches = 0;
  cudaError_t e = fva::launch_route(qr, kr, D, p, kk, topp_mask, topk_idx, logits_out, nullptr, nullptr, workspace,
                                    static_cast<cudaStream_t>(stream), &launches);
  return finish(e, launches, "fva_route");
}

int fva_route_repair(const void* qr, const void* kr, fva_geom g, double p, int32_t k, uint8_t* topp_mask,
                     int32_t* topk_idx, int32_t* counts, int32_t* idx, int64_t* head_work, int32_t* worklist,
                     void* workspace, size_t workspace_bytes, void* stream) {
  fva::Dims D;
  int rc = check_geom(g, D, false);
  if (rc) return rc;
  if (!qr || !kr || !counts || !idx || !head_work || !worklist) return fail(FVA_ERR_INVALID_ARG, "null pointer");
  if (!(p > 0.0) || !(p <= 1.0)) return fail(FVA_ERR_INVALID_ARG, "p must satisfy 0 < p <= 1 (got %g)", p);
  if (k < 1) return fail(FVA_ERR_INVALID_ARG, "k must be >= 1 (got %d)", k);
  if (D.Nb > fva::kMaxNb) return fail(FVA_ERR_UNSUPPORTED, "Nb = %d blocks exceeds %d", D.Nb, fva::kMaxNb);
  if (!aligned16(qr) || !aligned16(kr)) return fail(FVA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  if ((rc = check_ws(workspace, workspace_bytes, route_ws_total(D)))) return rc;
  const int kk = k < D.Nb ? k : D.Nb;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* lpt_ws = static_cast<unsigned char*>(workspace) + fva::route_workspace_bytes(D);
  int launches = 0;
  cudaError_t e = fva::launch_route(qr, kr, D, p, kk, topp_mask, topk_idx, nullptr, counts, idx, workspace, s,
                                    &launches);
  if (e == cudaSuccess) e = fva::launch_lpt(counts, D, head_work, worklist, lpt_ws, s, &launches);
  return finish(e, launches, "fva_route_repair");
}

int fva_route_repair_pooled(const double* qbar, const double* kbar, fva_geom g, double p, int32_t k,
                            uint8_t* topp_mask, int32_t* topk_idx, int32_t* counts, int32_t* idx,
                            int64_t* head_work, int32_t* worklist, void* workspace, size_t workspace_bytes,
                            void* stream) {
  fva::Dims D;
  int rc = check_geom(g, D, false);
  if (rc) return rc;
  if (!qbar || !kbar || !counts || !idx || !head_work || !worklist) return fail(FVA_ERR_INVALID_ARG, "null pointer");
  if (!(p > 0.0) || !(p <= 1.0)) return fail(FVA_ERR_INVALID_ARG, "p must satisfy 0 < p <= 1 (got %g)", p);
  if (k < 1) return fail(FVA_ERR_INVALID_ARG, "k must be >= 1 (got %d)", k);
  if (D.Nb > fva::kMaxNb) return fail(FVA_ERR_UNSUPPORTED, "Nb = %d blocks exceeds %d", D.Nb, fva::kMaxNb);
  if (!aligned16(qbar) || !aligned16(kbar)) return fail(FVA_ERR_INVALID_ARG, "qbar and kbar must be 16-byte aligned");
  if ((rc = check_ws(workspace, workspace_bytes, fva::lpt_workspace_bytes(D)))) return rc;
  const int kk = k < D.Nb ? k : D.Nb;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  int launches = 0;
  cudaError_t e = fva::launch_select_pooled(qbar, kbar, D, p, kk, topp_mask, topk_idx, nullptr, counts, idx, s,
                                            &launches);
  if (e == cudaSuccess) e = fva::launch_lpt(counts, D, head_work, worklist, workspace, s, &launches);
  return finish(e, launches, "fva_route_repair_pooled");
}

static size_t sasa_lpt_offset(const fva::Dims& D) { return (fva::sasa_workspace_bytes(D) + 255) & ~static_cast<size_t>(255); }

size_t fva_sasa_workspace_size(fva_geom g) {
  fva::Dims D;
  if (check_geom(g, D, false)) return 0;
  return sasa_lpt_offset(D) + fva::lpt_workspace_bytes(D);
}

int fva_route_repair_sasa(const double* qbar, const double* kbar, fva_geom g, double p, int32_t k, int32_t num_ranks,
                          double alpha, int32_t* counts, int32_t* idx, int64_t* head_work, int32_t* worklist,
                          int32_t* extra, void* workspace, size_t workspace_bytes, void* stream) {
  fva::Dims D;
  int rc = check_geom(g, D, false);
  if (rc) return rc;
  if (!qbar || !kbar || !counts || !idx || !head_work || !worklist || !workspace)
    return fail(FVA_ERR_INVALID_ARG, "null pointer");
  if (!(p > 0.0) || !(p <= 1.0)) return fail(FVA_ERR_INVALID_ARG, "p must satisfy 0 < p <= 1 (got %g)", p);
  if (k < 1) return fail(FVA_ERR_INVALID_ARG, "k must be >= 1 (got %d)", k);
  if (num_ranks < 1 || num_ranks > fva::kMaxVirtualRanks || g.H % num_ranks != 0)
    return fail(FVA_ERR_INVALID_ARG, "num_ranks must divide H and lie in [1, %d] (got %d)", fva::kMaxVirtualRanks,
                num_ranks);
  if (!(alpha >= 0.0) || !(alpha <= 1.0)) return fail(FVA_ERR_INVALID_ARG, "alpha must lie in [0, 1] (got %g)", alpha);
  if (D.Nb > fva::kMaxNb) return fail(FVA_ERR_UNSUPPORTED, "Nb = %d blocks exceeds %d", D.Nb, fva::kMaxNb);
  if (!aligned16(qbar) || !aligned16(kbar)) return fail(FVA_ERR_INVALID_ARG, "qbar and kbar must be 16-byte aligned");
  if ((rc = check_ws(workspace, workspace_bytes, sasa_lpt_offset(D) + fva::lpt_workspace_bytes(D)))) return rc;
  const int kk = k < D.Nb ? k : D.Nb;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  int launches = 0;
  cudaError_t e = fva::launch_sasa(qbar, kbar, D, p, kk, num_ranks, alpha, counts, idx, extra, workspace, s,
                                   &launches);
  if (e == cudaSuccess)
    e = fva::launch_lpt(counts, D, head_work, worklist, static_cast<unsigned char*>(workspace) + sasa_lpt_offset(D), s,
                        &launches);
  return finish(e, launches, "fva_route_repair_sasa");
}

size_t fva_repair_workspace_size(fva_geom g) {
  fva::Dims D;
  if (check_geom(g, D, false)) return 0;
  return fva::lpt_workspace_bytes(D);
}

int fva_repair(const uint8_t* topp_mask, const int32_t* topk_idx, fva_geom g, int32_t k, int32_t* counts, int32_t* idx,
               int64_t* head_work, int32_t* worklist, void* workspace, size_t workspace_bytes, void* stream) {
  fva::Dims D;
  int rc = check_geom(g, D, false);
  if (rc) return rc;
  if (!topp_mask || !topk_idx || !counts || !idx || !head_work || !worklist)
    return fail(FVA_ERR_INVALID_ARG, "null pointer");
  if (k < 1) return fail(FVA_ERR_INVALID_ARG, "k must be >= 1 (got %d)", k);
  if (D.Nb > fva::kMaxNb) return fail(FVA_ERR_UNSUPPORTED, "Nb = %d blocks exceeds %d", D.Nb, fva::kMaxNb);
  if ((rc = check_ws(workspace, workspace_bytes, fva::lpt_workspace_bytes(D)))) return rc;
  int* de = dev_err_ptr(stream);
  if (!de) return fail(FVA_ERR_CUDA, "fva_repair: cannot resolve the device error word");
  const int kk = k < D.Nb ? k : D.Nb;
  int launches = 0;
  cudaError_t e = fva::launch_repair(topp_mask, topk_idx, D, kk, counts, idx, head_work, worklist, workspace, de,
                                     static_cast<cudaStream_t>(stream), &launches);
  return finish(e, launches, "fva_repair");
}

static int attn_common(const void* qr, const void* kr, const void* vr, const int32_t* counts, const int32_t* idx,
                       const int32_t* worklist, fva_geom g, float softmax_scale, void* out, void* stream,
                       bool natural, const char* name) {
  fva::Dims D;
  int rc = check_geom(g, D, true);
  if (rc) return rc;
  if (!qr || !kr || !vr || !counts || !idx || !out) return fail(FVA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(qr) || !aligned16(kr) || !aligned16(vr) || !aligned16(out))
    return fail(FVA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  if (!isfinite(softmax_scale)) return fail(FVA_ERR_INVALID_ARG, "softmax_scale must be finite");
  const float scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / sqrtf(static_cast<float>(D.d));
  int* de = dev_err_ptr(stream);
  if (!de) return fail(FVA_ERR_CUDA, "%s: cannot resolve the device error word", name);
  char msg[256] = "";
  int launches = 0;
  cudaError_t e = fva::launch_attention(qr, kr, vr, counts, idx, worklist, D, natural ? &g : nullptr, scale, out, de,
                                        claim_ptr(stream), static_cast<cudaStream_t>(stream), &launches, msg,
                                        sizeof(msg));
  if (msg[0]) {
    g_launches += launches;
    return fail(FVA_ERR_CUDA, "%s: %s", name, msg);
  }
  return finish(e, launches, name);
}

int fva_block_sparse_attn(const void* qr, const void* kr, const void* vr, const int32_t* counts, const int32_t* idx,
                          const int32_t* worklist, fva_geom g, float softmax_scale, void* out_r, void* stream) {
  return attn_common(qr, kr, vr, counts, idx, worklist, g, softmax_scale, out_r, stream, false,
                     "fva_block_sparse_attn");
}

int fva_block_sparse_attn_natural(const void* qr, const void* kr, const void* vr, const int32_t* counts,
                                  const int32_t* idx, const int32_t* worklist, fva_geom g, float softmax_scale,
                                  void* out, void* stream) {
  return attn_common(qr, kr, vr, counts, idx, worklist, g, softmax_scale, out, stream, true,
                     "fva_block_sparse_attn_natural");
}

int fva_debug_set_wait_limit(int64_t cycles) {
  fva::set_attn_wait_limit(cycles);
  g_err[0] = '\0';
  return FVA_OK;
}

int fva_get_device_error(void* stream, int32_t* code) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "fva_get_device_error");
  int* de = dev_err_ptr(stream);
  if (!de) return fail(FVA_ERR_CUDA, "fva_get_device_error: cannot resolve the device error word");
  int v = 0;
  e = cudaMemcpy(&v, de, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "fva_get_device_error");
  if (v) {
    const int zero = 0;
    e = cudaMemcpy(de, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "fva_get_device_error");
  }
  if (code) *code = v;
  if (v == fva::kDevErrTimeout) return fail(FVA_ERR_TIMEOUT, "a bounded device wait expired");
  if (v) return fail(FVA_ERR_INVALID_ARG, "a kernel rejected its input (device error %d)", v);
  g_err[0] = '\0';
  return FVA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------------
// fva_route_static: fva_route without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they route: a plugin
// running inside a host framework that owns every device allocation and hands its
// plugins no allocator, or a latency-critical serving loop whose memory plan is fixed
// before it starts and where a cudaMalloc (which may synchronise the device or fail
// under fragmentation) is not acceptable.  For them the routing scratch lives in one
// file-scope device array of fixed size, reserved on every GPU that loads this
// library and held until the process exits.
// ---------------------------------------------------------------------------------
namespace {

constexpr size_t kRouteStaticScratchBytes = FVA_ROUTE_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_route_scratch[kRouteStaticScratchBytes];

// Device address of g_route_scratch on the current device.  In host code the symbol
// only names a host-side stand-in, so the address must come from the runtime; it is
// looked up once per device, with that device current, on the first call there.
void* route_scratch_ptr() {
  static std::atomic<void*> ptrs[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  void* p = ptrs[dev].load();
  if (!p) {
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess) return nullptr;
    ptrs[dev].store(p);
  }
  return p;
}

}  // namespace

extern "C" int fva_route_static(const void* qr, const void* kr, fva_geom g, double p, int32_t k,
                                uint8_t* topp_mask, int32_t* topk_idx, double* logits_out, void* stream) {
  fva::Dims D;
  int rc = check_geom(g, D, false);
  if (rc) return rc;
  if (!qr || !kr || !topp_mask || !topk_idx) return fail(FVA_ERR_INVALID_ARG, "null pointer");
  if (!(p > 0.0) || !(p <= 1.0)) return fail(FVA_ERR_INVALID_ARG, "p must satisfy 0 < p <= 1 (got %g)", p);
  if (k < 1) return fail(FVA_ERR_INVALID_ARG, "k must be >= 1 (got %d)", k);
  if (D.Nb > fva::kMaxNb) return fail(FVA_ERR_UNSUPPORTED, "Nb = %d blocks exceeds %d", D.Nb, fva::kMaxNb);
  if (!aligned16(qr) || !aligned16(kr)) return fail(FVA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  const size_t need = route_ws_total(D);   // the size fva_route_workspace_size() reports
  if (need > kRouteStaticScratchBytes)
    return fail(FVA_ERR_UNSUPPORTED,
                "fva_route_static: this geometry needs %zu bytes of routing scratch, more than the %zu-byte "
                "static scratch; use fva_route with a caller workspace",
                need, kRouteStaticScratchBytes);
  void* scratch = route_scratch_ptr();
  if (!scratch) return fail(FVA_ERR_CUDA, "fva_route_static: cannot resolve the static scratch address");
  const int kk = k < D.Nb ? k : D.Nb;
  int launches = 0;
  cudaError_t e = fva::launch_route(qr, kr, D, p, kk, topp_mask, topk_idx, logits_out, nullptr, nullptr, scratch,
                                    static_cast<cudaStream_t>(stream), &launches);
  return finish(e, launches, "fva_route_static");
}
