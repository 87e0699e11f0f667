// Host-side launchers shared between the API translation unit and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/fva.h"

namespace fva {

// Derived sizes of a validated geometry.
struct Dims {
  int B, H, N, d, S, Nb, nT, nY, nX;
  const int32_t* order;   // tile numbering (device, Nb entries) or nullptr for raster
  long long BH() const { return static_cast<long long>(B) * H; }
  long long rows() const { return BH() * Nb; }   // (b, h, query-block) rows / work items
};

constexpr int kMaxNb = 2048;

// Reorder / inverse reorder of one bf16 [B,H,N,d] tensor.
cudaError_t launch_reorder(const void* src, void* dst, const fva_geom& g, const Dims& D, bool inverse,
                           int* dev_err, cudaStream_t s, int* launches);

// Forward reorder that also writes the float64 mean of every tile ([B*H*Nb, d]).
cudaError_t launch_reorder_pool(const void* src, void* dst, double* pooled, const fva_geom& g, const Dims& D,
                                int* dev_err, cudaStream_t s, int* launches);

// Routing: block means (float64), float64 logits, Top-p / Top-k selection; with
// counts != nullptr also the repaired, compacted per-row lists (idx, counts).
// topp_mask, topk_idx and logits_out may each be null (not written).
cudaError_t launch_route(const void* qr, const void* kr, const Dims& D, double p, int kk, uint8_t* topp_mask,
                         int32_t* topk_idx, double* logits_out, int32_t* counts, int32_t* idx, void* ws,
                         cudaStream_t s, int* launches);
size_t route_workspace_bytes(const Dims& D);
// Scoring and selection (and compaction when counts != nullptr) from block means the
// caller already holds (e.g. written by launch_reorder_pool).
cudaError_t launch_select_pooled(const double* qbar, const double* kbar, const Dims& D, double p, int kk,
                                 uint8_t* topp_mask, int32_t* topk_idx, double* logits_out, int32_t* counts,
                                 int32_t* idx, cudaStream_t s, int* launches);

// Repair + compaction + per-head work + LPT work list (ws: lpt_workspace_bytes).
cudaError_t launch_repair(const uint8_t* topp_mask, const int32_t* topk_idx, const Dims& D, int kk, int32_t* counts,
                          int32_t* idx, int64_t* head_work, int32_t* worklist, void* ws, int* dev_err,
                          cudaStream_t s, int* launches);

// Slack-aware augmentation from block means: selection (recording each row's ranked
// prefix), per-row floors from the virtual-rank budgets, selection again with them.
cudaError_t launch_sasa(const double* qbar, const double* kbar, const Dims& D, double p, int kk, int num_ranks,
                        double alpha, int32_t* counts, int32_t* idx, int32_t* extra, void* ws, cudaStream_t s,
                        int* launches);
size_t sasa_workspace_bytes(const Dims& D);
constexpr int kMaxVirtualRanks = 1024;

// Per-head work W_h and the LPT work list from the per-row counts; ws holds
// lpt_workspace_bytes(D) (per-head histograms, then list offsets), 256-byte aligned.
cudaError_t launch_lpt(const int32_t* counts, const Dims& D, int64_t* head_work, int32_t* worklist, void* ws,
                       cudaStream_t s, int* launches);
size_t lpt_workspace_bytes(const Dims& D);

// Pipeline wait limit (cycles) of the attention launches that follow; <= 0 restores
// the default.  Test-only: lets a test make a wait expire on purpose.
void set_attn_wait_limit(long long cycles);

// Block-sparse attention (tcgen05).
// natural != nullptr: O is written in natural token order of that geometry.
// claim: a device counter private to this stream (zeroed here before the launch) from which
// the CTAs claim work positions, or nullptr for positions at a grid stride.
cudaError_t launch_attention(const void* qr, const void* kr, const void* vr, const int32_t* counts, const int32_t* idx,
                             const int32_t* worklist, const Dims& D, const fva_geom* natural, float scale, void* out,
                             int* dev_err, unsigned long long* claim, cudaStream_t s, int* launches, char* msg,
                             size_t msg_len);

}  // namespace fva
