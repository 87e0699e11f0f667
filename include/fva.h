/*
 * fva.h — C ABI of the B200 (sm_100a) adaptive block-sparse attention path.
 *
 * The method is the one of "FVAttn: Adaptive Sparse Attention with Runtime Load
 * Balancing for Video Generation" (abstract; §2 background on dynamic block-sparse
 * routing; §3.1 pipeline overview), restricted to one GPU:
 *
 *   fva_reorder          video-aware block organisation: latent T x Y x X tokens -> 3D tiles
 *   fva_route            pooled Q/K block scores, Top-p CDF cut, Top-k floor
 *   fva_repair           forced diagonal + floor, compaction into per-row key-block lists,
 *                        per-head realised workload, heavy-first (LPT) work list
 *   fva_route_repair     the two above, fused
 *   fva_reorder_pool, fva_route_repair_pooled
 *                        the same with the pooling done by the reorder pass
 *   fva_route_repair_sasa  with slack-aware augmentation of the lists
 *   fva_block_sparse_attn  flash-style attention over the kept block pairs
 *   fva_inverse_reorder  back to natural token order
 *   fva_block_sparse_attn_natural  attention with the inverse reorder fused
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All tensor pointers are DEVICE pointers owned by the caller; nothing here
 *   allocates device memory.  Scratch comes from a caller-provided workspace whose
 *   size the matching *_workspace_size() query returns (bytes, 256-aligned start).
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   Every call only enqueues work on that stream and returns; nothing synchronises
 *   except fva_get_device_error().
 * - bf16 tensors hold IEEE bfloat16 bit patterns.  "[B,H,N,d]" means row-major,
 *   d fastest, N = T*Y*X tokens, contiguous, 16-byte aligned.
 * - Token order: natural n = (t*Y + y)*X + x.  Reordered position n' = b*S + r with
 *   b the raster index of the tile over (T/tt, Y/ty, X/tx) and r the raster index of
 *   the token inside the tile over (tt, ty, tx); S = tt*ty*tx, Nb = N/S.
 * - Return value: FVA_OK or an FVA_ERR_* code; on error nothing was enqueued and
 *   fva_last_error() (thread-local) describes it.
 */
#ifndef FVA_H
#define FVA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  FVA_OK = 0,
  FVA_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, grid not divisible by tile, p/k out of range, short workspace */
  FVA_ERR_UNSUPPORTED = 2,   /* a valid request this build does not implement (see each call) */
  FVA_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed; fva_last_error() has the CUDA message */
  FVA_ERR_TIMEOUT = 4        /* a bounded device-side wait expired (reported by fva_get_device_error) */
};

/*
 * Problem geometry: batch B, heads H, latent grid T x Y x X, head_dim d, tile tt x ty x tx.
 * tile_order: NULL for raster numbering of the tiles, else a DEVICE int32 array of Nb
 * entries, tile_order[b] = raster index (bt * nY + by) * nX + bx of the tile numbered b
 * (a permutation of [0, Nb), e.g. the Hilbert numbering from fva_tile_order).  Only the
 * token permutation uses it: fva_reorder, fva_reorder_pool, fva_inverse_reorder and
 * fva_block_sparse_attn_natural; an entry outside [0, Nb) raises device error 2 and its
 * tile is skipped.
 */
typedef struct fva_geom {
  int32_t B, H, T, Y, X, d, tt, ty, tx;
  const int32_t* tile_order;
} fva_geom;

enum { FVA_TILES_RASTER = 0, FVA_TILES_HILBERT = 1 };

/*
 * fva_tile_order — host-side table of a tile numbering (§3.1 overview: blocks are
 * reordered along a Hilbert curve so that spatially adjacent tokens fall into nearby
 * blocks).  order_out (HOST, Nb int32) receives the raster index of the tile numbered
 * b.  FVA_TILES_HILBERT: the tile grid (nT, nY, nX) is placed in the smallest
 * power-of-two cube holding it and its tiles are numbered by ascending 3D Hilbert index
 * of (bt, by, bx) in that cube (Skilling's transposed-index construction); the caller
 * copies the table to the device and passes it as g.tile_order.  No GPU work.
 */
int fva_tile_order(fva_geom g, int32_t kind, int32_t* order_out);

/*
 * fva_reorder — video-aware block organisation (abstract; §3.1 overview, block
 * reordering; tiles are 3D boxes numbered in raster order).
 *   x  : bf16 [B,H,N,d] natural order (input).
 *   xr : bf16 [B,H,N,d] tile-major order (output): xr[.., b*S + r, :] = x[.., n(b, r), :].
 * Exact copy.  Requires T%tt == Y%ty == X%tx == 0, d in {64, 128}, x != xr.
 */
int fva_reorder(const void* x, void* xr, fva_geom g, void* stream);

/*
 * fva_inverse_reorder — the inverse permutation of fva_reorder (restores natural
 * token order on the output; §3.1 overview, final stage).  Same constraints.
 */
int fva_inverse_reorder(const void* xr, void* x, fva_geom g, void* stream);

/*
 * fva_reorder_pool — fva_reorder that also writes the routing block means (the pooled
 * Q or K of §3.1) while the tile passes through: the pooling step costs no second read
 * of the tensor.
 *   x, xr  : as in fva_reorder.
 *   pooled : float64 [B,H,Nb,d] output, pooled[b,h,i,:] = mean of the S rows of tile i
 *            (8-byte aligned; 16-byte aligned if it feeds fva_route_repair_pooled).
 * The means are summed in the same order as fva_route's own pooling, so they are
 * bit-identical to what fva_route computes internally.
 */
int fva_reorder_pool(const void* x, void* xr, double* pooled, fva_geom g, void* stream);

/* Workspace bytes fva_route and fva_route_repair need for geometry g: the float64
 * pooled Q and K, then the scratch of the LPT work-list sort (as fva_repair's). */
size_t fva_route_workspace_size(fva_geom g);

/*
 * fva_route — routing frontend (§2 background: block importance and binary mask;
 * Top-p retains the fewest key blocks whose summed normalised importance is >= p;
 * Top-k floor; §3.1 overview: block similarities from pooled Q/K).
 *   qr, kr     : bf16 [B,H,N,d], tile-major (fva_reorder output).
 *   p          : Top-p threshold, 0 < p <= 1 (p >= 1 keeps every block).
 *   k          : Top-k floor, k >= 1 (clamped to Nb).
 *   topp_mask  : uint8 [B,H,Nb,Nb] output, 1 where key block j is in row i's Top-p set.
 *   topk_idx   : int32 [B,H,Nb,min(k,Nb)] output, the min(k,Nb) highest-ranked key
 *                blocks of each row, in ascending block id.
 *   logits_out : optional float64 [B,H,Nb,Nb] output of Qbar_i.Kbar_j/sqrt(d), or NULL.
 * Arithmetic: per-block means and logits in float64; rows ranked by logit descending,
 * ties to the lower block id.  Softmax weights 2^((L - max L) log2 e) in float32,
 * normalised and truncated to 2^-31 fixed point; the running mass is an exact integer
 * sum, so the result is deterministic and the cumulative mass at any cut is within
 * 2.5e-6 of the exact one for Nb <= 640 and within 6e-6 up to Nb = 2048 (a kept set
 * differs from the exact rule only where the cumulative mass at the cut lies that close
 * to p).  Requires Nb <= 2048.
 * Two kernel launches on `stream`: pooling, then scoring and selection.
 */
int fva_route(const void* qr, const void* kr, fva_geom g, double p, int32_t k,
              uint8_t* topp_mask, int32_t* topk_idx, double* logits_out,
              void* workspace, size_t workspace_bytes, void* stream);

/*
 * fva_route_static — fva_route for callers that cannot allocate device memory.
 * The paper has no counterpart: this is a deployment variant of fva_route.
 *
 * Who needs it: code that routes where it may not call cudaMalloc — e.g. a plugin
 * inside a host framework that owns every device allocation and gives plugins no
 * allocator, or a serving loop whose device memory plan is fixed up front, where an
 * allocation (which can synchronise the device or fail under fragmentation) is not
 * acceptable.  Same arguments, results and arithmetic as fva_route, minus the
 * workspace: the routing scratch is one file-scope device array of
 * FVA_ROUTE_STATIC_SCRATCH_BYTES (64 MiB), reserved on every GPU that loads this
 * library and held until the process exits.
 *   - Geometries whose fva_route_workspace_size() exceeds that size are rejected with
 *     FVA_ERR_UNSUPPORTED and a message; nothing is enqueued.  (The 720p layer,
 *     B=1 H=40 d=128 with 600 blocks, needs about 47 MiB; with 64-token tiles, 1200
 *     blocks, it needs about 94 MiB and does not fit.)
 *   - Nothing in the scratch needs to start at zero: each call writes every scratch
 *     byte it later reads.  The array keeps the last call's contents.
 *   - All calls on a device share the one array: calls whose GPU execution overlaps
 *     (different streams, no ordering between them) race and give wrong results.
 *   - The first call on a device looks up the array's device address with that device
 *     current (cudaGetSymbolAddress); make that first call before any stream capture.
 *   - Allocates nothing (no cudaMalloc, cudaFree or allocating library routine).
 */
#define FVA_ROUTE_STATIC_SCRATCH_BYTES ((size_t)64 << 20)
int fva_route_static(const void* qr, const void* kr, fva_geom g, double p, int32_t k,
                     uint8_t* topp_mask, int32_t* topk_idx, double* logits_out, void* stream);

/*
 * fva_route_repair — fva_route followed by fva_repair, fused (same outputs, same
 * arithmetic; the pages describe the two steps, not their split into calls).
 * The per-row repair and compaction run inside fva_route's selection kernel (no
 * mask round trip through memory); three more launches on `stream` build head_work
 * and the LPT work list.
 *   workspace        : fva_route_workspace_size(g) bytes, 256-byte aligned.
 *   topp_mask, topk_idx : as in fva_route, or NULL when the caller does not need them.
 *   counts, idx, head_work, worklist : as in fva_repair (required).
 */
int fva_route_repair(const void* qr, const void* kr, fva_geom g, double p, int32_t k,
                     uint8_t* topp_mask, int32_t* topk_idx, int32_t* counts, int32_t* idx,
                     int64_t* head_work, int32_t* worklist,
                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * fva_route_repair_pooled — fva_route_repair from block means the caller already holds
 * (fva_reorder_pool outputs for Q and K): scoring, Top-p / Top-k selection, repair,
 * W_h and the LPT list, with the same outputs and arithmetic.
 *   qbar, kbar : float64 [B,H,Nb,d], 16-byte aligned.
 *   workspace  : fva_repair_workspace_size(g) bytes, 256-byte aligned (the LPT sort's
 *                per-head histograms; nothing in it needs to start at zero).
 * Four launches: scoring and selection, then the three passes of the LPT sort.
 */
int fva_route_repair_pooled(const double* qbar, const double* kbar, fva_geom g, double p, int32_t k,
                            uint8_t* topp_mask, int32_t* topk_idx, int32_t* counts, int32_t* idx,
                            int64_t* head_work, int32_t* worklist, void* workspace, size_t workspace_bytes,
                            void* stream);

/*
 * fva_route_repair_sasa — fva_route_repair_pooled with slack-aware augmentation, a
 * single-GPU reading of §3.3 (SASA): the heads form num_ranks virtual ranks of
 * H / num_ranks consecutive heads (the head layout of Ulysses sequence parallelism,
 * §2); W_r = kept block pairs of rank r after routing and repair, W* = max_r W_r (the
 * critical path); rank r receives B_r = floor(alpha * (W* - W_r)) extra block pairs,
 * spread round-robin over its rows in item order; a row's ranked prefix (the Top-p set
 * with the floor, following the routing's importance order) grows by its share, capped
 * at Nb, so no rank's workload passes W* and p is unchanged.  Same outputs as
 * fva_route_repair_pooled, computed on the augmented lists.
 *   num_ranks : divides H, 1..1024.     alpha : 0..1 (0: no augmentation).
 *   extra     : optional int32 [B,H,Nb] output, the ranked positions added to each row.
 *   workspace : fva_sasa_workspace_size(g) bytes, 256-byte aligned.
 * Six launches: selection, budgets, selection with the extended floors, the three
 * passes of the LPT sort (its scratch lies in the same workspace).
 */
size_t fva_sasa_workspace_size(fva_geom g);
int fva_route_repair_sasa(const double* qbar, const double* kbar, fva_geom g, double p, int32_t k,
                          int32_t num_ranks, double alpha, int32_t* counts, int32_t* idx,
                          int64_t* head_work, int32_t* worklist, int32_t* extra,
                          void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes fva_repair (and fva_route_repair_pooled) need: B*H*(Nb+1) int32 of
 * per-head count histograms for the LPT sort, rounded up to 256. */
size_t fva_repair_workspace_size(fva_geom g);

/*
 * fva_repair — runtime mask repair and compaction (abstract: the materialised mask
 * is repaired at run time; §2 sequence parallelism: realised per-head workload).
 *   topp_mask, topk_idx, k : fva_route outputs and the same k.
 *   counts    : int32 [B,H,Nb] output, kept key blocks per query block (>= 1).
 *   idx       : int32 [B,H,Nb,Nb] output; row (b,h,i) holds counts[b,h,i] ascending key
 *               block ids in its first entries; entries past the count are not written.
 *   head_work : int64 [B,H] output, W_h = sum over i of counts (kept block pairs).
 *   worklist  : int32 [B*H*Nb] output, item ids u = (b*H + h)*Nb + i ordered by count
 *               descending, ties by u ascending (longest processing time first).
 *   workspace : fva_repair_workspace_size(g) bytes, 256-byte aligned.
 * Kept set of row i = Top-p set U Top-k floor U {i}.  Requires Nb <= 2048.
 * The work list is a stable counting sort by count in three passes (per-head
 * histograms, list offsets, scatter): O(B*H*Nb) work, deterministic.
 */
int fva_repair(const uint8_t* topp_mask, const int32_t* topk_idx, fva_geom g, int32_t k,
               int32_t* counts, int32_t* idx, int64_t* head_work, int32_t* worklist,
               void* workspace, size_t workspace_bytes, void* stream);

/*
 * fva_block_sparse_attn — block-sparse flash attention over the kept pairs (§3.1
 * overview: block-sparse attention after routing; §2: only selected block pairs
 * are evaluated).  Bidirectional, no causal mask.
 *   qr, kr, vr : bf16 [B,H,N,d] tile-major.
 *   counts,idx : fva_repair outputs (every listed id must be in [0, Nb); an id outside
 *                it sets device error 2 and is replaced by the row's own block i).  A
 *                count above Nb is read as Nb; a row with count <= 0 gets all-zero output.
 *   worklist   : fva_repair's LPT order, or NULL for item-id order (an entry outside
 *                [0, B*H*Nb) sets device error 2 and is skipped).
 *   softmax_scale : <= 0 selects 1/sqrt(d).
 *   out_r      : bf16 [B,H,N,d] tile-major output, O_i = softmax(Q_i K_J^T * scale) V_J
 *                over the union J of the kept key blocks of query block i.
 * tcgen05 tensor-core MMAs (bf16 in, fp32 accumulate in TMEM), fp32 online softmax,
 * bf16 round-to-nearest output.  Requires d in {64, 128} and S = tt*ty*tx in {64, 128}.
 * Scheduling: one persistent CTA per SM.  S = 128: CTA c takes list positions c, c + grid,
 * c + 2 grid, ...  S = 64: adjacent query blocks 2p, 2p+1 of a head run as one item over the
 * union of their lists (each row still sees only its own list); the list's entries for odd
 * blocks carry no work, and each CTA claims the next position from a counter private to
 * `stream` (an 8-byte memset on `stream` precedes the kernel), so free CTAs take items in
 * list order (greedy) and all CTAs work through nearby positions at a time.  A process's
 * 64th and later streams on a device share one error word and get no counter: their
 * positions come at the grid stride instead (same results).
 */
int fva_block_sparse_attn(const void* qr, const void* kr, const void* vr,
                          const int32_t* counts, const int32_t* idx, const int32_t* worklist,
                          fva_geom g, float softmax_scale, void* out_r, void* stream);

/*
 * fva_block_sparse_attn_natural — fva_block_sparse_attn writing O in natural token
 * order: the inverse reorder (§3.1, final stage) fused into the epilogue, so the
 * output is written once and not permuted in a second pass.  Same arguments; `out` is
 * bf16 [B,H,N,d] in natural order (bit-identical to fva_inverse_reorder of the
 * tile-major result).
 */
int fva_block_sparse_attn_natural(const void* qr, const void* kr, const void* vr,
                                  const int32_t* counts, const int32_t* idx, const int32_t* worklist,
                                  fva_geom g, float softmax_scale, void* out, void* stream);

/*
 * fva_get_device_error — synchronises `stream`, then reads and clears the device
 * error word of that stream: the word that kernels this library launched on `stream`
 * set when a bounded wait expired (1) or an input index was out of range (2).
 * *code receives the raw word (0 = none).  Each of the first 63 distinct streams used
 * on a device has its own word; any further stream shares one word with the others
 * beyond 63.  Returns FVA_OK, FVA_ERR_TIMEOUT if a wait expired, FVA_ERR_INVALID_ARG
 * for a rejected input, or FVA_ERR_CUDA.
 */
int fva_get_device_error(void* stream, int32_t* code);

/*
 * fva_debug_set_wait_limit — TEST ONLY.  Sets the limit, in SM clock cycles, of every
 * pipeline wait in the attention launches enqueued after this call (process-wide);
 * cycles <= 0 restores the default (about 2 s).  A test sets a limit far below a
 * copy's latency so that a wait expires on purpose: the kernel then aborts, waits
 * for every copy and product it had issued, frees its tensor memory and reports
 * FVA_ERR_TIMEOUT through fva_get_device_error.  Always returns FVA_OK.
 */
int fva_debug_set_wait_limit(int64_t cycles);

/* Thread-local description of the last error returned on this thread ("" if none). */
const char* fva_last_error(void);

/* Number of kernel launches this library has enqueued since load (process-wide). */
int64_t fva_launch_count(void);

/* ABI version (major*100 + minor). */
int32_t fva_version(void);

#ifdef __cplusplus
}
#endif
#endif /* FVA_H */
