/*
 * veda.h -- C ABI of libveda.so: the per-layer hot path of Veda's distilled
 * tile-skipping sparse attention on NVIDIA B200 (sm_100a).
 *
 * Source of the method: "Technical Summary: Veda - Scalable Video Diffusion
 * via Distilled Sparse Attention" (gist.science, arXiv 2605.30325), cited as
 * "Veda summary" with its section. The pages name the steps; layouts, tie
 * rules and padding are this library's readings, stated at each call.
 *
 * Conventions for every call
 *   - Memory: the caller owns every buffer; the library allocates no device
 *     memory. Device pointers must be 16-byte aligned.
 *   - Asynchrony: every call only enqueues kernels on `stream` and returns;
 *     nothing synchronises except veda_check_status.
 *   - Errors: argument errors are detected on the host before any launch and
 *     return VEDA_ERR_INVALID_ARG / VEDA_ERR_UNSUPPORTED with a message in
 *     veda_last_error() (thread-local). Launch failures return VEDA_ERR_CUDA.
 *     Kernels never trap: a device-side error (a wait that exceeded its time
 *     limit, an index outside its range) is written to layer->dev_status and
 *     read back by veda_check_status.
 *   - Layouts (row-major, contiguous):
 *       original tokens  x   [B, N, heads, d] bf16, N = T*H*W,
 *                            token n = (t*H + y)*W + x
 *       permuted tokens  xp  [B, heads, n_cap, d] bf16 (per-head tile order)
 *       descriptors      desc[B, heads, nt_cap, 3d] fp32 ([avg | max | min])
 *       tile scores          [B, heads, nt_cap, nt_cap] fp32
 *       key-tile lists   idx [B, heads, nt_cap, k_cap] int32 (ascending, -1 pad)
 *       tile mask        mask[B, heads, nt_cap, nt_cap] uint8 (0/1)
 *     Rows/columns of a head beyond its own tile count (nt_h <= i < nt_cap)
 *     and padding slots are written as zeros (-1 in idx).
 */
#ifndef VEDA_H
#define VEDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* cudaStream_t;

typedef enum {
  VEDA_OK = 0,
  VEDA_ERR_INVALID_ARG = -1,  /* bad sizes, pointers, tilings (host check) */
  VEDA_ERR_UNSUPPORTED = -2,  /* valid but outside this build's limits      */
  VEDA_ERR_CUDA = -3,         /* a CUDA runtime/driver call failed          */
  VEDA_ERR_TIMEOUT = -4,      /* device: a pipeline wait exceeded its limit */
  VEDA_ERR_BAD_INDEX = -5     /* device: a tile index outside [0, nt_h)     */
} veda_status;

/* A head's tiling pi_{l,h} = (p_t, p_h, p_w): a factorisation of the tile
 * size into time, height and width extents (Veda summary 2.2). */
typedef struct {
  int32_t pt, ph, pw;
} veda_tiling;

/* One attention layer's geometry.
 *   B, heads   batch and head count (heads <= 128)
 *   d          head dimension, 64 or 128
 *   T, H, W    latent token grid (N = T*H*W tokens)
 *   tile       tokens per tile, 64 or 128; tilings[h].pt*ph*pw == tile
 *   tilings    HOST array [heads], read during each call only
 *   dev_status DEVICE int32 owned by the caller, zero before first use;
 *              kernels store a veda_status code here instead of trapping.
 * Padding (a reading; the pages give no rule): p_h | H and p_w | W are
 * required; T is padded at its end to a multiple of p_t. Tiles are numbered
 * row-major over (t/p_t, y/p_h, x/p_w) and tokens inside a tile row-major
 * over (t%p_t, y%p_h, x%p_w), so each tile's valid tokens are a prefix of
 * length min(p_t, T - t0)*p_h*p_w. */
typedef struct {
  int32_t B, heads, d, T, H, W, tile;
  const veda_tiling* tilings;
  int32_t* dev_status;
} veda_layer;

/* Host-only geometry of a layer (no CUDA call). Writes nt[h] (tiles of head
 * h), n_pad[h] = nt[h]*tile, *n_cap = max n_pad, *nt_cap = max nt. Any output
 * pointer may be NULL. Returns VEDA_ERR_INVALID_ARG for a bad tiling. */
int veda_layout(const veda_layer* L, int32_t* nt, int32_t* n_pad, int32_t* n_cap,
                int32_t* nt_cap);

/* Head-aware tiling permutation (Veda summary 2.2, Head-Aware Tiling).
 * inverse = 0: x [B,N,heads,d] -> xp [B,heads,n_cap,d]; slot s of head h
 *   receives token perm_h[s]; padding slots are zero. If `perm` is not NULL
 *   it receives the index map [heads, n_cap] int32 (original token, or -1).
 * inverse = 1: xp -> x, the inverse gather; padding rows are dropped.
 *   `perm` is ignored. */
int veda_permute(const veda_layer* L, const void* x, void* xp, int32_t* perm,
                 int inverse, cudaStream_t stream);

/* TripPool descriptors (Veda summary 2.1, Statistic-Aware Estimator): for
 * each tile and channel, [mean | max | min] over the tile's valid tokens.
 * xp [B,heads,n_cap,d] bf16 -> desc [B,heads,nt_cap,3d] fp32. */
int veda_trippool(const veda_layer* L, const void* xp, float* desc, cudaStream_t stream);

/* The forward permutation and TripPool in one pass (Veda summary 2.1 and
 * 2.2; the pages name tighter kernel fusion as future work): x -> xp and
 * perm exactly as veda_permute(..., inverse = 0), and desc [B,heads,nt_cap,
 * 3d] fp32 as veda_trippool would compute from xp, without reading xp back.
 * max/min are bit-identical to veda_trippool; the mean sums the same values
 * in another order (fp32 rounding). `perm` may be NULL. All pointers are
 * caller-owned device memory, 16-byte aligned. */
int veda_permute_trippool(const veda_layer* L, const void* x, void* xp, int32_t* perm, float* desc,
                          cudaStream_t stream);

/* Head-specific MLP estimator and tile scores (Veda summary 2.1,
 * Head-Specific Projections): per head h,
 *   q_i = W2q^T GELU(W1q^T dq_i + b1q) + b2q,  k_j likewise with the k weights,
 *   scores[i, j] = scale * q_i . k_j          (i, j < nt_h), fp32 FFMA.
 * GELU is the exact erf form. Weights fp32: w1 [heads, 3d, hidden],
 * b1 [heads, hidden], w2 [heads, hidden, out_dim], b2 [heads, out_dim];
 * hidden <= 256 and out_dim <= 128, both multiples of 4. emb_ws is caller scratch
 * of veda_tile_scores_ws_bytes() bytes (the q and k embeddings). */
int veda_tile_scores(const veda_layer* L, const float* dq, const float* dk,
                     const float* w1q, const float* b1q, const float* w2q, const float* b2q,
                     const float* w1k, const float* b1k, const float* w2k, const float* b2k,
                     int32_t hidden, int32_t out_dim, float scale, float* scores,
                     float* emb_ws, cudaStream_t stream);
size_t veda_tile_scores_ws_bytes(const veda_layer* L, int32_t out_dim);

/* veda_tile_scores without a scratch argument, for callers that may not
 * allocate device memory: applications that load this library as a plug-in
 * and own every byte of device memory in a pre-planned pool, and real-time
 * loops that must not call an allocator between frames. The pages describe
 * no such call; it is a deployment variant of the call above with identical
 * results. The embeddings live in a device array built into the library
 * (16 MiB, held by every GPU that loads the library until the process
 * exits); a layer needing more (veda_tile_scores_ws_bytes > 16 MiB) is
 * rejected with VEDA_ERR_UNSUPPORTED. The first call on each device looks up
 * that device's copy of the array with cudaGetSymbolAddress; with CUDA's
 * lazy module loading this is also when the driver loads the library's
 * device code on that device and so reserves the array, which can fail
 * (VEDA_ERR_CUDA) if the device has no room left. Make that first call once
 * per device at initialisation, before any stream capture and outside
 * per-frame loops; later calls reserve nothing. The looked-up address is kept
 * for the life of the process, so the call is not supported across a
 * cudaDeviceReset. All calls share the array: calls whose kernels may overlap
 * on the GPU race and must be serialised by the caller. The call itself
 * allocates no device memory. */
int veda_tile_scores_noalloc(const veda_layer* L, const float* dq, const float* dk,
                             const float* w1q, const float* b1q, const float* w2q, const float* b2q,
                             const float* w1k, const float* b1k, const float* w2k, const float* b2k,
                             int32_t hidden, int32_t out_dim, float scale, float* scores,
                             cudaStream_t stream);

/* Top-k key tiles per query tile (Veda summary 2.1 and 4: only the highest
 * scoring key tiles are kept). k: HOST array [heads], 1 <= k[h] <= nt_h,
 * k[h] <= k_cap. Ranking is on the fp32 value; exact ties (and -0.0 vs +0.0)
 * go to the lower tile index. idx rows are ascending and -1 padded to k_cap;
 * `mask` (may be NULL) is the dense 0/1 form. */
int veda_topk_mask(const veda_layer* L, const float* scores, const int32_t* k, int32_t k_cap,
                   int32_t* idx, uint8_t* mask, cudaStream_t stream);

/* Tile scores and the top-k mask in one call (Veda summary 2.1; the pages
 * name tighter kernel fusion as future work): the per-head MLP of
 * veda_tile_scores into emb_ws, then one kernel that builds whole score rows
 * in shared memory and selects from them, so the score matrix need not go
 * through HBM. Arguments as in veda_tile_scores and veda_topk_mask; `scores`
 * may be NULL (then it is not written) or receive the same matrix
 * veda_tile_scores writes. idx, mask and scores are bit-identical to
 * veda_tile_scores followed by veda_topk_mask. A score row must fit shared
 * memory (4*nt_cap + 4*out_dim + 8192 <= 204800 bytes, true for every layer
 * the library accepts), else VEDA_ERR_UNSUPPORTED. Measured slower than the
 * two separate calls on the 153,600-token layer (1.07 vs 0.85 ms). */
int veda_tile_scores_topk(const veda_layer* L, const float* dq, const float* dk,
                          const float* w1q, const float* b1q, const float* w2q, const float* b2q,
                          const float* w1k, const float* b1k, const float* w2k, const float* b2k,
                          int32_t hidden, int32_t out_dim, float scale, const int32_t* k, int32_t k_cap,
                          int32_t* idx, uint8_t* mask, float* scores, float* emb_ws, cudaStream_t stream);

/* Tile-skipping sparse attention (Veda summary 2.3): for each query row i of
 * query tile a, O_i = sum_j softmax_j(scale * q_i . k_j) v_j over the valid
 * keys j of the key tiles idx[a, 0..k[h]) only; the softmax is renormalised
 * over those keys and the other tiles are never read. idx == NULL runs the
 * dense path (every tile kept; k and k_cap ignored). qp/kp/vp/op are
 * [B,heads,n_cap,d] bf16; lse (may be NULL) [B,heads,n_cap] fp32 receives
 * the natural-log softmax normaliser. Padding rows of op are zero.
 * Tensor cores: tcgen05.mma (bf16 in, fp32 accumulate in TMEM); K/V tiles
 * arrive by TMA. */
int veda_sparse_attn(const veda_layer* L, const void* qp, const void* kp, const void* vp,
                     const int32_t* idx, const int32_t* k, int32_t k_cap, float scale,
                     void* op, float* lse, cudaStream_t stream);

/* veda_sparse_attn followed by the inverse permutation (Veda summary 2.2: the
 * output returns to token order), in one kernel: each output row is written
 * straight to its token, so the permuted output is never stored and read
 * back (the pages name tighter kernel fusion as future work). o: [B, N, heads,
 * d] bf16, N = T*H*W, every row written; identical values to veda_sparse_attn
 * followed by veda_permute(..., inverse=1). lse (may be NULL) keeps the
 * permuted layout [B, heads, n_cap] of veda_sparse_attn. Other arguments and
 * errors as in veda_sparse_attn. */
int veda_sparse_attn_unpermute(const veda_layer* L, const void* qp, const void* kp, const void* vp,
                               const int32_t* idx, const int32_t* k, int32_t k_cap, float scale,
                               void* o, float* lse, cudaStream_t stream);

/* Tile-skipping sparse attention with no permuted copies at all (Veda summary
 * 2.2 and 2.3): q, k, v and o are in token order [B, N, heads, d] bf16. Each
 * tile of the head-aware tiling is gathered by TMA straight from token order
 * (one 5D tensor map per distinct tiling, whose box is the tile's rows in the
 * tiling's in-tile order), and each output row is written to its token. The
 * values equal those of veda_permute on q, k, v, veda_sparse_attn and the
 * inverse veda_permute. idx, k, k_cap, scale as in veda_sparse_attn; lse (may
 * be NULL) has the permuted layout [B, heads, n_cap]. At most 8 distinct
 * tilings per layer (VEDA_ERR_UNSUPPORTED beyond). */
int veda_sparse_attn_tokens(const veda_layer* L, const void* q, const void* k_in, const void* v,
                            const int32_t* idx, const int32_t* k, int32_t k_cap, float scale,
                            void* o, float* lse, cudaStream_t stream);

/* Temporal caching of tile scores across diffusion steps (Veda summary 5
 * names temporal caching of tile scores and adaptive sparsity across
 * timesteps as future work; this rule is the library's reading). For every
 * (batch element, head) bh: with D = the step's TripPool descriptors dq, dk
 * and R = dq_ref, dk_ref (the descriptors of the step whose scores are
 * cached), drift^2 = (|Dq-Rq|^2 + |Dk-Rk|^2) / (|Rq|^2 + |Rk|^2) over the
 * head's valid tiles, summed in fp64 in a fixed order. refresh[bh] = 1 when
 * age[bh] < 0 (never scored), age[bh] + 1 >= max_age, or drift^2 > tau^2;
 * then age[bh] = 0 and R takes D; else refresh[bh] = 0 and age[bh] += 1.
 * dq/dk/dq_ref/dk_ref: [B, heads, nt_cap, 3d] fp32 device; age, refresh:
 * [B*heads] int32 device (initialise age to -1). tau >= 0, max_age >= 1
 * (1 = refresh every step). ws: veda_score_cache_ws_bytes(L) bytes of device
 * scratch (the per-chunk partial sums). Feed `refresh` to
 * veda_tile_scores_heads and veda_topk_mask_heads: heads with 0 keep their
 * scores, idx and mask. */
size_t veda_score_cache_ws_bytes(const veda_layer* L);
int veda_score_cache_step(const veda_layer* L, const float* dq, const float* dk, float* dq_ref, float* dk_ref,
                          float tau, int32_t max_age, int32_t* age, int32_t* refresh, void* ws,
                          cudaStream_t stream);

/* veda_tile_scores and veda_topk_mask restricted to the (batch element,
 * head) pairs with head_on[b*heads + h] != 0 (device int32 [B*heads], may be
 * NULL = all): the other heads' scores, emb_ws rows, idx and mask are left as
 * they are. */
int veda_tile_scores_heads(const veda_layer* L, const float* dq, const float* dk,
                           const float* w1q, const float* b1q, const float* w2q, const float* b2q,
                           const float* w1k, const float* b1k, const float* w2k, const float* b2k,
                           int32_t hidden, int32_t out_dim, float scale, float* scores,
                           float* emb_ws, const int32_t* head_on, cudaStream_t stream);
int veda_topk_mask_heads(const veda_layer* L, const float* scores, const int32_t* k, int32_t k_cap,
                         int32_t* idx, uint8_t* mask, const int32_t* head_on, cudaStream_t stream);

/* Oracle tile map and distillation loss (Veda summary 2.1, Target
 * Construction and Optimization; 2.3, Training Efficiency): for the selected
 * heads heads_sel[0..n_heads_sel) (HOST array) and query tiles
 * qtile_rows [n_heads_sel, n_rows] (DEVICE int32; NULL = tiles 0..n_rows-1),
 *   pass 1: lse_i = log sum_j exp(scale q_i . k_j) over all valid keys;
 *   pass 2: tilemap[s, r, b] = max over valid rows i of the tile and valid
 *           keys j of key tile b of exp(scale q_i . k_j - lse_i),
 * i.e. max-pooling of the full softmax attention matrix over the tile region.
 * tilemap [n_heads_sel, n_rows, nt_cap] fp32 (zero beyond nt_h); lse (may be
 * NULL) [n_heads_sel, n_rows, tile] fp32. If `scores` (the [B=1 batch slice
 * of] veda_tile_scores output) is not NULL, kl_rows [n_heads_sel, n_rows]
 * receives KL(t || softmax(scores row)) with t the tile-map row normalised to
 * sum 1, and *kl_out (device fp32) their mean over rows, then heads.
 * ws (may be NULL): veda_full_attn_tilemax_ws_bytes(...) bytes of device
 * scratch (partial sums, and every selected row's largest logit per key tile:
 * 4 * n_heads_sel * n_rows * tile * nt_cap bytes of it). With it the logits
 * are computed once instead of twice: one sweep, whose key range may be
 * split over several CTAs so that small maps fill every SM, stores partial
 * sums and row maxima; a second kernel combines the sums in a fixed order and
 * reduces the maxima. Without it each CTA sweeps its keys twice. Results are
 * the same up to fp32 rounding of the log-sum-exp. Only B == 1 layers are
 * accepted. */
size_t veda_full_attn_tilemax_ws_bytes(const veda_layer* L, int32_t n_heads_sel, int32_t n_rows);
int veda_full_attn_tilemax(const veda_layer* L, const void* qp, const void* kp,
                           const int32_t* heads_sel, int32_t n_heads_sel,
                           const int32_t* qtile_rows, int32_t n_rows, float scale,
                           float* tilemap, float* lse, const float* scores,
                           float* kl_rows, float* kl_out, float* ws, cudaStream_t stream);

/* The row-wise KL of veda_full_attn_tilemax for a map already built (Veda
 * summary 2.1, Optimization): kl_rows [n_heads_sel, n_rows] and *kl_out, as
 * that call computes them when given `scores`. Lets a caller build the map on
 * one stream, concurrently with the score and top-k calls, and take the KL
 * once both are done. Arguments as in veda_full_attn_tilemax. */
int veda_tilemap_kl(const veda_layer* L, const int32_t* heads_sel, int32_t n_heads_sel,
                    const int32_t* qtile_rows, int32_t n_rows, const float* tilemap,
                    const float* scores, float* kl_rows, float* kl_out, cudaStream_t stream);

/* Recall of the predicted key-tile lists against the tile map (Veda summary
 * 2.1, Target Construction: the max-pooled full-attention map is the target
 * the estimator is aligned to; Veda summary 1 and 4 judge the kept tiles by
 * how much of the attention they hold). For the selected heads heads_sel
 * (HOST array) and query tiles qtile_rows [n_heads_sel, n_rows] (DEVICE
 * int32; NULL = tiles 0..n_rows-1), with tilemap the output of
 * veda_full_attn_tilemax for the same heads and rows:
 *   map top-k: the k[h] tiles of the map row ranked exactly as
 *              veda_topk_mask ranks a score row (fp32 value, exact ties and
 *              -0.0/+0.0 to the lower tile index);
 *   hits[s, r] = |set(idx[0, h, a, 0..k[h])) & map top-k|, a = the query tile;
 *   recall[s]  = sum_r hits[s, r] / (n_rows * k[h]);
 *   recall[n_heads_sel] = the mean of recall[0..n_heads_sel) in head order.
 * idx: the predicted lists [1, heads, nt_cap, k_cap] int32 (veda_topk_mask
 * output); k: HOST array [heads] as given to veda_topk_mask. hits
 * [n_heads_sel, n_rows] int32 and recall [n_heads_sel + 1] fp32 are DEVICE
 * outputs; map_idx (may be NULL) [n_heads_sel, n_rows, k_cap] int32 receives
 * the map's own top-k lists (ascending, -1 padded). A query tile outside its
 * head or a predicted entry outside [0, nt_h) is reported as
 * VEDA_ERR_BAD_INDEX in dev_status (that row then counts the valid entries
 * only). Only B == 1 layers are accepted. */
int veda_tilemap_recall(const veda_layer* L, const int32_t* heads_sel, int32_t n_heads_sel,
                        const int32_t* qtile_rows, int32_t n_rows, const float* tilemap, const int32_t* idx,
                        const int32_t* k, int32_t k_cap, int32_t* hits, int32_t* map_idx, float* recall,
                        cudaStream_t stream);

/* Estimator training (Veda summary 2.1, Optimization: the head-specific
 * projections are trained with the row-wise KL against the tile map, with
 * stop-gradient on the pooled descriptors; 2.3, Training Efficiency: on
 * random subsets of query tiles). For the selected heads heads_sel (HOST,
 * distinct) and their sampled query tiles qtile_rows [n_heads_sel, n_rows]
 * (DEVICE; NULL = tiles 0..n_rows-1), with tilemap the output of
 * veda_full_attn_tilemax for the same heads and rows, computes
 *   loss = mean over heads of mean over rows of KL(t || softmax(s_row)),
 *   s_row[j] = scale * MLP_q(dq[row]) . MLP_k(dk[j]) over the head's tiles,
 * and writes its gradient with respect to every weight array into g_* (same
 * shapes as the weights: g_w1q [heads,3d,hidden], g_b1q [heads,hidden],
 * g_w2q [heads,hidden,out_dim], g_b2q [heads,out_dim], and the key side);
 * heads not selected get zeros. Query and key weights get separate
 * gradients (sum them when one MLP serves both). *loss (device fp32, may be
 * NULL) receives the loss. Scores are recomputed in fp32 from the weights
 * given. ws: veda_estimator_grad_ws_bytes(...) bytes of device scratch.
 * fp32 arithmetic; every reduction in a fixed order (bit-reproducible).
 * Only B == 1 layers are accepted. */
size_t veda_estimator_grad_ws_bytes(const veda_layer* L, int32_t n_heads_sel, int32_t n_rows,
                                    int32_t hidden, int32_t out_dim);
int veda_estimator_grad(const veda_layer* L, const float* dq, const float* dk,
                        const float* w1q, const float* b1q, const float* w2q, const float* b2q,
                        const float* w1k, const float* b1k, const float* w2k, const float* b2k,
                        int32_t hidden, int32_t out_dim, float scale,
                        const int32_t* heads_sel, int32_t n_heads_sel,
                        const int32_t* qtile_rows, int32_t n_rows, const float* tilemap,
                        float* g_w1q, float* g_b1q, float* g_w2q, float* g_b2q,
                        float* g_w1k, float* g_b1k, float* g_w2k, float* g_b2k,
                        float* loss, float* ws, cudaStream_t stream);

/* Calibration metric of the head-aware tiling search (Veda summary 2.2:
 * tilings are chosen per head, offline, to fit each head's locality):
 * err[h] (device fp32 [heads]) = sum over batch, tokens and channels of
 * (a - b)^2 for head h, with a and b [B,N,heads,d] bf16 attention outputs in
 * the original token order (e.g. full attention and the tile-skipping
 * output under one candidate tiling). Fixed-order reduction. */
int veda_output_sq_error(const veda_layer* L, const void* a, const void* b, float* err, cudaStream_t stream);

/* Diagnostic (no counterpart on the pages): launches one thread that waits,
 * through the bounded wait every pipeline kernel uses, on a barrier nothing
 * arrives on. After limit_ms (1..10000) the wait gives up and records
 * VEDA_ERR_TIMEOUT in L->dev_status; the kernel then returns normally, so a
 * following veda_check_status reports the timeout and the context remains
 * usable. Lets callers verify the failure path without faulting a GPU. */
int veda_selftest_wait_timeout(const veda_layer* L, uint32_t limit_ms, cudaStream_t stream);

/* Synchronises `stream`, returns the first device-side status recorded in
 * L->dev_status (VEDA_OK if none) and clears it. */
int veda_check_status(const veda_layer* L, cudaStream_t stream);

/* Message of the last failing call on this thread ("" if none). */
const char* veda_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* VEDA_H */
