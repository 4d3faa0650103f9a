/*
 * sparse_attn.h — C ABI of libsparse_attn.so: content-adaptive block-sparse
 * self-attention over spatio-temporal video tokens, in the form of
 * "NABLA - Neighborhood Adaptive Block-Level Attention per la Generazione
 * Efficiente di Video" (gist.science/it/paper/2507.13546), section
 * "Metodologia: NABLA".
 *
 * The path is split in two calls:
 *   sparse_attn_plan  fractal flattening (as addressing) + block pooling of Q
 *                     and K + reduced attention map + per-row CDF threshold
 *                     + optional STA union  ->  block lists in a workspace;
 *   sparse_attn_fwd   exact attention over the kept (q-block, k-block) pairs,
 *                     written back in natural token order.
 * One plan may serve many fwd calls with the same Q/K statistics. Around
 * them: the gradients over the same mask (sparse_attn_fwd_lse,
 * sparse_attn_bwd), the exact block max-pooled attention map that measures a
 * mask's recall (sparse_attn_block_heatmap), per-head block shapes (*_heads),
 * and the whole path as one CUDA graph launch (sparse_attn_graph_*).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     allocates nothing and keeps no state between calls, except the graph
 *     object of sparse_attn_graph_create (owned by the caller until
 *     sparse_attn_graph_destroy) and the built-in workspace of
 *     sparse_attn_forward_noalloc.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream). Argument errors are reported before anything is launched.
 *   - Q, K, V and the output use the natural video layout [B, H, S, d] with
 *     S = T*Hh*Ww tokens ordered (t, h, w), t outermost, d innermost,
 *     contiguous, bf16 (raw 16-bit storage), 16-byte aligned.
 *   - Device-side failures (a bounded wait that ran out, an out-of-range block
 *     index) are recorded in a status word inside the workspace and reported
 *     by sparse_attn_check. No kernel of this library traps.
 */
#ifndef SPARSE_ATTN_H
#define SPARSE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Problem description. The method's parameters follow the NABLA page:
 * P is the spatial patch edge of "Fractal Flattening" (Metodologia 1), N the
 * block length of "Sottocampionamento" and the N x N attention-map block
 * (Metodologia 2), thr the "CDF Thresholding" parameter (Metodologia 2), and
 * (sta_t, sta_h, sta_w) the static window of "Integrazione Ibrida con STA"
 * (Metodologia 3), in block units. */
typedef struct sa_desc {
  int B, H;          /* batch, heads */
  int T, Hh, Ww;     /* latent grid: frames, height, width (S = T*Hh*Ww) */
  int d;             /* head dimension: 64 or 128 */
  int N, P;          /* block tokens and patch edge; requires N == P*P = 64,
                        Hh % P == 0 and Ww % P == 0 */
  float thr;         /* [0, 1): keep the smallest descending-probability set
                        of k-blocks whose mass reaches 1 - thr; 0 = dense */
  int sta_t, sta_h, sta_w; /* odd STA window in blocks, or 0,0,0 = no STA */
  int out_fp32;      /* 0: output bf16; 1: output fp32 (same layout) */
  int debug_flags;   /* 0 in normal use; SA_DEBUG_* bits for tests */
  int pt, ph, pw;    /* block shape: 0,0,0 = the P x P patch of one frame
                        (1, P, P); otherwise a three-dimensional tile of pt
                        frames x ph rows x pw columns with pt*ph*pw == N, T % pt,
                        Hh % ph and Ww % pw all 0 (the head-aware tiling of
                        "Veda - Diffusione Video Scalabile tramite
                        Attenzione Sparsa Distillata", section 2.2); P is then not used. Block
                        coordinates, tile pairing and the STA window are in
                        units of these tiles. */
} sa_desc;

/* Test-only: the attention kernel's loader never signals its first K/V
 * stage, so the compute warps' bounded wait runs out and the call reports
 * SA_ERR_DEVICE_TIMEOUT from sparse_attn_check (no fault, no hang). */
#define SA_DEBUG_STALL_LOADER 1

typedef enum sa_status {
  SA_OK = 0,
  SA_ERR_INVALID_ARG = 1,     /* NULL pointer, non-positive size, thr out of
                                 range, even STA window, misaligned pointer */
  SA_ERR_UNSUPPORTED = 2,     /* valid but not implemented: d not in {64,128},
                                 N != 64, block shape not N tokens, grid not
                                 divisible by the block shape, more than 6144
                                 blocks per head, B*H above 65535 */
  SA_ERR_WORKSPACE = 3,       /* workspace smaller than
                                 sparse_attn_workspace_size() */
  SA_ERR_CUDA = 4,            /* a CUDA runtime call or launch failed */
  SA_ERR_DEVICE_TIMEOUT = 5   /* a kernel's bounded wait ran out */
} sa_status;

/* Bytes of device workspace a plan for `desc` needs (written to *bytes). */
sa_status sparse_attn_workspace_size(const sa_desc* desc, size_t* bytes);

/* Builds the block mask M = M_nabla OR M_STA for every (batch, head):
 *   1. fractal flattening: block b of a head is the P x P patch (hp, wp) of
 *      frame t, b = (t*(Hh/P) + hp)*(Ww/P) + wp, tokens row-major inside it
 *      (NABLA, Metodologia 1); with a tile shape (pt, ph, pw) block
 *      b = (tb*(Hh/ph) + hb)*(Ww/pw) + wb holds frames tb*pt.., rows hb*ph..,
 *      columns wb*pw.., tokens in (t, h, w) row-major order inside it;
 *   2. Qbar, Kbar = mean of the N tokens of each block, fp32 (Metodologia 2,
 *      "Sottocampionamento");
 *   3. A = row softmax(Qbar Kbar^T / sqrt(d)) (Metodologia 2, "Attenzione
 *      Ridotta"); the scaled logits are written to the workspace (fp32,
 *      nb x nb per head) and read back once by the threshold step, which
 *      needs a whole row at a time;
 *   4. per row, k-block j is kept iff the mass of the blocks ranked before it
 *      (descending probability, ties by ascending index) is below 1 - thr
 *      (Metodologia 2, "CDF Thresholding"); thr == 0 keeps every block;
 *   5. union with the STA window |dt|<=sta_t/2, |dhp|<=sta_h/2, |dwp|<=sta_w/2
 *      (Metodologia 3).
 * q, k: [B,H,S,d] bf16 device tensors in natural order. workspace: device
 * buffer of at least sparse_attn_workspace_size() bytes, 256-byte aligned;
 * its previous contents are ignored and overwritten. */
sa_status sparse_attn_plan(const sa_desc* desc, const void* q, const void* k,
                           void* workspace, size_t ws_bytes, void* stream);

/* Diagnostics for measuring the plan's kernels. Runs sparse_attn_plan `reps`
 * times on `stream` with CUDA events between its stages (the pages define no
 * such split; it follows the steps listed above: pooling, reduced map, CDF
 * threshold with the STA union, per-tile union lists, tile order), waits for
 * each run, and writes every stage's mean device time in microseconds to
 * stage_us[0 .. *n_stages - 1]. max_stages: the length of stage_us (at least
 * the stage count, else SA_ERR_INVALID_ARG). Blocks the calling thread;
 * creates and destroys its own events; not for stream capture.
 * sparse_attn_plan_stage_name(i) names stage i (NULL outside the range). */
sa_status sparse_attn_plan_profile(const sa_desc* desc, const void* q, const void* k,
                                   void* workspace, size_t ws_bytes, int reps,
                                   float* stage_us, int max_stages, int* n_stages,
                                   void* stream);
const char* sparse_attn_plan_stage_name(int i);

/* O_i = sum over kept k-blocks of softmax(q_i . k_j / sqrt(d)) v_j for every
 * query token i, i.e. exact attention with every dropped N x N block at -inf
 * ("Espansione", NABLA Metodologia 2), written to `out` [B,H,S,d] in natural
 * token order (bf16, or fp32 if desc->out_fp32). q, k, v as for the plan; the
 * workspace must hold a plan made for the same desc (q, k may differ from the
 * plan's, e.g. when a plan is reused across steps). */
sa_status sparse_attn_fwd(const sa_desc* desc, const void* q, const void* k,
                          const void* v, const void* workspace, size_t ws_bytes,
                          void* out, void* stream);

/* Fractal flattening of one [B,H,S,d] bf16 tensor (inverse = 0: natural ->
 * fractal order, position p of a head holds token perm[p]) or its inverse
 * (inverse = 1). x and y must not overlap. The attention path itself reads
 * the natural layout through TMA addressing and does not call this. */
sa_status sparse_attn_permute(const sa_desc* desc, const void* x, void* y,
                              int inverse, void* stream);

/* Device views into a planned workspace (pointers into `workspace`; valid as
 * long as it is). Block indices are in fractal block order. */
typedef struct sa_mask_views {
  const float* qbar;     /* [B*H][nb][d] pooled queries */
  const float* kbar;     /* [B*H][nb][d] pooled keys */
  const int32_t* cnt;    /* [B*H][nb] kept k-blocks per q-block */
  const int32_t* idx;    /* [B*H][nb][nb] kept k-block ids, ascending, first
                            cnt entries valid */
  const int32_t* tile_cnt;  /* [B*H][ntile] union length per query tile */
  const int32_t* tile_idx;  /* [B*H][ntile][nb] union entries: k-block id in
                               bits 0-15, bit 16 = first q-block keeps it,
                               bit 17 = second q-block keeps it, bit 18 set on
                               the first entry of each leading pair of entries
                               that are one patch in frames t and t+1 (these
                               pairs come first, then the other blocks in
                               ascending order) */
  int nb;                /* blocks per head */
  int ntile;             /* query tiles per head (pairs of q-blocks) */
  const float* logits;   /* [B*H][nb][logits_ld] the reduced map's scaled
                            logits Qbar Kbar^T / sqrt(d) as the plan computed
                            them (fp32, before the row softmax); the first nb
                            of each row are valid */
  int logits_ld;         /* row pitch of logits, in floats */
} sa_mask_views;

sa_status sparse_attn_get_mask(const sa_desc* desc, const void* workspace,
                               size_t ws_bytes, sa_mask_views* views);

/* Query tile -> its two q-blocks (second = -1 for a lone block). Tiles pair
 * block (t, hp, wp) with (t+1, hp, wp) for even t; with an odd T the last
 * frame pairs (hp, wp) with (hp, wp+1). */
sa_status sparse_attn_tile_blocks(const sa_desc* desc, int tile, int* qa, int* qb);

/* Waits for `stream`, then reports SA_ERR_DEVICE_TIMEOUT if a kernel of the
 * last plan/fwd on this workspace recorded a device-side failure, SA_ERR_CUDA
 * if the stream holds a CUDA error, else SA_OK. */
sa_status sparse_attn_check(const sa_desc* desc, const void* workspace,
                            size_t ws_bytes, void* stream);

/* Static, NUL-terminated description of a status code. */
const char* sparse_attn_status_string(sa_status status);

/* Bytes of the workspace built into the library for
 * sparse_attn_forward_noalloc (64 MiB). */
#define SA_NOALLOC_SCRATCH_BYTES (64u << 20)

/* Plan + forward without a caller-provided workspace. (No counterpart in the
 * NABLA paper: this exists for the library's users, not for the method.)
 *
 * Some callers cannot allocate device memory on their own: a runtime that
 * owns every byte of GPU memory and hands out only what it planned at start-up,
 * code on a latency-critical path where cudaMalloc's implicit synchronisation
 * is not acceptable, or a host program that simply has no allocator for the
 * device. This call lets them run the whole path with only their own q, k, v
 * and out buffers: the workspace is a fixed SA_NOALLOC_SCRATCH_BYTES array in
 * the library's device image (each GPU that loads the library holds one copy
 * until the process exits). The call allocates nothing.
 *
 * q, k, v, out, stream and desc are as for sparse_attn_plan/sparse_attn_fwd.
 * Returns SA_ERR_WORKSPACE, before launching anything, when the problem's
 * workspace (sparse_attn_workspace_size) is larger than the built-in array.
 *
 * - Every call made outside stream capture looks the array's device address
 *   up (with the call's device current), so a device reset, which reloads
 *   the library's device image, is followed safely. A call made while its
 *   stream is being captured cannot look it up: it uses the address the last
 *   uncaptured call on that device found, so make one uncaptured call on the
 *   device first (and again after any device reset); otherwise it returns
 *   SA_ERR_CUDA.
 * - All calls on a device share the one array, which keeps the previous
 *   call's contents (the plan rewrites everything it later reads). Calls whose
 *   work may overlap on the GPU (different streams, or several threads)
 *   race on it: serialise them.
 * - Device-side status (a bounded wait that ran out) lands in the shared
 *   array and is not reported by this call; use the workspace entry points
 *   with sparse_attn_check when that status matters. */
sa_status sparse_attn_forward_noalloc(const sa_desc* desc, const void* q,
                                      const void* k, const void* v, void* out,
                                      void* stream);

/* ---- Per-head block shapes ------------------------------------------------
 * The head-aware tiling of "Veda - Diffusione Video Scalabile tramite
 * Attenzione Sparsa Distillata" (gist.science/it/paper/2605.30325, section
 * 2.2, "Tiling Consapevole delle Teste"): each head may
 * use its own block shape. tiles is a HOST array of B*H triples
 * (pt, ph, pw), in (batch, head) order; each must satisfy the single-shape
 * rules of sa_desc (pt*ph*pw == N, the grid divisible by it; 0,0,0 = the
 * P x P patch). desc->pt/ph/pw are ignored. Consecutive heads with equal
 * triples form a run, which is planned and run as one problem with H = run
 * length on its slice of q, k, v, out (a head's [S, d] rows are contiguous)
 * and its own 256-byte-aligned slice of the workspace, so results equal
 * separate single-shape calls head by head. Errors: those of the
 * single-shape calls, for the first run that fails; a NULL tiles is
 * SA_ERR_INVALID_ARG. */

/* Workspace bytes for all runs together. */
sa_status sparse_attn_workspace_size_heads(const sa_desc* desc, const int* tiles, size_t* bytes);

/* sparse_attn_plan for every run (q, k: the full [B, H, S, d] tensors). */
sa_status sparse_attn_plan_heads(const sa_desc* desc, const int* tiles, const void* q,
                                 const void* k, void* workspace, size_t ws_bytes, void* stream);

/* sparse_attn_fwd for every run; out: the full [B, H, S, d] output. */
sa_status sparse_attn_fwd_heads(const sa_desc* desc, const int* tiles, const void* q,
                                const void* k, const void* v, const void* workspace,
                                size_t ws_bytes, void* out, void* stream);

/* sparse_attn_check over every run's status word (synchronises stream). */
sa_status sparse_attn_check_heads(const sa_desc* desc, const int* tiles, const void* workspace,
                                  size_t ws_bytes, void* stream);

/* The forward with log-sum-exp, the gradients and the block max-pooled map
 * with per-head shapes: the single-shape calls on every run's slices of the
 * full [B, H, ...] tensors (lse [B*H][S], heat [B*H][nb][nb]) and of the
 * workspace. The runs go one after another on `stream`, so one scratch
 * buffer of the largest run's size (the *_scratch_size_heads calls) serves
 * all of them. */
sa_status sparse_attn_fwd_lse_heads(const sa_desc* desc, const int* tiles, const void* q,
                                   const void* k, const void* v, const void* workspace,
                                   size_t ws_bytes, void* out, float* lse, void* stream);
sa_status sparse_attn_bwd_scratch_size_heads(const sa_desc* desc, const int* tiles,
                                             size_t* bytes);
sa_status sparse_attn_bwd_heads(const sa_desc* desc, const int* tiles, const void* q,
                               const void* k, const void* v, const void* out, const void* dout,
                               const float* lse, const void* workspace, size_t ws_bytes, void* dq,
                               void* dk, void* dv, void* scratch, size_t scratch_bytes,
                               void* stream);
sa_status sparse_attn_block_heatmap_scratch_size_heads(const sa_desc* desc, const int* tiles,
                                                       size_t* bytes);
sa_status sparse_attn_block_heatmap_heads(const sa_desc* desc, const int* tiles, const void* q,
                                          const void* k, void* workspace, size_t ws_bytes,
                                          float* heat, void* scratch, size_t scratch_bytes,
                                          void* stream);

/* Host-only: run number `run` (0-based) as a single-shape problem: its
 * descriptor (*sub, B = 1, H = run length), first flattened head (*head0)
 * and workspace slice (*ws_offset, *ws_bytes), e.g. for sparse_attn_get_mask
 * on that slice. SA_ERR_INVALID_ARG when run is past the last run. */
sa_status sparse_attn_heads_run(const sa_desc* desc, const int* tiles, int run, sa_desc* sub,
                                int* head0, size_t* ws_offset, size_t* ws_bytes);

/* ---- Whole path as one launch (CUDA graph) --------------------------------
 * Plan reuse across calls and steps is the pages' recurring economy (the
 * SVG2 page caches centroids across denoising steps, the TRA page reuses its
 * masks, the Veda page caches tile scores over time). These calls capture
 * sparse_attn_plan (with_plan = 1) and sparse_attn_fwd on fixed buffers into
 * a CUDA graph once; each replay runs the whole path with a single launch on
 * whatever the buffers then hold. with_plan = 0 captures only the forward,
 * reusing the plan already in the workspace. The graph object is the one
 * thing the library allocates (host memory and the driver's graph), owned by
 * the caller until sparse_attn_graph_destroy. Arguments are validated as by
 * the captured calls; nothing runs during creation. */
typedef struct sa_graph sa_graph;

sa_status sparse_attn_graph_create(const sa_desc* desc, const void* q, const void* k,
                                   const void* v, void* workspace, size_t ws_bytes, void* out,
                                   int with_plan, sa_graph** graph);

/* One replay on `stream` (asynchronous; sparse_attn_check reports device
 * timeouts as for the captured calls). */
sa_status sparse_attn_graph_launch(sa_graph* graph, void* stream);

/* Releases the graph (NULL is a no-op). */
sa_status sparse_attn_graph_destroy(sa_graph* graph);

/* ---- Gradients (training use of the mask) ---------------------------------
 * The NABLA page uses the same block mask when training a DiT ("Risultati
 * Sperimentali"), which needs the gradients of the masked attention. With
 * s = q.k / sqrt(d) on the kept blocks, P the softmax over a row's kept keys
 * and O = P V:  dV = P^T dO, dP = dO V^T, D_i = sum_c dO_ic O_ic,
 * dS = P (dP - D), dQ = dS K / sqrt(d), dK = dS^T Q / sqrt(d). */

/* sparse_attn_fwd that also writes each query row's log-sum-exp of its kept
 * scaled scores (natural log) to lse: device fp32 [B*H][S], natural token
 * order, 4-byte aligned. */
sa_status sparse_attn_fwd_lse(const sa_desc* desc, const void* q, const void* k,
                              const void* v, const void* workspace, size_t ws_bytes,
                              void* out, float* lse, void* stream);

/* Bytes of device scratch sparse_attn_bwd needs: an fp32 dQ accumulator
 * [B*H][S][d], two fp32 [B*H][S] row statistics and the transposed block
 * lists (int32 [B*H][ntile] counts and [B*H][ntile][nb] entries). */
sa_status sparse_attn_bwd_scratch_size(const sa_desc* desc, size_t* bytes);

/* dq, dk, dv = gradients of sum(out * dout) with respect to q, k, v, over the
 * mask of the plan in `workspace` (made for the same desc; its status word
 * collects device timeouts, see sparse_attn_check, and keeps them until the
 * next sparse_attn_plan clears it). q, k, v: as for
 * sparse_attn_fwd; out, lse: what sparse_attn_fwd_lse wrote for them (out
 * bf16, or fp32 if desc->out_fp32); dout: [B,H,S,d] bf16 (it is a
 * tensor-core operand). dq, dk, dv: [B,H,S,d], natural order, bf16 (fp32 if
 * desc->out_fp32), overwritten. scratch: at least
 * sparse_attn_bwd_scratch_size() bytes, 256-byte aligned, contents ignored.
 * All tensor pointers 16-byte aligned (lse 4). */
sa_status sparse_attn_bwd(const sa_desc* desc, const void* q, const void* k, const void* v,
                          const void* out, const void* dout, const float* lse,
                          const void* workspace, size_t ws_bytes, void* dq, void* dk,
                          void* dv, void* scratch, size_t scratch_bytes, void* stream);

/* ---- Block max-pooled attention map (mask diagnostics) -------------------
 * "Veda - Diffusione Video Scalabile tramite Attenzione Sparsa Distillata"
 * (gist.science/it/paper/2605.30325), section 2.1 ("Costruzione
 * dell'Obiettivo"): the reference a block mask is measured
 * against is the full, unmasked attention P = softmax(Q K^T / sqrt(d)) of a
 * head, max-pooled over every N x N block:
 *   heat[bh][i][j] = max over q in block i, k in block j of P[q][k],
 * blocks in fractal block order (the order of sparse_attn_get_mask's ids).
 * Computed exactly, densely (one pass over every key per query: about the
 * cost of a dense Q K^T); meant for measuring a mask's recall, not for the
 * attention path. */

/* Bytes of device scratch sparse_attn_block_heatmap needs for `desc`
 * (256 x nb fp32 per CTA of its grid, at most 148 CTAs). */
sa_status sparse_attn_block_heatmap_scratch_size(const sa_desc* desc, size_t* bytes);

/* q, k: as for sparse_attn_plan. workspace: as for sparse_attn_plan; only its
 * status word is used: cleared on `stream` before the launch, so the next
 * sparse_attn_check reports this call (a timed-out wait leaves heat
 * incomplete); the planned lists are left as they are. heat: device fp32
 * [B*H][nb][nb], 4-byte aligned, owned by the caller, overwritten (zeroed
 * first, on `stream`). scratch: device buffer of at least
 * sparse_attn_block_heatmap_scratch_size() bytes, 16-byte aligned, contents
 * ignored (SA_ERR_WORKSPACE when smaller). */
sa_status sparse_attn_block_heatmap(const sa_desc* desc, const void* q, const void* k,
                                    void* workspace, size_t ws_bytes, float* heat,
                                    void* scratch, size_t scratch_bytes, void* stream);

/* ---- Token Radius Attention mask (a second mask builder) -----------------
 * "Token Radius Attention per la Generazione di Video Efficiente"
 * (gist.science/it/paper/2608.02504), section 2, "La Pipeline TRA". Each query
 * token gets a key budget from the entropy of its full attention row, the
 * budget becomes a spatial radius that shrinks with the distance in frames,
 * and token votes turn the per-token discs into a block mask in the same
 * workspace format as sparse_attn_plan's, so that sparse_attn_fwd,
 * sparse_attn_fwd_lse, sparse_attn_bwd and the graph calls run on it
 * unchanged. */

/* Step 1 ("Entropy-to-Budget", the dense warm-up): the entropy in nats of
 * every query's full, unmasked attention row, H_i = -sum_j p_ij ln p_ij with
 * p = softmax(q_i . k_j / sqrt(d)) over all keys, written to entropy: device
 * fp32 [B*H][S] in natural token order, 4-byte aligned, owned by the caller.
 * One dense pass (the cost of a dense Q K^T). q, k: as for sparse_attn_plan.
 * workspace: as for sparse_attn_plan; only its status word is used (cleared
 * on `stream` first, so sparse_attn_check reports this call). */
sa_status sparse_attn_token_entropy(const sa_desc* desc, const void* q, const void* k,
                                    void* workspace, size_t ws_bytes, float* entropy,
                                    void* stream);

typedef struct sa_radius {
  float tau;     /* > 0: keys per query k_i = min(S, tau exp(H_i)) */
  float gamma;   /* >= 0: the radius at a distance of delta frames is
                    r_i exp(-gamma delta) */
  int vote_min;  /* 1..N: query tokens of a q-block that must reach a k-block
                    for the block pair to be kept */
} sa_radius;

/* Steps 2-3 ("Budget-to-Radius", "Kernel CUDA Fusi"): with
 * Z(t) = sum over the frames t' of exp(-2 gamma |t' - t|) and r_i^2 =
 * k_i / (pi Z(t_i)), key (t', h', w') is in query i's support iff
 * (h' - h_i)^2 + (w' - w_i)^2 <= r_i^2 exp(-2 gamma |t' - t_i|) (token units);
 * query i votes for a k-block iff its support holds one of the block's keys;
 * q-block a keeps k-block b iff at least vote_min of its N queries vote for b.
 * A query's own position is always in its support, so no row is empty.
 * Writes the per-q-block lists, the per-tile union lists and the tile order
 * into `workspace` exactly as sparse_attn_plan does (desc->thr and the STA
 * window are not used; the pooled means are not written). entropy: device
 * fp32 [B*H][S], natural order (e.g. from sparse_attn_token_entropy, possibly
 * of an earlier step: the page reuses the warm-up entropies across steps).
 * SA_ERR_INVALID_ARG for tau <= 0, gamma < 0, non-finite values or vote_min
 * outside 1..N; SA_ERR_UNSUPPORTED beyond T = 4096 frames, Hh or Ww = 1024
 * tokens, or 6144 blocks per head. */
sa_status sparse_attn_plan_radius(const sa_desc* desc, const sa_radius* radius,
                                  const float* entropy, void* workspace, size_t ws_bytes,
                                  void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_ATTN_H */
