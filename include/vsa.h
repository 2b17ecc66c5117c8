/*
 * vsa.h -- C ABI of libvsa, the B200 (sm_100a) VSA tile-sparse attention layer
 * for reference-to-video.
 *
 * The layer works in five steps (pages: "ComfyUI-Ref2VA-VSA proves a sparse
 * attention gate can be transplanted ..." (SnackOnAI), "The Code, Annotated";
 * "Ref2VA VSA: Sparse Attention Node for H3 Reference-to-Video" (ComfyUI wiki),
 * "The two-tier attention patch"; "Veda Sparse Attention" (ComfyUI wiki), the
 * node input table):
 *   1. plan + permute: prefix segments into segment-pure tiles, video into
 *      3-D cubes, tokens scattered into a zero-padded tile layout;
 *   2. coarse attention over per-tile mean-pooled Q/K/V;
 *   3. per-head top-k over the video key tiles (prefix tiles are sinks);
 *   4. block-sparse attention over the kept tiles (prefix queries dense);
 *   5. out = o_fine + sigmoid(g) * o_coarse, g = the gate projection.
 *
 * Conventions for every call below
 *   - Tensors are row-major with the last dimension contiguous.  "bf16" means
 *     IEEE bfloat16 stored as uint16.  [B,H,N,D] is the natural token order,
 *     [B,H,N_pad,D] the padded tile layout (row r = tile r / R, slot r % R).
 *   - Device pointers are owned by the caller, must be on the plan's device
 *     and 16-byte aligned; nothing is allocated behind the caller's back
 *     except the plan's own tables (vsa_plan_create).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream); launches are
 *     asynchronous on it, and the calling thread's current device must be the
 *     plan's device.
 *   - Arguments are checked synchronously before any launch; a failed check
 *     returns an error and launches nothing.  vsa_last_error() then holds a
 *     message (thread-local).  Faults found by a kernel (a wait that timed out,
 *     an index out of range) are recorded in the plan's device status word and
 *     reported by vsa_sync_status().
 *   - Supported: D in {64, 128}; R = tile_t*tile_h*tile_w in {64, 128}.
 *   - Every call that launches work opens an NVTX range named after itself
 *     (a no-op unless a profiler is attached).
 */
#ifndef VSA_H_
#define VSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define VSA_API_VERSION 1

typedef enum vsa_status {
  VSA_OK = 0,
  VSA_ERR_INVALID_ARG = 1,     /* null/misaligned pointer, bad size, wrong device   */
  VSA_ERR_UNSUPPORTED = 2,     /* D not in {64,128}, R not in {64,128}               */
  VSA_ERR_PLAN = 3,            /* geometry gives a non-injective or impure plan      */
  VSA_ERR_WORKSPACE = 4,       /* workspace missing or smaller than required         */
  VSA_ERR_CUDA = 5,            /* a CUDA runtime/driver call failed                  */
  VSA_ERR_DEVICE_TIMEOUT = 6,  /* a kernel wait exceeded its bound and bailed out    */
  VSA_ERR_DEVICE_INDEX = 7     /* a kernel met a kept-tile index outside its range   */
} vsa_status;

typedef struct vsa_plan_s* vsa_plan;

/* Geometry of one layer call.  prefix_lens[s] is the length of prefix segment s
 * (text, reference image(s), reference audio, ...) in sequence order; zero-length
 * segments are allowed and take no tile.  The video follows the prefix, flattened
 * t-major, then h, then w.  tile_* is the video cube: 4x4x4 = 64 rows (VSA) or
 * 4x8x4 = 128 rows (Veda's 128-token key tiles); prefix tiles use the same R. */
typedef struct vsa_geometry {
  int32_t n_prefix_segments;
  const int64_t* prefix_lens;        /* host pointer, n_prefix_segments entries */
  int32_t grid_t, grid_h, grid_w;    /* latent video grid                       */
  int32_t tile_t, tile_h, tile_w;    /* cube extent                             */
} vsa_geometry;

/* Step 1 (host).  Build the plan: every prefix segment is cut into R-row tiles
 * (its last tile may be short) and each segment starts a fresh tile; then the
 * video is cut into cubes (clipped at the grid's far edges) visited t0, h0, w0,
 * tokens inside a cube in lexicographic (t, h, w) order at the head of the
 * tile.  Source: SnackOnAI, "The Code, Annotated", snippet one; clipped cubes
 * reproduce that page's "It In Action" count (26 + 660 tiles, 43,904 rows).
 * `device` >= 0 uploads the tables to that CUDA device (synchronously);
 * device = -1 builds a host-only plan (tables and keep counts only, no
 * launches).  Returns VSA_ERR_PLAN when the map is not injective, a tile would
 * mix segments, or the grid is negative.  *out is owned by the caller and
 * released with vsa_plan_destroy. */
vsa_status vsa_plan_create(const vsa_geometry* geom, int device, vsa_plan* out);

/* Sizes of a plan: N real tokens, N_pad = T * R padded rows, T tiles, of which
 * n_p prefix tiles, R rows per tile.  Any output pointer may be NULL. */
vsa_status vsa_plan_info(vsa_plan plan, int64_t* n_tokens, int64_t* n_padded,
                         int32_t* n_tiles, int32_t* n_prefix_tiles, int32_t* tile_rows);

/* Host copies of the plan tables (any pointer may be NULL):
 *   untile[N]     token -> padded row;
 *   row_src[N_pad] padded row -> token, -1 for a pad row;
 *   block_len[T]  live rows of each tile (real rows sit at the head);
 *   tile_seg[T]   prefix segment of the tile, -1 for a video tile. */
vsa_status vsa_plan_tables(vsa_plan plan, int32_t* untile, int32_t* row_src,
                           int32_t* block_len, int32_t* tile_seg);

/* Number k of video key tiles each video query tile keeps (step 3).
 * keep_tiles >= 0: Veda integer mode, k = min(keep_tiles, n_v) ("Veda Sparse
 * Attention", generated_sparsity = 24 keeps exactly 24 key tiles).
 * keep_tiles < 0: ratio mode, k = min(n_v, ceil(clamp(keep_ratio,0,1) * n_v - 1e-9))
 * (SnackOnAI snippet two: keep_ratio = 1 - sparsity; the ceiling reproduces
 * that page's 165 and 66 of 660 tiles).  k = 0 with no prefix tile is
 * rejected (VSA_ERR_INVALID_ARG): a query tile would have no key. */
vsa_status vsa_keep_count(vsa_plan plan, double keep_ratio, int32_t keep_tiles, int32_t* k);

/* Frees the plan's host and device tables and its status block (after a
 * device synchronisation when the plan has a device).  The caller must not
 * use the plan, nor any runner built on it, afterwards.  NULL is a no-op. */
vsa_status vsa_plan_destroy(vsa_plan plan);

/* Bytes of device workspace vsa_coarse_topk needs for B, H, D, k
 * (vsa_sparse_attn needs none and accepts ws = NULL).  Layout (fp32): the
 * pooled means, qbar at offset 0, kbar at B*H*T*D*4, vbar at 2*B*H*T*D*4, each
 * [B,H,T,D]; then, at 3*B*H*T*D*4, the coarse kernel's score rows (32 rows of
 * ceil4(T) floats for each of its 2 x (SM count) persistent CTAs), which hold
 * nothing on return. */
vsa_status vsa_workspace_size(vsa_plan plan, int B, int H, int D, int k, size_t* bytes);

/* Step 1 (device).  x_t[b,h,untile[n],:] = x[b,h,n,:]; pad rows are written 0.
 * x: bf16 [B,H,N,D]; x_t: bf16 [B,H,N_pad,D].  Source: SnackOnAI snippet two
 * (x_t = zeros(padded); x_t[untile] = x).  Applied to Q, K, V and the gate. */
vsa_status vsa_permute(vsa_plan plan, const void* x, void* x_t, int B, int H, int D,
                       void* stream);

/* Inverse of vsa_permute: x[b,h,n,:] = x_t[b,h,untile[n],:] (pad rows dropped). */
vsa_status vsa_unpermute(vsa_plan plan, const void* x_t, void* x, int B, int H, int D,
                         void* stream);

/* Steps 2 and 3.  Pools q_t, k_t, v_t (bf16 [B,H,N_pad,D]) into fp32 per-tile
 * means over the live rows (into `ws`), then for every query tile i and head:
 *   s[i,j] = scale * <qbar_i, kbar_j> over all T tiles (fp32),
 *   o_coarse[b,h,i,:] = sum_j softmax_j(s[i,:]) vbar_j        (fp32 [B,H,T,D]),
 * and for every video query tile i (n_p <= i < T) the k video key tiles j with
 * the largest s[i,j], ties to the lower j, written in ascending j order to
 * topk_idx[b,h,i-n_p,:] (int32 [B,H,n_v,k], global tile indices).  topk_score
 * (nullable, fp32 [B,H,n_v,k]) receives s[i,j] of each kept tile.  Sources:
 * the wiki page's "two-tier attention patch" (top-k strictly over generated-
 * video key tiles, prefix exempt), Veda's head-aware top-k; the mean pooling
 * and the coarse softmax are this library's reading of "coarse tile
 * selection" (SnackOnAI, "References", the VSA paper).  k may be 0 (nothing
 * written to topk_idx) when n_p > 0. */
vsa_status vsa_coarse_topk(vsa_plan plan, const void* q_t, const void* k_t, const void* v_t,
                           int B, int H, int D, float scale, int k,
                           float* o_coarse, int32_t* topk_idx, float* topk_score,
                           void* ws, size_t ws_bytes, void* stream);

/* Steps 1 and 2 fused for one of Q, K, V: the permute of vsa_permute, and in
 * the same pass the fp32 mean over each tile's live rows, written to
 * pooled[b,h,t,:] (fp32 [B,H,T,D]; 16-byte aligned).  Same permuted output as
 * vsa_permute; the pooled means equal those vsa_coarse_topk computes up to
 * fp32 summation order.  For a layer, point `pooled` at the workspace slot of
 * the tensor (qbar, kbar or vbar, see vsa_workspace_size) and finish with
 * vsa_coarse_topk_pooled.  Sources: SnackOnAI snippet two (the permute) and
 * this library's reading of "coarse tile selection" (mean pooling). */
vsa_status vsa_permute_pool(vsa_plan plan, const void* x, void* x_t, int B, int H, int D,
                            float* pooled, void* stream);

/* Steps 2 (coarse part) and 3 of vsa_coarse_topk from pooled means already in
 * `ws` (qbar, kbar, vbar in the layout of vsa_workspace_size, as written by
 * vsa_permute_pool): no pooling pass and no q_t/k_t/v_t arguments.  Same
 * outputs, validation and errors as vsa_coarse_topk. */
vsa_status vsa_coarse_topk_pooled(vsa_plan plan, int B, int H, int D, float scale, int k,
                                  float* o_coarse, int32_t* topk_idx, float* topk_score,
                                  void* ws, size_t ws_bytes, void* stream);

/* Reference-tile thinning (the Veda node's reference_sparsity, "Veda Sparse
 * Attention" input table: the generated-video keep setting applied to the
 * reference tokens, 0 % = full attention).  Reading taken: each generated-
 * video query tile keeps only its top k_ref reference (prefix) key tiles by
 * coarse score instead of all n_p of them; reference query tiles stay dense.
 *
 * vsa_keep_count_ref: k_ref for n_p reference tiles, the keep rule of
 * vsa_keep_count: keep_tiles >= 0 -> min(keep_tiles, n_p), else
 * min(n_p, ceil(clamp(keep_ratio,0,1) * n_p - 1e-9)). */
vsa_status vsa_keep_count_ref(vsa_plan plan, double keep_ratio, int32_t keep_tiles, int32_t* k_ref);

/* For every video query tile i (n_p <= i < T) and (b,h): the k_ref reference
 * tiles j < n_p with the largest s[i,j] = scale * <qbar_i, kbar_j> (fp32, the
 * same scores vsa_coarse_topk ranks), ties to the lower j, ascending, into
 * topk_ref_idx (int32 [B,H,n_v,k_ref]).  Reads the pooled means qbar, kbar
 * from `ws` (the layout of vsa_workspace_size, as left by vsa_coarse_topk or
 * vsa_permute_pool).  n_p <= 256 (else VSA_ERR_UNSUPPORTED); k_ref in
 * [0, n_p]. */
vsa_status vsa_select_reference(vsa_plan plan, int B, int H, int D, float scale, int k_ref,
                                int32_t* topk_ref_idx, const void* ws, size_t ws_bytes,
                                void* stream);

/* Sparse attention with thinned reference tiles: a video query tile attends to
 * its k_ref kept reference tiles (topk_ref_idx [B,H,n_v,k_ref]) and its k kept
 * video tiles; prefix query tiles stay dense.  gate == NULL: o_fine in the
 * padded layout (as vsa_sparse_attn); gate and o_coarse given: the fused
 * gated combine writing natural order (as vsa_sparse_attn_combine).  k_ref =
 * n_p with topk_ref_idx = NULL is the unthinned layer.  k + k_ref >= 1.
 * lse_t nullable. */
vsa_status vsa_sparse_attn_ref(vsa_plan plan, const void* q_t, const void* k_t, const void* v_t,
                               const int32_t* topk_idx, int k, const int32_t* topk_ref_idx,
                               int k_ref, int B, int H, int D, float scale, const void* gate,
                               const float* o_coarse, void* out, float* lse_t, void* stream);

/* Head projection, the gate's bias-free linear (SnackOnAI, "The Code,
 * Annotated", snippet three: gate = x W_gate^T viewed as [.., heads,
 * head_dim]; with act = 0 any projection of that shape):
 *   y[b,h,n,d] = act( sum_c x[b,n,c] * w[h*D+d, c] ),  act 0: identity, 1: sigmoid.
 * x: bf16 [B,N,C] (N = the plan's real tokens, natural order), w: bf16 [H*D,C]
 * (nn.Linear weight layout), y: bf16 [B,H,N,D] natural order, the layout
 * vsa_sparse_attn_combine reads the gate in.  fp32 accumulation, bf16 round to
 * nearest even.  All pointers 16-byte aligned, C a multiple of 8 (TMA row
 * stride).  A tcgen05 GEMM on the device of the plan; asynchronous on `stream`. */
vsa_status vsa_project(vsa_plan plan, const void* x, const void* w, int B, int H, int D, int C,
                       int act, void* y, void* stream);

/* Tile before projecting (SnackOnAI, "The Code, Annotated", snippet two: the
 * layer input x is tiled first and the tiled x_t is projected, so that Q, K, V
 * and the gate come out in tile order without four sequence-sized copies).
 * vsa_permute_rows: x_t[b, untile[n], :] = x[b, n, :], pad rows 0; x bf16
 * [B,N,C] natural order, x_t bf16 [B,N_pad,C]; C a multiple of 8, pointers
 * 16-byte aligned.  vsa_project_tiled: vsa_project on the tiled rows,
 * x_t bf16 [B,N_pad,C] -> y_t bf16 [B,H,N_pad,D] (pad rows of a zero-padded x_t
 * hold act(0): 0 for the identity).  A row permutation commutes with the
 * row-wise product, so vsa_project_tiled(vsa_permute_rows(x)) equals
 * vsa_permute(vsa_project(x)) element for element. */
vsa_status vsa_permute_rows(vsa_plan plan, const void* x, void* x_t, int B, int C, void* stream);
vsa_status vsa_project_tiled(vsa_plan plan, const void* x_t, const void* w, int B, int H, int D,
                             int C, int act, void* y_t, void* stream);

/* Allocation-free variant of vsa_coarse_topk (the pages have no counterpart:
 * this is a library convenience).  For callers that cannot call cudaMalloc --
 * a host application that owns all device memory and gives plugins no
 * allocator, or a latency-critical loop that cannot afford cudaMalloc's
 * implicit device-wide synchronisation -- the pooled-mean scratch lives in a
 * fixed 16 MiB array in the library's device memory, held on every GPU that
 * loads the library until the process exits.  Same arguments and results as
 * vsa_coarse_topk, without ws / ws_bytes; allocates nothing.
 * Limit: the call needs 3*B*H*T*D*4 bytes of scratch and returns
 * VSA_ERR_WORKSPACE, launching nothing, when that exceeds 16 MiB.
 * The first call on a device resolves the array's device address with
 * cudaGetSymbolAddress (once per device, that device current); make that first
 * call before any stream capture.  The address is cached per device together
 * with the CUDA context that was current when it was resolved, and resolved
 * again when a call finds another context current.  cudaDeviceReset
 * invalidates every device resource the library holds, plans included:
 * destroy and recreate plans after a reset.  All calls share the array, which
 * keeps the last call's contents (nothing in it needs to start at zero);
 * calls that overlap on the GPU race on it and must be serialised by the
 * caller. */
vsa_status vsa_coarse_topk_noalloc(vsa_plan plan, const void* q_t, const void* k_t,
                                   const void* v_t, int B, int H, int D, float scale, int k,
                                   float* o_coarse, int32_t* topk_idx, float* topk_score,
                                   void* stream);

/* Step 4.  For every live query row of tile i and head: softmax over the live
 * key rows of S_i, o_fine = sum p v, with S_i = all T tiles when i < n_p
 * (prefix queries are dense) and S_i = {0..n_p-1} U topk_idx[b,h,i-n_p,:]
 * otherwise (prefix tiles are always-kept sinks).  Source: SnackOnAI snippet
 * two (sink_blocks / sink_q = [0, num_prefix_tiles), block_len, scale =
 * head_dim^-0.5 there; here `scale` is an argument).  o_fine_t: bf16
 * [B,H,N_pad,D], pad rows written 0.  lse_t (nullable): fp32 [B,H,N_pad],
 * natural-log log-sum-exp of each live row's scaled scores (0 on pad rows).
 * topk_idx must hold valid, distinct video tile indices (as vsa_coarse_topk
 * writes them).  A kernel that meets an index outside [n_p, T) replaces it
 * with tile n_p, so the outputs of that query tile are then undefined, and
 * records VSA_ERR_DEVICE_INDEX for vsa_sync_status.  ws may be NULL. */
vsa_status vsa_sparse_attn(vsa_plan plan, const void* q_t, const void* k_t, const void* v_t,
                           const int32_t* topk_idx, int B, int H, int D, int k, float scale,
                           void* o_fine_t, float* lse_t, void* ws, size_t ws_bytes,
                           void* stream);

/* Steps 4 and 5 fused: the attention of vsa_sparse_attn, with the gated combine
 * of vsa_gate_combine applied in its epilogue to the fp32 attention output (no
 * bf16 rounding of o_fine in between) and the result written in natural token
 * order: out[b,h,n,:] = o_fine + sigmoid(gate[b,h,n,:]) * o_coarse[b,h,tile(n),:].
 * gate: bf16 [B,H,N,D] in NATURAL order (the to_gate_compress projection split
 * into heads, no permute needed); o_coarse: fp32 [B,H,T,D] from
 * vsa_coarse_topk; out: bf16 [B,H,N,D]; lse_t as for vsa_sparse_attn.  Sources
 * as for the two unfused calls; fusing them saves the o_fine round trip
 * through HBM, the permute of the gate and one launch. */
vsa_status vsa_sparse_attn_combine(vsa_plan plan, const void* q_t, const void* k_t,
                                   const void* v_t, const int32_t* topk_idx, int B, int H, int D,
                                   int k, float scale, const void* gate, const float* o_coarse,
                                   void* out, float* lse_t, void* stream);

/* Step 5.  out = o_fine + sigmoid(g) * o_coarse[tile(row)], element-wise over
 * D, fp32 arithmetic, bf16 round-to-nearest-even store.  o_fine_t and gate_t:
 * bf16 [B,H,N_pad,D] (the gate is the bias-free to_gate_compress projection of
 * the layer input, split into heads and permuted like Q: SnackOnAI snippet
 * two, gate_t passed as coarse_gate); o_coarse: fp32 [B,H,T,D].
 * out_natural = 0: out is bf16 [B,H,N_pad,D] with pad rows 0;
 * out_natural = 1: out is bf16 [B,H,N,D] in natural token order (the
 * unpermute fused in). */
vsa_status vsa_gate_combine(vsa_plan plan, const void* o_fine_t, const void* gate_t,
                            const float* o_coarse, void* out, int out_natural,
                            int B, int H, int D, void* stream);

/* ---------------------------------------------------------------- runner
 * The whole layer over inputs in HOST memory, layer after layer, with the
 * transfers overlapped with the computation (an engineering addition: the
 * pages describe the layer, not how its inputs reach the GPU).  The runner
 * owns two sets of device buffers (natural and tiled Q/K/V, the gate, the
 * workspace, o_coarse, the selection, the output) and three CUDA streams:
 * while layer i computes, the inputs of layer i+1 are copied in and the
 * output of layer i-1 is copied out.  Each layer is steps 1 to 5 as
 * vsa_permute_pool (x3), vsa_coarse_topk_pooled and vsa_sparse_attn_combine
 * compute them, so a layer's output is bit-identical to that chain's. */
typedef struct vsa_runner_s* vsa_runner;

/* Allocates the runner's device buffers (on the plan's device, which must be
 * current) for B, H, D, k and scale as the layer calls take them.  The plan
 * must outlive the runner.  Errors: VSA_ERR_INVALID_ARG / VSA_ERR_UNSUPPORTED
 * for arguments the layer calls would reject, VSA_ERR_CUDA when an allocation
 * fails (nothing is kept; *out = NULL). */
vsa_status vsa_runner_create(vsa_plan plan, int B, int H, int D, int k, float scale,
                             vsa_runner* out);

/* Runs n_layers layers: layer i reads q[i], k[i], v[i], g[i] (host bf16
 * [B,H,N,D], natural token order; g the gate projection split into heads) and
 * writes out[i] (host bf16 [B,H,N,D]).  Host buffers should be page-locked
 * (cudaHostAlloc / cudaHostRegister) for the copies to be asynchronous; they
 * must stay valid and untouched until the run has finished.  The run starts
 * after the work already queued on `stream` and `stream` waits for its last
 * copy-out; the call itself returns once everything is queued.  Kernel faults
 * are recorded in the plan's status word (vsa_sync_status).  Runs of one
 * runner must not overlap in time with each other, and nothing else may use
 * the plan's attention kernels concurrently.  On an error return the layers
 * queued before the failing call may still run; `stream` then does not wait
 * for them, vsa_runner_destroy does. */
vsa_status vsa_runner_run(vsa_runner runner, int n_layers, const void* const* q,
                          const void* const* k, const void* const* v, const void* const* g,
                          void* const* out, void* stream);

/* Device time of the last vsa_runner_run, in ms, from before its first
 * copy-in to after its last copy-out (waits for the run to finish). */
vsa_status vsa_runner_elapsed(vsa_runner runner, float* ms);

/* Waits for the runner's streams, then frees its buffers, streams and events.
 * NULL is a no-op. */
vsa_status vsa_runner_destroy(vsa_runner runner);

/* ---------------------------------------------------------------- backward
 * Gradients of a loss through steps 5 .. 1, for training (SnackOnAI, "The
 * Architecture, Unpacked": the coarse stage and the gate are learned; the VSA
 * paper it builds on trains its sparse kernel).  The top-k selection passes no
 * gradient: the backward runs under the forward's topk_idx (and topk_ref_idx).
 * A training step calls, in this order: vsa_permute of d_out (natural -> tiled),
 * vsa_combine_backward, vsa_coarse_backward, vsa_sparse_attn_backward, and
 * vsa_unpermute of dq_t, dk_t, dv_t and d_gate_t.  All launches asynchronous on
 * `stream`; the caller owns every buffer. */

/* Bytes of the workspace that vsa_coarse_backward and vsa_sparse_attn_backward
 * need (the larger of the two: they may share one buffer, called in turn). */
vsa_status vsa_backward_workspace_size(vsa_plan plan, int B, int H, int D, size_t* bytes);

/* Backward of step 5 for out = o_fine + sigmoid(g) * o_coarse[tile]:
 *   d_gate_t = d_out * o_coarse[tile] * s (1 - s),  s = sigmoid(g)
 *   d_o_coarse[t] = sum over the live rows of tile t of d_out * s
 *   delta[r] = sum_d d_out[r] o_fine[r]  (the row statistic of the fine
 *              softmax backward)
 * d_out_t, o_fine_t, gate_t: bf16 [B,H,N_pad,D] tiled (d_out_t with pad rows 0,
 * as vsa_permute writes it; o_fine_t as vsa_sparse_attn writes it).  o_coarse:
 * fp32 [B,H,T,D].  Writes delta fp32 [B,H,N_pad] and d_gate_t bf16
 * [B,H,N_pad,D] (0 on pad rows), d_o_coarse fp32 [B,H,T,D]. */
vsa_status vsa_combine_backward(vsa_plan plan, const void* d_out_t, const void* o_fine_t,
                                const void* gate_t, const float* o_coarse, int B, int H, int D,
                                float* delta, void* d_gate_t, float* d_o_coarse, void* stream);

/* Backward of the coarse attention of step 2 (o_coarse = softmax(scale qbar
 * kbar^T) vbar over all T tiles): d_qbar, d_kbar, d_vbar fp32 [B,H,T,D] from
 * the pooled means qbar, kbar, vbar fp32 [B,H,T,D] (as vsa_permute_pool writes
 * them) and d_o_coarse.  fp32 arithmetic.  ws: at least
 * vsa_backward_workspace_size bytes, 16-byte aligned. */
vsa_status vsa_coarse_backward(vsa_plan plan, const float* qbar, const float* kbar,
                               const float* vbar, const float* d_o_coarse, int B, int H, int D,
                               float scale, float* d_qbar, float* d_kbar, float* d_vbar, void* ws,
                               size_t ws_bytes, void* stream);

/* Backward of step 4 (and of the pooling of step 2): for every query tile i
 * and key tile j of its key set (as in vsa_sparse_attn / vsa_sparse_attn_ref),
 * P = exp(scale Q_i K_j^T - lse_i) on live rows and columns, dP = dO_i V_j^T,
 * dS = P (dP - delta_i), and
 *   dq_t = scale sum_j dS K_j + d_qbar[tile] / block_len[tile]
 *   dk_t = scale sum_i dS^T Q_i + d_kbar[tile] / block_len[tile]
 *   dv_t = sum_i P^T dO_i + d_vbar[tile] / block_len[tile]
 * on live rows (pad rows written 0).  q_t, k_t, v_t, d_out_t: bf16
 * [B,H,N_pad,D]; lse_t: fp32 [B,H,N_pad] from the forward; delta from
 * vsa_combine_backward; d_qbar, d_kbar, d_vbar: fp32 [B,H,T,D] from
 * vsa_coarse_backward, or all three NULL (no pooling term).  topk_ref_idx and
 * k_ref as for vsa_sparse_attn_ref (NULL with k_ref = n_p: every reference
 * tile).  Outputs bf16 [B,H,N_pad,D].  fp32 accumulation in tensor memory; P and
 * dS are rounded to bf16 before their products.  An index outside its range is
 * skipped and recorded (VSA_ERR_DEVICE_INDEX).  ws: at least
 * vsa_backward_workspace_size bytes. */
vsa_status vsa_sparse_attn_backward(vsa_plan plan, const void* q_t, const void* k_t,
                                    const void* v_t, const void* d_out_t, const int32_t* topk_idx,
                                    int k, const int32_t* topk_ref_idx, int k_ref,
                                    const float* lse_t, const float* delta, const float* d_qbar,
                                    const float* d_kbar, const float* d_vbar, int B, int H, int D,
                                    float scale, void* dq_t, void* dk_t, void* dv_t, void* ws,
                                    size_t ws_bytes, void* stream);

/* Self-test of the bounded device wait every kernel of the library uses: one
 * CTA whose two waiting threads wait on an mbarrier that nothing completes.
 * The waits give up after their bound (2 s of wall time), the kernel records
 * VSA_ERR_DEVICE_TIMEOUT in the plan's status word (read it with
 * vsa_sync_status) and returns; result (device int32[2], 16-byte aligned)
 * receives 0 for each wait that gave up.  The context stays usable. */
vsa_status vsa_check_bounded_wait(vsa_plan plan, int32_t* result, void* stream);

/* Test hook for the attention kernels' failure path (the pages have no
 * counterpart).  Sets the bound of every mbarrier wait of the kernels that
 * vsa_sparse_attn, vsa_sparse_attn_combine, vsa_sparse_attn_ref and
 * vsa_sparse_attn_backward launch from then on, process-wide, in ns of wall
 * time; 0 (or anything above it) restores the 2 s default.  With a bound of
 * a few microseconds their waits run out: the kernel records
 * VSA_ERR_DEVICE_TIMEOUT in the plan's status word, drains its own TMA loads
 * and MMAs, frees its tensor memory and returns, and the outputs of that
 * launch are undefined.  Not for production use; not thread safe against
 * launches running concurrently in other host threads.  Returns VSA_OK. */
vsa_status vsa_debug_set_wait_limit(uint64_t ns);

/* Synchronise `stream`, then read and clear the plan's device status word.
 * Returns VSA_OK, VSA_ERR_DEVICE_TIMEOUT, VSA_ERR_DEVICE_INDEX or VSA_ERR_CUDA. */
vsa_status vsa_sync_status(vsa_plan plan, void* stream);

/* Message of the calling thread's last failed call ("" if none). */
const char* vsa_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* VSA_H_ */
