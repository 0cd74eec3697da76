/*
 * rtr.h -- C ABI of librtr: frame-causal attention with a reference-preserving
 * rolling KV cache on NVIDIA B200 (sm_100a).
 *
 * The method is RTR-DiT's streaming rerenderer, as described by the
 * papernotes.org note "DiT as Real-Time Rerenderer: Streaming Video
 * Stylization with Autoregressive Diffusion Transformer":
 *
 *   - Method > Key Designs 2: 3D self-attention under a temporal causal mask,
 *       Attn(Q,K,V) = softmax(Q K^T / sqrt(d) + M) V,
 *       M_ij = 0 iff floor(j/k) <= floor(i/k), else -inf,
 *     d = head dimension, k = spatial tokens per latent frame.
 *   - Method > Key Designs 4: a fixed-length rolling KV cache (new frames
 *     appended, oldest evicted) whose reference-image tokens live in a
 *     resident slot at the front that eviction never touches; a fixed-length
 *     cross-attention cache that is reinitialised when the text prompt or the
 *     reference image is switched, while the 3D cache keeps its most recent
 *     frame and a new reference image is anchored at the front.
 *   - Method > Key Designs 1: the reference latent is one extra latent frame
 *     placed before the first frame; text enters through cross-attention;
 *     TV2V runs without a reference.
 *   - Method > Overall Architecture and Key Designs 3: the tokens pass through
 *     DiT blocks (rtr_dit_block_forward runs one block around the attention),
 *     and training runs gradient descent through the block-causal attention
 *     (rtr_attn_block_causal_backward).
 *
 * Conventions shared by every call
 *   - Device tensors are row-major.  Q, K, V and outputs use the layout
 *     [tokens][heads][head_dim] (what a DiT's QKV projection produces).
 *   - Element types: RTR_BF16 (bfloat16, arithmetic in fp32 with fp32
 *     accumulation on the tensor cores) or RTR_F32 (float32 storage, fp32
 *     arithmetic).  head_dim is 64 or 128.
 *   - Ownership: the library owns cache and cross-attention buffers; the
 *     caller owns every q/k/v/out pointer.  Those must be device pointers on
 *     the handle's device, 16-byte aligned, and stay valid until the work
 *     enqueued on `stream` has finished.
 *   - Asynchrony: data work is enqueued on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream).  Host-side cache state (index maps, valid
 *     flags) changes when the call returns.  Calls on one handle must be
 *     ordered by the caller (one stream, or events).
 *   - Errors: arguments are checked before anything is enqueued; a failing
 *     call returns a status and leaves the handle unchanged.  Nothing aborts.
 *     Device-side failures (a bounded wait that expired) are latched in a
 *     per-device status word read by rtr_get_device_status.
 *   - Not thread-safe per handle; distinct handles may be used concurrently.
 */
#ifndef RTR_H
#define RTR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RTR_OK = 0,
    RTR_E_INVAL = 1,        /* bad argument (shape, pointer, alignment, range) */
    RTR_E_NOMEM = 2,        /* device allocation failed */
    RTR_E_STATE = 3,        /* call not valid in the handle's current state */
    RTR_E_CUDA = 4,         /* a CUDA runtime/driver call failed */
    RTR_E_TIMEOUT = 5,      /* a kernel's bounded wait expired (device status) */
    RTR_E_UNSUPPORTED = 6   /* valid request this library does not implement */
} rtr_status;

typedef enum { RTR_BF16 = 0, RTR_F32 = 1 } rtr_dtype;

/* Same type as cudaStream_t, spelled without the CUDA headers. */
typedef struct CUstream_st *rtr_stream_t;

typedef struct rtr_kvcache rtr_kvcache;
typedef struct rtr_xattn rtr_xattn;

/* Human-readable name of a status code (static storage). */
const char *rtr_status_string(rtr_status s);

/* ---------------------------------------------------------------------------
 * Reference-preserving rolling KV cache (Key Designs 4; reference frame from
 * Key Designs 1).
 *
 * Per layer the cache holds K and V, each [heads][(ref_frames + S) *
 * k][head_dim], with S = window_frames physical window slots
 * (window_frames + commit_frames for rtr_kvcache_create_ex): rows
 * [0, ref_frames*k) are the anchored reference slot, window slot s occupies
 * rows (ref_frames+s)*k ... +k-1.  Frame f (counted from creation) lives in
 * slot f mod S; at most window_frames frames are held.  All slots start
 * empty and the reference starts invalid.  Buffers are zeroed at creation.
 *
 * rtr_kvcache_create: layers >= 1, heads >= 1, head_dim in {64, 128}, k >= 1,
 *   ref_frames >= 0, window_frames >= 1, dt RTR_BF16 or RTR_F32, device a
 *   CUDA ordinal.  On success *out receives the handle.  RTR_E_NOMEM if the
 *   device allocation fails.
 */
rtr_status rtr_kvcache_create(int layers, int heads, int head_dim, int k,
                              int ref_frames, int window_frames, rtr_dtype dt,
                              int device, rtr_kvcache **out);

/* rtr_kvcache_create with commit room: the ring gets commit_frames physical
 * slots beyond the window_frames it holds (0 <= commit_frames <=
 * window_frames; 0 is rtr_kvcache_create).  The spare slots let
 * rtr_attn_frame_causal_commit write a chunk of up to commit_frames frames
 * while the frames that chunk attends to stay in place.  Memory per layer
 * grows by 2 * heads * commit_frames * k * head_dim elements.  (Every bf16
 * cache with k a multiple of 8 also holds 512 bytes of TMA store descriptors
 * per reference frame and ring slot, through which the fused writes of
 * rtr_attn_frame_causal_commit and rtr_attn_block_causal_prefill_cache go.)
 * This is a layout choice of the library; the held frames, and so every
 * attention result, are the same as with rtr_kvcache_create. */
rtr_status rtr_kvcache_create_ex(int layers, int heads, int head_dim, int k,
                                 int ref_frames, int window_frames,
                                 int commit_frames, rtr_dtype dt, int device,
                                 rtr_kvcache **out);

/* Frees the buffers after synchronising the device.  NULL is ignored. */
void rtr_kvcache_destroy(rtr_kvcache *c);

/* Anchor (or overwrite in place) layer `layer`'s reference: copies
 * k_ref / v_ref, each [ref_frames*k][heads][head_dim], into the reference
 * slot and marks it valid.  The window is untouched.  RTR_E_STATE if the
 * cache has ref_frames == 0. */
rtr_status rtr_kvcache_set_reference(rtr_kvcache *c, int layer,
                                     const void *k_ref, const void *v_ref,
                                     rtr_stream_t stream);

/* Mark the reference of `layer` (or of every layer if layer == -1) absent:
 * TV2V, or a switch to a text-only condition.  No data moves. */
rtr_status rtr_kvcache_clear_reference(rtr_kvcache *c, int layer);

/* Append n_frames latent frames to layer `layer`: k_new / v_new are
 * [n_frames*k][heads][head_dim].  Frame f = frames_appended + i goes to slot
 * f mod S; once the window is full the oldest frames drop out of it
 * (eviction; with S == window_frames the new frame overwrites the evicted
 * one's slot); the reference slot is never written.  Then
 * frames_appended += n_frames and count = min(window_frames, count +
 * n_frames).  1 <= n_frames <= window_frames, else RTR_E_INVAL. */
rtr_status rtr_kvcache_append_frame(rtr_kvcache *c, int layer,
                                    const void *k_new, const void *v_new,
                                    int n_frames, rtr_stream_t stream);

/* Condition switch: keep only the n_frames most recent window frames of
 * `layer` (every layer if layer == -1): count = min(count, n_frames).  The
 * page keeps one frame as the bridge (n_frames = 1).  Index-map work only. */
rtr_status rtr_kvcache_retain_last(rtr_kvcache *c, int layer, int n_frames);

/* Host copy of layer `layer`'s index map.  slot_frame (S entries: window_frames
 * + commit_frames; may be NULL): frame index held by each slot, -1 if empty.
 * ref_valid (may be NULL): 1 if a reference is anchored.  frames_appended
 * (may be NULL): frames appended since creation.  count (may be NULL): frames
 * currently held. */
rtr_status rtr_kvcache_get_index_map(const rtr_kvcache *c, int layer,
                                     int32_t *slot_frame, int32_t *ref_valid,
                                     int64_t *frames_appended, int32_t *count);

/* Restore the index map of `layer`, e.g. after copying a snapshot's K / V
 * bytes back in through rtr_kvcache_device_ptrs: a stream saved with
 * rtr_kvcache_get_index_map and a device-to-host copy of the buffers resumes
 * from the same state (the pages' stream state is exactly this cache).
 * Requires 0 <= count <= min(window_frames, frames_appended), ref_valid 0 or
 * 1 (1 only with ref_frames > 0); else RTR_E_INVAL and nothing changes.  No
 * data moves: the caller restores the bytes of the slots the map names, at
 * the same physical slots (frame f in slot f mod S). */
rtr_status rtr_kvcache_set_index_map(rtr_kvcache *c, int layer,
                                     int64_t frames_appended, int32_t count,
                                     int32_t ref_valid);

/* Guard bands: every K / V buffer of a cache (and of a cross-attention cache)
 * is allocated with 64 KB on each side holding a fixed byte pattern.  These
 * synchronise the device and return RTR_OK if all bands are intact,
 * RTR_E_STATE if any byte changed (a kernel wrote outside its buffer), or
 * RTR_E_CUDA. */
rtr_status rtr_kvcache_check_guards(const rtr_kvcache *c);

/* Device pointers of layer `layer`'s K and V buffers (layout above), for
 * inspection and snapshotting.  The library keeps ownership. */
rtr_status rtr_kvcache_device_ptrs(const rtr_kvcache *c, int layer,
                                   void **k, void **v);

/* ---------------------------------------------------------------------------
 * Frame-causal attention of the current chunk (Key Designs 2 and 4).
 *
 * The chunk's queries q ([n_cur_frames*k][heads][head_dim]) attend to the
 * logical key sequence [reference (if anchored) | window frames oldest to
 * newest | the chunk's own k_cur / v_cur (same layout as q)].  Chunk frame c
 * sits at logical frame R' + count + c (R' = ref_frames if the reference is
 * valid, else 0), so under M it sees every cached key and chunk frames
 * 0..c.  out receives [n_cur_frames*k][heads][head_dim] in the cache's
 * element type.  scale <= 0 selects 1/sqrt(head_dim).  The cache is not
 * modified; commit the chunk afterwards with rtr_kvcache_append_frame.
 * Softmax is a permutation-invariant sum, so the kernel visits cached keys
 * in physical slot order; only the rounding order differs from the logical
 * order.
 */
rtr_status rtr_attn_frame_causal(const rtr_kvcache *c, int layer,
                                 const void *q, const void *k_cur,
                                 const void *v_cur, int n_cur_frames,
                                 void *out, float scale, rtr_stream_t stream);

/* rtr_attn_frame_causal with the MMA form chosen explicitly, as in
 * rtr_attn_block_causal_prefill_ex: cta_group 1 (the default kernel) or 2
 * (the CTA-pair kernel); other values RTR_E_INVAL. */
rtr_status rtr_attn_frame_causal_ex(const rtr_kvcache *c, int layer,
                                    const void *q, const void *k_cur,
                                    const void *v_cur, int n_cur_frames,
                                    void *out, float scale, int cta_group,
                                    rtr_stream_t stream);

/* rtr_attn_frame_causal with an fp32 output: out receives
 * [n_cur_frames*k][heads][head_dim] fp32, the normalised rows before the
 * bf16 rounding that rtr_attn_frame_causal applies (its bf16 output is
 * exactly these values rounded to nearest even).  The pages fix no output
 * precision; this entry point measures the bf16 path's error without its
 * final rounding.  out must be 16-byte aligned; ownership stays with the
 * caller.  On
 * an fp32 cache this is rtr_attn_frame_causal.  Errors as for
 * rtr_attn_frame_causal. */
rtr_status rtr_attn_frame_causal_f32out(const rtr_kvcache *c, int layer,
                                        const void *q, const void *k_cur,
                                        const void *v_cur, int n_cur_frames,
                                        float *out, float scale, rtr_stream_t stream);

/* rtr_attn_frame_causal followed by the commit of the chunk, as in
 * rtr_kvcache_append_frame(c, layer, k_cur, v_cur, n_cur_frames), with the
 * chunk written by the attention launch itself (Key Designs 4: the chunk's
 * K/V enter the rolling cache once it is generated).  The kernel already
 * holds each chunk key / value tile in shared memory to attend to it, so the
 * separate append's re-read of k_cur / v_cur and its launch go away.
 *
 * Call it for the last denoising step of a chunk; earlier steps use
 * rtr_attn_frame_causal.  Requires a cache from rtr_kvcache_create_ex with
 * commit_frames >= n_cur_frames (else RTR_E_INVAL): frames g..g+n-1 (g =
 * frames_appended) go to slots (g+i) mod S, which the held frames do not
 * occupy, so no key this call reads is overwritten.  On success the index
 * map advances exactly as after rtr_kvcache_append_frame; outputs and cache
 * bytes are those of the two separate calls.  For fp32 storage the commit
 * runs as a second kernel. */
rtr_status rtr_attn_frame_causal_commit(rtr_kvcache *c, int layer,
                                        const void *q, const void *k_cur,
                                        const void *v_cur, int n_cur_frames,
                                        void *out, float scale,
                                        rtr_stream_t stream);

/* See rtr_kvcache_check_guards. */
rtr_status rtr_crossattn_check_guards(const rtr_xattn *x);

/* Test hook: of the library's next device allocations (cache buffers,
 * scratch), let `after` succeed and make the `n` that follow fail as if the
 * device were out of memory, so that tests can reach every RTR_E_NOMEM path.
 * (0, 0) clears it.  Negative arguments: RTR_E_INVAL. */
rtr_status rtr_test_fail_allocs(int after, int n);

/* Block-causal attention over one whole sequence (Key Designs 2: training
 * sees all frames at once under M).  q, k, v, out: [n_tokens][heads]
 * [head_dim]; token i belongs to frame floor(i / k_per_frame).  scale <= 0
 * selects 1/sqrt(head_dim).  n_tokens == 0 is a no-op. */
rtr_status rtr_attn_block_causal_prefill(const void *q, const void *k,
                                         const void *v, int n_tokens,
                                         int heads, int head_dim,
                                         int k_per_frame, rtr_dtype dt,
                                         void *out, float scale,
                                         int device, rtr_stream_t stream);

/* rtr_attn_block_causal_prefill with the tensor-core kernel's MMA form
 * chosen explicitly: cta_group = 1 is the default kernel (one CTA per
 * 128-row MMA); cta_group = 2 runs the CTA-pair kernel (tcgen05
 * cta_group::2: one MMA covers 256 query rows on two SMs, each SM holding
 * half of every key / value tile).  Both return the same attention within
 * rounding; the CTA pair was measured slower and is kept for comparison.
 * Other values: RTR_E_INVAL.  fp32 ignores cta_group. */
rtr_status rtr_attn_block_causal_prefill_ex(const void *q, const void *k,
                                            const void *v, int n_tokens,
                                            int heads, int head_dim,
                                            int k_per_frame, rtr_dtype dt,
                                            void *out, float scale,
                                            int cta_group, int device,
                                            rtr_stream_t stream);

/* rtr_attn_block_causal_prefill that also returns each row's log-sum-exp,
 * the statistic the backward pass needs: lse[h * n_tokens + i] = log
 * sum_{j visible to i} exp(scale * q_i . k_j) (natural log), fp32
 * [heads][n_tokens], caller-owned device memory.  bf16 only
 * (RTR_E_UNSUPPORTED for RTR_F32). */
rtr_status rtr_attn_block_causal_prefill_lse(const void *q, const void *k,
                                             const void *v, int n_tokens,
                                             int heads, int head_dim,
                                             int k_per_frame, rtr_dtype dt,
                                             void *out, float *lse,
                                             float scale, int device,
                                             rtr_stream_t stream);

/* Block-causal prefill that also fills layer `layer` of cache c with the
 * sequence's K/V (papernotes.org note "DiT as Real-Time Rerenderer", Key
 * Designs 2 and 4: a context attended once under M becomes the cache that
 * streaming continues from).  q, k, v, out: [n_frames * k][heads][head_dim]
 * in the cache's element type, k, heads and head_dim; out is exactly what
 * rtr_attn_block_causal_prefill(q, k, v, n_frames * k, ..., k_per_frame = k)
 * returns.  The attention reads only this sequence, never the cache.
 *
 * with_reference = 1: the first R (ref_frames) frames are the reference.
 * They are written to the resident slot, which becomes valid; that needs
 * R >= 1, else RTR_E_STATE.  The remaining n_frames - R frames are appended
 * to the window as by rtr_kvcache_append_frame.  with_reference = 0: all
 * n_frames frames are appended and the reference slot is left as it is.
 * The appended count must be <= window_frames (else RTR_E_INVAL).  The
 * index map then reads as after rtr_kvcache_set_reference (when
 * with_reference = 1) followed by rtr_kvcache_append_frame.
 *
 * One launch attends and writes for bf16 caches, when with_reference = 0
 * or when frames_appended is a multiple of the ring's slot count (a fresh
 * cache, for instance).  Otherwise the copy kernels run after the
 * attention; if the second of those fails, the reference part stays
 * written.  Pointers are caller-owned device memory, 16-byte aligned. */
rtr_status rtr_attn_block_causal_prefill_cache(rtr_kvcache *c, int layer,
                                               const void *q, const void *k,
                                               const void *v, int n_frames,
                                               int with_reference, void *out,
                                               float scale,
                                               rtr_stream_t stream);

/* Weights of one DiT block (see rtr_dit_block_forward): bf16, row-major,
 * [in][out] so that y = x W + b; D = heads * head_dim of the cache, F =
 * d_ffn.  wqkv [D][3D] holds the q, k and v projections side by side (q in
 * columns [0, D), k in [D, 2D), v in [2D, 3D)); bqkv [3D]; wo, wq2, wo2 [D][D]
 * with biases bo, bq2, bo2 [D]; w1 [D][F], b1 [F]; w2 [F][D], b2 [D].  Every
 * pointer is caller-owned device memory, 16-byte aligned. */
typedef struct rtr_dit_weights {
    const void *wqkv, *bqkv;
    const void *wo, *bo;
    const void *wq2, *bq2;
    const void *wo2, *bo2;
    const void *w1, *b1;
    const void *w2, *b2;
    int d_ffn;
} rtr_dit_weights;

/* One DiT block on the current chunk of n_cur_frames latent frames
 * (papernotes.org note "DiT as Real-Time Rerenderer", Method > Overall
 * Architecture: the patchified tokens go through DiT blocks whose 3D
 * attention carries the temporal causal mask; Key Designs 1: text enters
 * through cross attention; Key Designs 4: the rolling caches).  hidden: the
 * chunk's tokens [n][D] bf16, n = n_cur_frames * k, updated in place to
 *
 *   h  = LN(x)(1 + scale1) + shift1;   q, k, v = h Wqkv + bqkv
 *   q, k rotated by the 3D rotary encoding of (frame t0 + i / k,
 *        row (i % k) / grid_w, column i % grid_w), grid_h * grid_w = k
 *   x1 = x + gate1 (A Wo + bo),  A = rtr_attn_frame_causal on cache c
 *   x2 = x1 + (A2 Wo2 + bo2),    A2 = rtr_attn_cross on x of (LN(x1) Wq2 + bq2)
 *   x3 = x2 + gate2 (GELU(h3 W1 + b1) W2 + b2),  h3 = LN(x2)(1 + scale2) + shift2
 *
 * LN: no affine, eps 1e-6.  GELU: tanh form.  Rotary encoding: each head's
 * d channels split into (frame, row, column) parts of d - 2P, P, P channels,
 * P = 2 floor(d / 6); pair (2j, 2j+1) of a part of size S turns by
 * pos * 10000^(-2j/S).  modulation: bf16 [6][D] = shift1, scale1, gate1,
 * shift2, scale2, gate2 (from the timestep, computed by the caller).  Every
 * tensor a later step consumes is stored in bf16; accumulation is fp32.
 * The six projections are this library's tensor-core GEMM with the bias,
 * rotary, GELU and gated-residual steps fused into its output stage (as
 * rtr_dit_qkv_rope and rtr_dit_linear).
 *
 * commit = 1 appends the chunk's rotated keys and values to the cache after
 * its attention, as rtr_kvcache_append_frame would (n_cur_frames <= W), in
 * the attention launch itself when the cache has that much commit room.
 * Requires bf16 caches of equal heads and head_dim on one device, text set
 * in x for this layer (else RTR_E_STATE), d_ffn a multiple of 8.  The
 * library keeps a per-stream activation buffer of about n * (10 D + 2 F)
 * bytes.  Argument errors leave everything unchanged; a CUDA error in a
 * step after the commit returns RTR_E_CUDA with the commit already applied
 * to the index map. */
rtr_status rtr_dit_block_forward(rtr_kvcache *c, const rtr_xattn *x, int layer,
                                 const rtr_dit_weights *w,
                                 const void *modulation, void *hidden,
                                 int n_cur_frames, int grid_h, int grid_w,
                                 int t0, int commit, rtr_stream_t stream);

/* The block's weights packed once for its projections.  Each matrix is
 * stored as the tensor core's shared-memory tiles, contiguously, so that a
 * projection moves a stage of weights with one bulk copy (or, on CTA-pair
 * tiles, one 16 KB box per CTA and K block) instead of one transfer per
 * 128-byte row (measured on B200: about 81 against 44-49 bytes per clock
 * per SM).  Weights are fixed during inference, so a caller packs
 * a block's weights once and passes the handle to every
 * rtr_dit_block_forward_packed call.  d_model = heads * head_dim and
 * w->d_ffn must be multiples of 64; pointers as for rtr_dit_block_forward.
 * The library allocates the packed copy (the six matrices and their biases,
 * about the size of the weights) on `device`; the call returns once packing
 * is done, after which the source weights may be freed or changed (the
 * handle keeps its own copy).  Release with rtr_dit_packed_destroy. */
typedef struct rtr_dit_packed rtr_dit_packed;
rtr_status rtr_dit_pack_weights(const rtr_dit_weights *w, int d_model,
                                int device, rtr_stream_t stream,
                                rtr_dit_packed **out);
void rtr_dit_packed_destroy(rtr_dit_packed *pw);

/* rtr_dit_block_forward with weights packed by rtr_dit_pack_weights: the
 * same block, bit for bit (each output element is the same K-ordered fp32
 * accumulation of the same products, whichever tile shape the projection
 * picks; only the operands' transfer differs).  pw must be packed for
 * d_model = heads * head_dim of c on c's device (else RTR_E_INVAL). */
rtr_status rtr_dit_block_forward_packed(rtr_kvcache *c, const rtr_xattn *x,
                                        int layer, const rtr_dit_packed *pw,
                                        const void *modulation, void *hidden,
                                        int n_cur_frames, int grid_h,
                                        int grid_w, int t0, int commit,
                                        rtr_stream_t stream);

/* The projections of the DiT block, for callers that assemble their own
 * blocks: out = epilogue(a w + bias) on the tensor cores, with the epilogue
 * applied to the fp32 product before anything is stored and each output
 * rounded once to bf16 (papernotes.org note "DiT as Real-Time Rerenderer",
 * Method > Overall Architecture).  a: bf16 [m][k] activations; w: bf16
 * [k][n] weights ([in][out], y = x w + b); bias: bf16 [n]; n and k
 * multiples of 8.
 *   RTR_EPI_BIAS            out[m][n] = a w + bias
 *   RTR_EPI_BIAS_GELU       out[m][n] = GELU_tanh(a w + bias)
 *   RTR_EPI_GATED_RESIDUAL  out[m][n] += gate * (a w + bias), in place;
 *                           gate bf16 [n], or null for 1
 * gate must be null for the other two.  Caller-owned device memory,
 * 16-byte aligned; out must not overlap a or w.  m == 0 is a no-op. */
typedef enum {
    RTR_EPI_BIAS = 0,
    RTR_EPI_BIAS_GELU = 1,
    RTR_EPI_GATED_RESIDUAL = 2
} rtr_epilogue;
rtr_status rtr_dit_linear(const void *a, const void *w, int m, int n, int k,
                          rtr_epilogue epilogue, const void *bias,
                          const void *gate, void *out, int device,
                          rtr_stream_t stream);

/* The block's QKV projection with the 3D rotary encoding fused: for the m
 * tokens of a chunk (a: bf16 [m][d_in]), the product with wqkv ([d_in][3D],
 * D = heads * head_dim; q, k and v side by side) plus bqkv ([3D]) is split
 * into q, k, v ([m][heads][head_dim] bf16 each), and q and k are turned by
 * the rotary encoding of token i at (frame t0 + i / k_per_frame, row
 * (i % k_per_frame) / grid_w, column i % grid_w), as rtr_dit_block_forward
 * describes.  head_dim 64 or 128; d_in a multiple of 8; 16-byte aligned
 * caller-owned device memory. */
rtr_status rtr_dit_qkv_rope(const void *a, const void *wqkv, const void *bqkv,
                            int m, int d_in, int heads, int head_dim,
                            int k_per_frame, int grid_w, int t0, void *q,
                            void *k, void *v, int device, rtr_stream_t stream);

/* The output tile rtr_dit_linear (epilogue as there) or, with qkv_rope = 1,
 * rtr_dit_qkv_rope picks for an m x n x k product on `device`: *rows x
 * *cols outputs per tile, *cta_pair = 1 when two CTAs of a cluster share
 * each tile (tcgen05 cta_group::2 MMAs, each CTA holding half the rows and
 * loading half the weight columns), and *ctas, the CTAs of the persistent
 * launch.  A planning query: it launches nothing (without a usable device
 * it plans for 148 SMs and no CTA pairs).  m, n, k >= 1; RTR_E_INVAL for
 * bad sizes or null outputs. */
rtr_status rtr_dit_linear_tile(int m, int n, int k, rtr_epilogue epilogue,
                               int qkv_rope, int device, int *rows, int *cols,
                               int *cta_pair, int *ctas);

/* The same planner for a hypothetical device, host arithmetic only: `sms`
 * SMs of which `pair_clusters` CTA pairs (clusters of two) can be resident
 * at once (0: pairs not available; at most sms / 2), weights packed by
 * rtr_dit_pack_weights (w_packed = 1, as rtr_dit_block_forward_packed
 * uses them) or row-major (0, as rtr_dit_linear and rtr_dit_block_forward
 * pass them).  Outputs as for rtr_dit_linear_tile; RTR_E_INVAL for bad
 * sizes or null outputs. */
rtr_status rtr_dit_plan_tile(int m, int n, int k, rtr_epilogue epilogue,
                             int qkv_rope, int w_packed, int sms,
                             int pair_clusters, int *rows, int *cols,
                             int *cta_pair, int *ctas);

/* Backward pass of the block-causal attention (Key Designs 2 and 3: the
 * causal student is trained with Self Forcing and DMD, whose gradients flow
 * through this attention).  Given the forward's inputs q, k, v, its output
 * out and row log-sum-exp lse (from rtr_attn_block_causal_prefill_lse, same
 * scale), and the upstream gradient dout, writes dq, dk, dv: the gradients
 * of sum(dout * out) with respect to q, k and v.  All tensors
 * [n_tokens][heads][head_dim] bf16 (lse fp32 [heads][n_tokens]); outputs
 * are computed in fp32 and rounded once to bf16.  Caller-owned device
 * memory, 16-byte aligned; the library uses a per-stream scratch buffer of
 * 8 * heads * n_tokens bytes (rounded up to 128-row tiles).  bf16 only
 * (RTR_E_UNSUPPORTED for RTR_F32); n_tokens == 0 is a no-op. */
rtr_status rtr_attn_block_causal_backward(const void *q, const void *k,
                                          const void *v, const void *out,
                                          const void *dout, const float *lse,
                                          int n_tokens, int heads,
                                          int head_dim, int k_per_frame,
                                          rtr_dtype dt, void *dq, void *dk,
                                          void *dv, float scale, int device,
                                          rtr_stream_t stream);

/* Block-causal prefill that allocates no device memory.  The paper has no
 * counterpart: this is a library addition for callers that cannot let a
 * library allocate -- e.g. a serving process whose device memory is reserved
 * up front by its own caching allocator, or a frame loop that must not stall
 * on the device-wide wait of cudaFree when rtr_attn_block_causal_prefill
 * grows its scratch buffer.
 *
 * Same arguments, layouts and results as rtr_attn_block_causal_prefill.  The
 * scratch (partial results of work split across SMs) lives in a static device
 * array of RTR_NOALLOC_SCRATCH_BYTES that every GPU loading the library holds
 * until process exit; a problem whose schedule needs more returns
 * RTR_E_INVAL (bf16, head_dim 128 on a 148-SM B200 needs 37.6 MiB at most).
 * The first call on a device looks up the array's device address; make that
 * first call before any stream capture.  All calls share the array: calls
 * that overlap on the GPU (different streams or host threads) race and must
 * be ordered by the caller.  No cudaMalloc, cudaFree or allocating library
 * routine is called. */
#define RTR_NOALLOC_SCRATCH_BYTES (40u << 20)
rtr_status rtr_attn_block_causal_prefill_noalloc(const void *q, const void *k,
                                                 const void *v, int n_tokens,
                                                 int heads, int head_dim,
                                                 int k_per_frame, rtr_dtype dt,
                                                 void *out, float scale,
                                                 int device,
                                                 rtr_stream_t stream);

/* ---------------------------------------------------------------------------
 * Cross-attention cache for the text condition (Key Designs 1 and 4).
 * Per layer K and V, each [heads][max_text][head_dim]; starts empty.
 */
rtr_status rtr_crossattn_create(int layers, int heads, int head_dim,
                                int max_text, rtr_dtype dt, int device,
                                rtr_xattn **out);
void rtr_crossattn_destroy(rtr_xattn *x);

/* Copy the projected text K / V ([n_text][heads][head_dim]) of `layer` into
 * the cache and mark it valid with n_text tokens (1 <= n_text <= max_text). */
rtr_status rtr_crossattn_set_text(rtr_xattn *x, int layer, const void *k_text,
                                  const void *v_text, int n_text,
                                  rtr_stream_t stream);

/* Condition switch: mark every layer's text cache empty (no data moves). */
rtr_status rtr_crossattn_reset(rtr_xattn *x);

/* Unmasked softmax attention of q ([n_q][heads][head_dim]) against layer
 * `layer`'s text keys; out as q.  RTR_E_STATE if the layer is empty. */
rtr_status rtr_attn_cross(const rtr_xattn *x, int layer, const void *q,
                          int n_q, void *out, float scale,
                          rtr_stream_t stream);

/* ---------------------------------------------------------------------------
 * Device status: synchronises `stream`, returns the latched device-side
 * status of `device` (RTR_OK or RTR_E_TIMEOUT) and clears it.
 */
rtr_status rtr_get_device_status(int device, rtr_stream_t stream);

/* ---------------------------------------------------------------------------
 * Scratch memory.  Calls that need scratch (split attention units, the
 * backward's row statistics, the DiT block's activations) keep one
 * library-owned device buffer per (stream, use), grown on demand and reused
 * by later calls on that stream.  A device keeps the buffers of its 8 most
 * recently used streams; the least recently used is freed (after a device
 * synchronisation) when a ninth stream needs one, so short-lived streams do
 * not accumulate buffers.  rtr_release_workspaces synchronises `device` and
 * frees all of its buffers now; *held_before (if not null) receives how many
 * there were.  Later calls allocate again as needed.
 */
rtr_status rtr_release_workspaces(int device, int *held_before);

/* Test hook for the failure path: the next `launches` bf16 attention
 * launches on `device` (any of the attention calls) deliberately issue no
 * loads.  Their bounded waits then expire after about one second each, the
 * kernel stops, frees its tensor memory and returns, and RTR_E_TIMEOUT is
 * latched for rtr_get_device_status.  The outputs of those launches are
 * unspecified.  No fault, trap or hang is involved; later launches run
 * normally.  launches == 0 cancels.  For tests only. */
rtr_status rtr_test_inject_wait_timeout(int device, int launches);

/* Number of kernels this library has launched since it was loaded (all
 * devices and streams).  Diagnostic: lets a caller count the launches of a
 * region of its own code. */
unsigned long long rtr_kernel_launches(void);

/* Library build information (static string). */
const char *rtr_build_info(void);

#ifdef __cplusplus
}
#endif
#endif /* RTR_H */
