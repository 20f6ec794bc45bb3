/*
 * nomas.h -- C ABI of the segment-causal joint attention library (sm_100a).
 *
 * One layer of a segment-autoregressive video MMDiT (Hy-Nomas): the current
 * segment's text and video tokens attend to each other and to a lifelong
 * key/value cache of earlier segments' video tokens; video positions carry
 * 3D RoPE. The cache holds either BF16 values (full history) or INT8 codes
 * with a per-(token, head) fp32 scale and a sliding window of latent frames.
 *
 * Sources (page title, section):
 *  - Hy-Nomas model card, "Segment-Autoregressive Diffusion Transformer":
 *    segment-wise causal joint attention with 3D RoPE and a per-layer KV
 *    cache supplying earlier segments; architecture table (16 heads x 128,
 *    RoPE split [16,56,56] over t/h/w, theta 256); "Attention is causal
 *    across segments"; cached keys and values are reused; full history
 *    (max_cache_segments=null) in the standard configuration.
 *  - same card, "Single-GPU Low-Memory Inference": INT8 KV storage with
 *    16-bit attention computation (the card names BF16; an INT8 cache is
 *    attended to here in FP16 with power-of-two exponents per query row and
 *    per 128-key tile, see nomas_seg_attn); a GPU history budget of 18
 *    latent frames.
 *  - "Hy-Nomas Explained" blog, "Segment-wise causal joint attention" and
 *    "Step 3: The Video Latent ...": 22 x 40 = 880 tokens per latent frame.
 *
 * Conventions for every call:
 *  - Pointers named "device" must point to device memory of the current
 *    CUDA device; the caller owns all memory. The library never allocates
 *    or frees memory, never synchronises (except nomas_device_status), and
 *    enqueues work only on the given stream (a cudaStream_t passed as
 *    void*; NULL means the legacy default stream).
 *  - Return value: NOMAS_OK (0) or a negative NOMAS_ERR_* code. All
 *    argument and state validation happens on the host before any launch:
 *    a call that returns an error has enqueued nothing and changed nothing.
 *  - BF16 tensors are passed as raw 16-bit patterns; layouts are row-major
 *    with the last index fastest.
 *  - Head dimension is fixed at 128 and the RoPE split at [16, 56, 56].
 *  - RoPE pairs are interleaved (2j, 2j+1) inside each axis block; pair j of
 *    a block of width d turns by pos * theta^(-2j/d). A video token's
 *    position is (t, h, w): t = absolute latent-frame index since the last
 *    nomas_cache_reset, (h, w) its grid cell; tokens of a frame are
 *    row-major (h, then w). Text tokens are not rotated.
 *  - A descriptor must not be used from two host threads at once. Device
 *    work of successive calls is ordered only by the stream(s) the caller
 *    passes.
 */
#ifndef NOMAS_H
#define NOMAS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---------------------------------------------------- */
#define NOMAS_OK 0
#define NOMAS_ERR_ARG (-1)       /* NULL pointer, bad size, head_dim != 128, ... */
#define NOMAS_ERR_ALIGN (-2)     /* pointer or stride not 16-byte aligned */
#define NOMAS_ERR_STATE (-3)     /* descriptor not reset, or changed since */
#define NOMAS_ERR_CAPACITY (-4)  /* full-history commit beyond capacity_frames */
#define NOMAS_ERR_WORKSPACE (-5) /* workspace NULL or smaller than required */
#define NOMAS_ERR_CUDA (-6)      /* a CUDA runtime/driver call failed */
#define NOMAS_ERR_DEVICE (-7)    /* current device is not sm_100 */
#define NOMAS_ERR_DEVICE_TIMEOUT (-8) /* a kernel gave up a bounded wait */

/* ---- cache modes ------------------------------------------------------ */
#define NOMAS_CACHE_BF16 0 /* cached K/V kept as BF16 (K after RoPE) */
#define NOMAS_CACHE_INT8 1 /* cached K/V as INT8 codes + fp32 per-(token, head) scales */

#define NOMAS_HEAD_DIM 128
#define NOMAS_MAX_GRID_HW 96 /* grid_h + grid_w limit (RoPE tables travel as launch arguments) */
#define NOMAS_MAX_CAMERA_TOKENS 4096 /* camera tokens per chunk accepted by nomas_camera_attn */

/*
 * One layer's K/V cache. The caller fills the configuration fields and the
 * device pointers, then calls nomas_cache_reset; the library maintains the
 * state fields afterwards (treat them as read-only).
 *
 * Slots: a slot holds one latent frame (grid_h * grid_w tokens). Cache
 * buffers are head-major:
 *   k, v      : [heads][capacity_frames * tokens_per_frame][128]
 *               int8 codes (INT8 mode) or BF16 bits (BF16 mode), device;
 *               16-byte aligned.
 *   k_scale,
 *   v_scale   : fp32 [heads][capacity_frames * tokens_per_frame], device,
 *               16-byte aligned (INT8 mode; must be NULL in BF16 mode).
 * window_frames > 0: the cache keeps only the last window_frames committed
 *   latent frames (FIFO at frame granularity); frame f lives in slot
 *   f mod window_frames; capacity_frames must equal window_frames.
 * window_frames == 0: full history; frame f lives in slot f and a commit
 *   that would pass capacity_frames fails with NOMAS_ERR_CAPACITY.
 * Eviction is bookkeeping only: an evicted slot is simply overwritten by a
 * later frame. Because slots fill from 0 and wrap only when full, the
 * visible history is always slots [0, valid_frames).
 */
typedef struct nomas_cache {
    /* configuration (caller) */
    int32_t mode;            /* NOMAS_CACHE_BF16 or NOMAS_CACHE_INT8 */
    int32_t heads;           /* attention heads (16 in Hy-Nomas) */
    int32_t head_dim;        /* must be 128 */
    int32_t grid_h, grid_w;  /* latent grid; tokens_per_frame = grid_h * grid_w */
    int32_t window_frames;   /* history budget in latent frames; 0 = full history */
    int32_t capacity_frames; /* slots allocated */
    float rope_theta;        /* 256 in Hy-Nomas */
    void *k, *v;             /* device, see above */
    float *k_scale, *v_scale;
    /* state (library) */
    int64_t frames_committed; /* absolute index of the next frame to commit */
    int32_t valid_frames;     /* frames visible to attention (slots [0, valid_frames)) */
    int32_t head_slot;        /* slot the next committed frame goes to */
    uint64_t check;           /* reset stamp over the configuration fields */
} nomas_cache;

/*
 * nomas_cache_reset -- validate the descriptor and empty the cache.
 * Host only: sets frames_committed = valid_frames = head_slot = 0 and stamps
 * the configuration. Cache memory is not touched (no kernel is launched).
 * Errors: NOMAS_ERR_ARG (c NULL, non-positive sizes, head_dim != 128,
 * unknown mode, window > 0 with capacity != window, grid_h + grid_w >
 * NOMAS_MAX_GRID_HW, theta <= 0, scales present in BF16 mode or missing in
 * INT8 mode), NOMAS_ERR_ALIGN (a buffer not 16-byte aligned).
 */
int nomas_cache_reset(nomas_cache *c);

/*
 * nomas_kv_commit -- append a finished segment's video K/V to the cache
 * (model card: cached keys and values are reused when generation advances;
 * single-GPU configuration: INT8 storage and an 18-frame history budget).
 *
 * k, v : device, BF16 bits, token-major [n_frames * tokens_per_frame][heads][128];
 *        consecutive tokens are token_stride elements apart
 *        (token_stride >= heads * 128, a multiple of 8); 16-byte aligned.
 *        Only video tokens are committed; text tokens are not cached.
 * n_frames : latent frames in the segment (>= 0; 0 is a no-op).
 * Frame i of the segment gets t = frames_committed + i. K is rotated with
 * 3D RoPE in fp32 (c, s = fp32 roundings of the double-precision cos/sin of
 * pos * theta^(-2j/d); y0 = fma(x0, c, -rn(x1*s)), y1 = fma(x0, s, rn(x1*c))),
 * V is not. INT8 mode: per (token, head) row of 128, absmax a, scale =
 * a / 127 (IEEE fp32 division; 0 when a == 0), code = round-half-even(x /
 * scale) clamped to [-127, 127]. BF16 mode: round-half-even to BF16.
 * With a window, frames of this segment that fall out of the window by its
 * end are not written. Host state is advanced at enqueue time.
 * Errors: NOMAS_ERR_ARG, NOMAS_ERR_ALIGN, NOMAS_ERR_STATE (descriptor not
 * reset or configuration changed), NOMAS_ERR_CAPACITY, NOMAS_ERR_CUDA.
 */
int nomas_kv_commit(nomas_cache *c, const void *k, const void *v, int64_t token_stride, int32_t n_frames,
                    void *stream);

/*
 * nomas_kv_commit_layers -- nomas_kv_commit of one finished segment into
 * n_layers per-layer caches at once (one launch per 128 layers instead of one
 * per layer). The pages describe the per-layer commit; batching the layers of
 * a model step is a service of this library.
 *   caches : host array of n_layers descriptors (distinct caches) that share
 *            mode, heads, grid, window, capacity, theta and ring state
 *            (frames_committed, valid_frames, head_slot), e.g. the layers of
 *            one model advanced in lockstep.
 *   k, v   : host arrays of n_layers device pointers, each laid out as for
 *            nomas_kv_commit, all with the same token_stride.
 * Every layer's cache receives exactly what nomas_kv_commit would write, and
 * every descriptor's state advances by n_frames.
 * Errors: as nomas_kv_commit, plus NOMAS_ERR_ARG (n_layers < 1, a NULL entry,
 * one cache given twice) and NOMAS_ERR_STATE (descriptors that differ in
 * configuration or state). All checks happen before anything is enqueued.
 */
int nomas_kv_commit_layers(nomas_cache *const *caches, const void *const *k, const void *const *v,
                           int64_t token_stride, int32_t n_layers, int32_t n_frames, void *stream);

/*
 * nomas_camera_attn -- per-latent-frame camera cross-attention (model card,
 * "Text and Camera Conditioning": after the video MLP of each double-stream
 * block the video tokens query the projected camera features; with per-chunk
 * camera attention and a chunk of one latent frame, each latent frame's
 * tokens see only their own chunk's camera tokens -- one token per latent
 * frame in the blog's reading, "Camera conditioning").
 *   out[i][h] = softmax_j(<q[i][h], k_cam[c][j][h]> / sqrt(128)) . v_cam[c][j][h]
 *   for video token i < n_frames * tokens_per_frame, head h, c = (i /
 *   tokens_per_frame) / chunk_frames, j < n_cam. No RoPE, no mask inside a
 *   chunk; fp32 arithmetic, BF16 output rounded to nearest even. With
 *   n_cam == 1 the output is that chunk's V exactly.
 * q     : device, BF16 bits, video tokens only, token-major [n_video][heads][128],
 *         q_stride elements between tokens (>= heads * 128, a multiple of 8).
 * k_cam, v_cam : device, BF16 bits, [ceil(n_frames / chunk_frames)][n_cam][heads][128],
 *         contiguous (projected camera keys and values).
 * out   : device, BF16 bits, [n_video][heads][128], out_stride elements between
 *         tokens (>= heads * 128, a multiple of 8); must not overlap the inputs.
 * All device pointers 16-byte aligned; 1 <= n_cam <= NOMAS_MAX_CAMERA_TOKENS;
 * chunk_frames >= 1; n_video * heads < 2^31. n_frames == 0 is a no-op.
 * Errors: NOMAS_ERR_ARG, NOMAS_ERR_ALIGN, NOMAS_ERR_DEVICE, NOMAS_ERR_CUDA;
 * all checks happen before the launch.
 */
int nomas_camera_attn(const void *q, int64_t q_stride, int32_t n_frames, int32_t tokens_per_frame, int32_t heads,
                      const void *k_cam, const void *v_cam, int32_t n_cam, int32_t chunk_frames, void *out,
                      int64_t out_stride, void *stream);

/*
 * Archive of frames leaving a window (model card, "Segment-Autoregressive
 * Diffusion Transformer" and "Single-GPU Low-Memory Inference": the single-GPU
 * configuration attends over a bounded set of history frames on the GPU and
 * keeps earlier history in an archive in system memory).
 *
 * nomas_kv_evicted_frames -- the frames that the next nomas_kv_commit(c, ...,
 * n_frames) drops from the window: *count frames, absolute indices
 * *first_frame, *first_frame + 1, ... (the oldest frames of the window, in
 * order). Host only: no GPU work, no device needed. With no window
 * (window_frames == 0) nothing is ever dropped (*count = 0). Frames of the
 * segment being committed that fall out of the window by its end (a segment
 * longer than the window) never enter the cache and are not counted.
 * Errors: NOMAS_ERR_ARG (n_frames < 0, NULL outputs), NOMAS_ERR_STATE, and
 * the descriptor checks of nomas_cache_reset.
 */
int nomas_kv_evicted_frames(const nomas_cache *c, int32_t n_frames, int32_t *count, int64_t *first_frame);

/*
 * nomas_kv_archive_evicted -- enqueue on `stream` device-to-host copies of the
 * frames nomas_kv_evicted_frames reports, out of the cache, as they are now.
 * Call it before that commit, on the commit's stream (or order the two
 * streams with an event), so that the copies read the frames before the
 * commit overwrites their slots. The caller owns the host buffers (pinned
 * memory makes the copies asynchronous; pageable memory works but the call
 * then waits for them). Archived frame i (0 <= i < *count) is stored
 * frame-major, in the cache's own encoding:
 *   host_k, host_v             : [count][heads][tokens_per_frame][128]
 *                                int8 codes (INT8 mode) or BF16 bits;
 *   host_k_scale, host_v_scale : [count][heads][tokens_per_frame] fp32
 *                                (INT8 mode; ignored and may be NULL in BF16 mode).
 * max_frames : frames the host buffers hold. *count and *first_frame are set
 * whenever the descriptor validates, also when the call then fails with
 * NOMAS_ERR_CAPACITY (*count > max_frames), so a caller can size its buffers.
 * *count == 0 enqueues nothing and needs no buffers.
 * Errors: NOMAS_ERR_ARG, NOMAS_ERR_STATE, NOMAS_ERR_CAPACITY,
 * NOMAS_ERR_DEVICE, NOMAS_ERR_CUDA; all checks happen before any copy.
 */
int nomas_kv_archive_evicted(const nomas_cache *c, int32_t n_frames, void *host_k, void *host_v,
                             float *host_k_scale, float *host_v_scale, int32_t max_frames, int32_t *count,
                             int64_t *first_frame, void *stream);

/*
 * nomas_seg_attn_workspace_bytes -- device workspace of the fastest plan of
 * nomas_seg_attn for this cache state and segment shape (0 on invalid
 * arguments): the rotated Q and K, the KV-split partials, and for an INT8
 * cache the tile exponent records, the Q row factors and an FP16 copy of the
 * visible window (2 * heads * visible_tokens * 256 bytes), which is then
 * converted once per call instead of in shared memory by every CTA that
 * reads a tile.
 * nomas_seg_attn_workspace_min_bytes -- the smallest workspace nomas_seg_attn
 * accepts: one KV split and no copy (an INT8 window is converted tile by
 * tile inside the attention kernel, to the same FP16 values).
 * Any size in between is accepted; nomas_seg_attn then runs the fastest plan
 * that fits (the copy first, then fewer KV splits). The first 256 bytes of a
 * workspace are a status header: zero them once before first use; the
 * library only sets error bits in it.
 */
size_t nomas_seg_attn_workspace_bytes(const nomas_cache *c, int32_t n_video_frames, int32_t n_text);
size_t nomas_seg_attn_workspace_min_bytes(const nomas_cache *c, int32_t n_video_frames, int32_t n_text);

/*
 * nomas_seg_attn -- segment-causal joint attention of the current segment
 * (model card: the current segment attends to all past KV cache and to
 * itself; attention is causal across segments, bidirectional inside one).
 *
 * q, k, v : device, BF16 bits, token-major [Nq][heads][128] with
 *           Nq = n_video_frames * tokens_per_frame + n_text, video tokens
 *           first; token_stride elements between tokens (>= heads*128,
 *           multiple of 8); 16-byte aligned. Video frame i of the segment
 *           has t = c->frames_committed + i (the segment directly follows
 *           the committed history).
 * out     : device, BF16 bits [Nq][heads][128] (contiguous), 16-byte aligned.
 * lse     : optional device fp32 [heads][Nq]: natural-log sum of exp of the
 *           scaled scores; NULL to skip.
 * For each head and query i: out_i = sum_j softmax_j(<R(p_i) q_i, k_j> / sqrt(128)) v_j
 * over the visible cached tokens (INT8 mode: code * scale) and all Nq
 * tokens of the current segment (keys rotated with their own positions).
 * The cache is read only; accumulation is fp32. BF16 cache: Q and current K
 * are rounded to BF16 after RoPE and the probabilities are BF16 for the P.V
 * product. INT8 cache: every tensor-core operand is FP16 times a power of
 * two held in fp32 -- Q per row, the current K per 128-key tile, the cache
 * K and V as code * RN16(scale * 2^-e) with one exponent e per 128-key tile
 * -- and the probabilities are FP16 for cache tiles and BF16 for the current
 * segment's tiles (whose V is the caller's BF16). Per-token scales more than
 * 2^100 apart within a head are outside this path's range.
 * workspace : device, >= nomas_seg_attn_workspace_min_bytes(...) bytes (a
 *             larger one selects a faster plan, up to
 *             nomas_seg_attn_workspace_bytes(...)), 256-byte aligned, not
 *             shared with a call running concurrently.
 * Errors: NOMAS_ERR_ARG, NOMAS_ERR_ALIGN, NOMAS_ERR_STATE,
 * NOMAS_ERR_WORKSPACE, NOMAS_ERR_DEVICE, NOMAS_ERR_CUDA.
 */
int nomas_seg_attn(const nomas_cache *c, const void *q, const void *k, const void *v, int64_t token_stride,
                   int32_t n_video_frames, int32_t n_text, void *out, float *lse, void *workspace,
                   size_t workspace_bytes, void *stream);

/*
 * nomas_device_status -- synchronise `stream`, read and clear the status
 * header of a workspace. Returns NOMAS_OK, NOMAS_ERR_DEVICE_TIMEOUT (a
 * kernel abandoned a bounded wait; its outputs are invalid) or
 * NOMAS_ERR_CUDA. This is the only call that blocks the host.
 */
int nomas_device_status(void *workspace, void *stream);

/*
 * nomas_seg_attn_static -- nomas_seg_attn for callers that cannot allocate
 * device memory. The pages have no counterpart to this call: it is a service
 * of this library. Some callers cannot provide the device workspace that
 * nomas_seg_attn needs: an operator plugin whose host framework passes it
 * only its inputs and outputs, or code running where a cudaMalloc would
 * synchronise the device or fail because all device memory is already
 * reserved. This call takes its scratch from a fixed array in the library's
 * device image instead: NOMAS_STATIC_SCRATCH_BYTES per GPU, held by every GPU
 * that loads the library until the process exits.
 *
 * Arguments, layouts, results and errors are those of nomas_seg_attn, minus
 * the workspace. The fixed array serves as a workspace of
 * NOMAS_STATIC_SCRATCH_BYTES: the call runs the fastest plan that fits in it
 * (as nomas_seg_attn does for any workspace size), and a shape whose minimum
 * exceeds it is rejected with NOMAS_ERR_WORKSPACE before anything is
 * enqueued. The call allocates and frees nothing.
 * The first call in a CUDA context (with that context current) sets the
 * array up: it looks up its device address and clears its status header
 * with an asynchronous memset on `stream`, ahead of the call's kernels; make
 * that first call before any stream capture. The set-up is redone in a new
 * context (after a device reset, for instance). All calls share the one
 * array and it keeps the last call's contents, so calls that overlap on the
 * GPU race with each other: order them (one stream, or events), the first
 * call included. Bounded device waits of this call that run out are reported
 * by nomas_seg_attn_static_status, not by nomas_device_status.
 */
#define NOMAS_STATIC_SCRATCH_BYTES (64u << 20)
int nomas_seg_attn_static(const nomas_cache *c, const void *q, const void *k, const void *v, int64_t token_stride,
                          int32_t n_video_frames, int32_t n_text, void *out, float *lse, void *stream);

/*
 * nomas_seg_attn_static_status -- nomas_device_status for the fixed array of
 * nomas_seg_attn_static in the current context: synchronise `stream`, read
 * and clear the array's status header. Returns NOMAS_OK,
 * NOMAS_ERR_DEVICE_TIMEOUT (a call's kernel abandoned a bounded wait; its
 * outputs are invalid) or NOMAS_ERR_CUDA. It sets the array up first if no
 * static call has run in this context yet. No counterpart on the pages: a
 * service of this library, like the static call itself.
 */
int nomas_seg_attn_static_status(void *stream);

/*
 * nomas_selftest_bounded_wait -- run the bounded-wait failure path of the
 * kernels on the device, without any fault. The pages have no counterpart:
 * this is a diagnostic of the library's failure detection. It enqueues one
 * tiny kernel on `stream` whose first role waits on an mbarrier that nothing
 * arrives on; after NOMAS_WAIT_NS (2 s) of device time the wait gives up,
 * sets the status bit in word 0 of `workspace` and raises the CTA's abort
 * flag, and the second role, waiting on another such barrier, returns on
 * seeing that flag.
 *   workspace  device pointer, 16-byte aligned, at least 16 bytes: word 0 is
 *              the status word read by nomas_device_status; the call clears
 *              words 1 and 2 and the kernel sets word 1 when the first role
 *              gave up and word 2 when the second role returned on the abort
 *              flag. Word 0 is not cleared first (status bits accumulate).
 * Returns NOMAS_OK once enqueued (then nomas_device_status on the same
 * workspace and stream returns NOMAS_ERR_DEVICE_TIMEOUT), NOMAS_ERR_ARG for a
 * null or unaligned workspace, NOMAS_ERR_CUDA if the launch fails.
 */
int nomas_selftest_bounded_wait(void *workspace, void *stream);

/*
 * nomas_selftest_div127 -- check on the device, for every non-negative fp32
 * bit pattern x (2^31 inputs), that the division the INT8 commit uses for its
 * row scale (absmax / 127 by Markstein's method: a product with RN(1/127), an
 * exact remainder by fma, one correction) returns the IEEE fp32 quotient
 * RN(x / 127) bit for bit. The pages have no counterpart: this is a
 * diagnostic of the library's commit arithmetic.
 *   result  device pointer, 8-byte aligned, two uint32 words: the call sets
 *           word 0 to the number of inputs whose results differ (NaN equals
 *           NaN) and word 1 to the smallest such input pattern (0xFFFFFFFF
 *           when there is none), once `stream` has passed the call.
 * Returns NOMAS_OK once enqueued, NOMAS_ERR_ARG for a null or unaligned
 * pointer, NOMAS_ERR_CUDA if a launch fails.
 */
int nomas_selftest_div127(void *result, void *stream);

/* Human-readable name of a status code (static storage). */
const char *nomas_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* NOMAS_H */
