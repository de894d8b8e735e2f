/*
 * fs_stream.h -- C ABI of the streaming KV-cache attention library (B200, sm_100a).
 *
 * One fs_stream_t holds one layer's streaming KV cache for a window of
 * `views` cameras x `frames` frames x `tok_per_frame` tokens, followed by
 * `text_len` text tokens, and runs the attention of a window's new tokens
 * against it. The method follows FlashDrive (arXiv 2608.12932):
 *   - "Streaming inference": each frame's KV cache is reused across windows,
 *     so a window step only adds its latest frame (FlashDrive README,
 *     z-lab/flashdrive, technique list).
 *   - View-major token layout with per-view insertion and a streaming causal
 *     mask (FlashDrive technical summary, gist.science, Methodology 1,
 *     "Token Layout").
 *   - Keys stored pre-RoPE and rotated on the fly at their shifted positions
 *     (same page, Methodology 1, "Positional Encoding").
 *   - The first call of a stream only prefills (FlashDrive README, "Library").
 *
 * Conventions shared by every call:
 *   - Inputs (Q, K, V) are bf16 (IEEE bfloat16 bit patterns); attention
 *     outputs are fp32 (see fs_stream_attend). All tensors are contiguous,
 *     row-major, in device memory unless the call says "host". The caller owns
 *     them and keeps them alive until the enqueued work has completed.
 *   - Token order: view 0's tokens, view 1's, ..., then the text tokens.
 *   - Q and out are [tokens][H][d]; K and V are [tokens][Hkv][d].
 *   - Query head h reads kv head h / (H/Hkv) (contiguous GQA groups).
 *   - Q, K and V are passed pre-RoPE; the library applies rotate-half RoPE
 *     (pair (i, i+d/2), angle pos * rope_base^(-2i/d)) itself.
 *   - Positions are indices in the current view-major window (0 .. L-1 with
 *     L = views*frames*tok_per_frame + text_len); query p sees key q iff
 *     pos(q) <= pos(p).
 *   - Work is enqueued asynchronously on the stream set with
 *     fs_stream_set_stream (default: the legacy default stream). Only
 *     fs_stream_sync, fs_stream_debug_export and fs_stream_destroy block.
 *   - Every call returns FS_OK or a negative FS_ERR_* code. A failed call
 *     changes no state (the ring head does not advance). The message of the
 *     last failure is available from fs_stream_last_error (per handle) or
 *     fs_last_error (calling thread, for failures without a handle).
 *   - A handle is not thread-safe: one host thread at a time per handle.
 *   - Supported input range. The tensor-core operands are fp16 (11-bit
 *     significands, largest finite value 65504): V as fp16; each rotated key
 *     element as an fp16 hi + lo pair; each rotated query element, scaled by
 *     log2(e)/sqrt(d), as an fp16 hi + lo pair. Rotation mixes the pair
 *     (i, i+d/2), so a rotated element is at most sqrt(2) times the larger of
 *     the two. Inputs are therefore supported when they are finite and
 *       |V| <= 65504,  |K| <= 46318 (65504/sqrt(2)),
 *       |Q| <= 46318 * sqrt(d) / log2(e)  (363,000 at d = 128; 256,000 at d = 64).
 *     The kernels check every converted element; one out of range (or NaN)
 *     sets a flag that the next fs_stream_sync or fs_stream_debug_export
 *     reports as FS_ERR_RANGE (the outputs since the previous check are then
 *     not valid; the flag is cleared).
 */
#ifndef FS_STREAM_H
#define FS_STREAM_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FS_OK                   0
#define FS_ERR_ARG             -1 /* null pointer, unsupported size, bad shape            */
#define FS_ERR_STATE           -2 /* call not valid in the stream's current state          */
#define FS_ERR_CUDA            -3 /* a CUDA runtime/driver call failed (message has it)    */
#define FS_ERR_DEVICE_TIMEOUT  -4 /* a bounded device-side wait gave up (no hang)          */
#define FS_ERR_OOM             -5 /* device or host allocation failed                       */
#define FS_ERR_RANGE           -6 /* an input exceeded the supported range (see below)      */

/* Stream states. */
#define FS_STATE_EXPECT_PREFILL 0 /* after create/reset: insert takes the whole window     */
#define FS_STATE_PREFILLED      1 /* window inserted, attend takes all L queries (causal)  */
#define FS_STATE_STREAMING      2 /* insert takes one new frame per view plus the text     */

/* Largest drafted block fs_stream_attend_ext accepts. */
#define FS_MAX_VERIFY_TOKENS 256
/* Largest persisted decode tail (accepted tokens after the text, fs_stream_append). */
#define FS_MAX_TAIL_TOKENS 1024

typedef struct fs_stream* fs_stream_t;

/* Sizes and state of a handle (filled by fs_stream_info). */
typedef struct fs_stream_info_t {
    int views, frames, tok_per_frame, text_len, H, Hkv, d;
    int window_len;      /* L = views*frames*tok_per_frame + text_len                    */
    int step_tokens;     /* views*tok_per_frame + text_len                               */
    int state;           /* FS_STATE_*                                                   */
    int insert_tokens;   /* tokens the next fs_stream_insert expects (L or step_tokens)  */
    int query_tokens;    /* queries the next fs_stream_attend expects (0: none allowed)  */
    int head;            /* ring slot holding each view's oldest frame                   */
    long long steps;     /* window steps inserted since the prefill                      */
    long long cache_bytes; /* device bytes owned by the handle (the shared RoPE table aside) */
    long long launches;  /* kernels this handle has launched since create                 */
    int tail_tokens;     /* persisted decode-tail tokens after the text (fs_stream_append)  */
    int rebase_every;    /* R: every R-th window step re-rotates the whole window           */
} fs_stream_info_t;

/*
 * fs_stream_create -- allocate one layer's static KV cache (FlashDrive README,
 * "System optimizations": static KV cache) on the current CUDA device.
 *   views, frames, tok_per_frame >= 1; text_len >= 0; H, Hkv >= 1 with H % Hkv == 0
 *   and 128 % (H/Hkv) == 0; d in {64, 128}; rope_base > 0 (10000 in the
 *   synthetic workloads). L + FS_MAX_TAIL_TOKENS + FS_MAX_VERIFY_TOKENS must be
 *   <= 262144 (2048 key tiles of 128 rows per kv head).
 * Device layout of the cache (owned by the handle, zero-initialised):
 *   K_cache, V_cache [Hkv][R][d] bf16 with R = L + FS_MAX_TAIL_TOKENS +
 *   FS_MAX_VERIFY_TOKENS rows per kv head: rows [0, views*frames*tok_per_frame)
 *   are the per-view rings (view v, slot s, token i at row
 *   (v*frames + s)*tok_per_frame + i), then text_len text rows, then the
 *   persisted decode tail, then scratch rows for a drafted block.
 *   Next to it the handle keeps the attention operands (each key rotated once,
 *   as fp16 hi + lo, and V as fp16, same layout), a device-resident ring state
 *   (head slot and step count, advanced by the insert kernel) and split-KV
 *   scratch. The cos/sin table is shared by handles of the same device, d,
 *   rope_base and size.
 * Keys are rotated once, when they enter the cache, at angle index p + k*n
 * (p: window position, k: window steps since the last re-base); queries at
 * their position + k*n. Every R-th window step (R = 16, or FS_REBASE_STEPS in
 * the environment at create, 1..4096) re-rotates the whole window at k = 0.
 * On success *out receives the handle and the state is FS_STATE_EXPECT_PREFILL.
 * Errors: FS_ERR_ARG, FS_ERR_OOM, FS_ERR_CUDA (nothing is leaked).
 */
int fs_stream_create(fs_stream_t* out, int views, int frames, int tok_per_frame, int text_len,
                     int H, int Hkv, int d, float rope_base);

/* Free everything the handle owns after synchronising its stream. NULL is a no-op. */
int fs_stream_destroy(fs_stream_t s);

/* Enqueue subsequent work on `cuda_stream` (a cudaStream_t; NULL = legacy default stream). */
int fs_stream_set_stream(fs_stream_t s, void* cuda_stream);

/* Back to FS_STATE_EXPECT_PREFILL: the next insert is a whole window again. Cache
 * contents are left in place but are no longer visible. */
int fs_stream_reset(fs_stream_t s);

/*
 * fs_stream_insert -- write pre-RoPE K/V into the cache (kernel kv_stream_insert).
 *   State EXPECT_PREFILL: K_new, V_new are [L][Hkv][d], the whole window in
 *     view-major order (each view's frames oldest first, then text). Frame f of
 *     each view goes to ring slot f, the head is set to slot 0 (oldest) and the
 *     state becomes PREFILLED.
 *   State PREFILLED or STREAMING: K_new, V_new are [step_tokens][Hkv][d]: the
 *     newest frame of view 0, of view 1, ..., then the fresh text. Each view's
 *     new frame overwrites the slot of that view's oldest frame (evict-oldest,
 *     "inserted at the end of each view's sequence", FlashDrive technical
 *     summary, Methodology 1, "Token Layout"); the text overwrites the text
 *     rows; the head advances by one slot and the state becomes STREAMING.
 * Pointers must be 16-byte aligned device pointers. Errors: FS_ERR_ARG,
 * FS_ERR_CUDA.
 */
int fs_stream_insert(fs_stream_t s, const void* K_new, const void* V_new);

/*
 * fs_stream_insert_batch -- fs_stream_insert for n layers in one kernel launch
 * (FlashDrive README, "System optimizations": static KV cache; one launch per
 * window step instead of one per layer). handles[i] receives K_new[i] and
 * V_new[i] (device pointers, sizes as for fs_stream_insert). All handles must
 * share the window shape, Hkv, d, rope_base, device and stream (handles[0]'s
 * stream runs the launch), be distinct, and be all in EXPECT_PREFILL or all
 * past it. Each layer's device ring state advances as in fs_stream_insert.
 * Errors: FS_ERR_ARG (nothing enqueued), FS_ERR_STATE, FS_ERR_CUDA.
 */
int fs_stream_insert_batch(fs_stream_t* handles, int n, const void* const* K_new, const void* const* V_new);

/*
 * fs_stream_insert_proj -- fs_stream_insert with the K/V projection fused in
 * (FlashDrive README, "System optimizations": fused projections; technical
 * summary, System Optimizations, "Kernel Fusion"). X holds the tokens' hidden
 * states instead of their K and V:
 *   X [tokens][d_model] bf16 (device; tokens = L on the prefill, else
 *   step_tokens, in fs_stream_insert's token order), W [2*Hkv*d][d_model] bf16
 *   (a linear layer's weight: rows 0 .. Hkv*d-1 give K, the rest V; head h of K
 *   is rows h*d .. h*d + d - 1). K = X W_k^T and V = X W_v^T are computed on the
 *   tensor cores in fp32, each element rounded once to bf16 (nearest, ties to
 *   even) and written into the ring exactly as fs_stream_insert writes K_new /
 *   V_new, state transitions included. d_model must be a multiple of 8.
 * Pointers: 16-byte aligned device pointers. Errors: FS_ERR_ARG, FS_ERR_CUDA.
 */
int fs_stream_insert_proj(fs_stream_t s, const void* X, const void* W, int d_model);

/*
 * fs_stream_attend -- attention of the last inserted tokens (kernel stream_attn).
 *   State PREFILLED: Q and out are [L][H][d]; query t sits at position t
 *     (plain causal attention over the view-major window).
 *   State STREAMING: Q and out are [step_tokens][H][d]; view v's new-frame
 *     token i sits at v*frames*tok_per_frame + (frames-1)*tok_per_frame + i,
 *     text token j at views*frames*tok_per_frame + j.
 * Keys are every cached token at its current window position, rotated on the
 * fly (FlashDrive technical summary, Methodology 1, "Positional Encoding");
 * scores are scaled by 1/sqrt(d). out is fp32 [tokens][H][d]: a bf16 store
 * would itself be off by up to half a bf16 ulp (2^-5 / 2 for |x| in [4, 8)),
 * more than the 1e-2 max-abs accuracy the path is held to.
 * Pointers: 16-byte aligned device pointers; out must not alias Q.
 * Errors: FS_ERR_ARG, FS_ERR_STATE (nothing inserted yet), FS_ERR_CUDA.
 */
int fs_stream_attend(fs_stream_t s, const void* Q, void* out);

/*
 * fs_stream_append -- persist n_acc accepted tokens (pre-RoPE K/V, [n_acc][Hkv][d]
 * bf16, device) at the end of the decode tail: the tokens a verified drafted
 * block contributed (FlashDrive README, "Speculative reasoning (DFlash)";
 * technical summary, Methodology 2: blocks of 8 drafted tokens, 5.6 accepted on
 * average). Tail token j sits at position L + j, after the text; every later
 * drafted block sees it. The next window insert (fs_stream_insert or
 * fs_stream_insert_batch) empties the tail: a new window starts a new
 * reasoning pass. tail + n_acc <= FS_MAX_TAIL_TOKENS.
 * State: PREFILLED or STREAMING. Errors: FS_ERR_ARG, FS_ERR_STATE, FS_ERR_CUDA.
 */
int fs_stream_append(fs_stream_t s, const void* K_acc, const void* V_acc, int n_acc);

/*
 * fs_stream_attend_ext -- verify a drafted block of n_x tokens in one forward
 * (FlashDrive README, "Speculative reasoning (DFlash)"; technical summary,
 * Methodology 2). The block's tokens sit at positions L + tail .. L + tail +
 * n_x - 1, after the text and the persisted decode tail; each sees the whole
 * cached window, the tail and, causally, the block.
 *   Q_x [n_x][H][d] bf16, out [n_x][H][d] fp32; K_x, V_x [n_x][Hkv][d] bf16
 *   (pre-RoPE); 1 <= n_x <=
 *   FS_MAX_VERIFY_TOKENS. The block's K/V go to the handle's scratch rows and are
 *   not kept: the window is unchanged afterwards.
 * State: PREFILLED or STREAMING. Errors: FS_ERR_ARG, FS_ERR_STATE, FS_ERR_CUDA.
 */
int fs_stream_attend_ext(fs_stream_t s, const void* Q_x, const void* K_x, const void* V_x,
                         int n_x, void* out);

/*
 * fs_stream_attend_ext_static -- fs_stream_attend_ext without any allocation.
 * The paper has no counterpart: this is a deployment variant for callers that
 * may not allocate device memory per call (a drafting / verification loop
 * under a device-memory budget fixed at start-up, where cudaMalloc / cudaFree
 * could synchronise the device and stall a step).
 *   Arguments, layouts, state rules and results are those of
 *   fs_stream_attend_ext (out equal within rounding: the key range may be split
 *   fewer times). The split-KV partials live in one fixed device array in the
 *   library (64 partial tiles of 128 query rows: 4 MiB + 64 KiB), not in the
 *   handle; no cudaMalloc, cudaFree or allocating library routine is called.
 *   Limit: 2 * ceil(ceil(n_x * H/Hkv / 128) / 2) * Hkv <= 64 (at H/Hkv = 4 and
 *   Hkv = 8: every n_x <= FS_MAX_VERIFY_TOKENS); larger calls fail with
 *   FS_ERR_ARG and a message naming the limit, before any work is enqueued.
 *   Set-up: the first call on a device looks up the array's address
 *   (cudaGetSymbolAddress, with that device current); make that first call
 *   before any stream capture on the device.
 *   Sharing: every call on a device uses the same array, which keeps the last
 *   call's contents (nothing in it needs to start at zero: each call writes
 *   every partial it reads). Calls that overlap on the GPU (other streams,
 *   other handles) race on the array; serialise them.
 * State: PREFILLED or STREAMING. Errors: FS_ERR_ARG, FS_ERR_STATE, FS_ERR_CUDA.
 */
int fs_stream_attend_ext_static(fs_stream_t s, const void* Q_x, const void* K_x, const void* V_x,
                                int n_x, void* out);

/*
 * fs_frame_attend -- the vision encoder's attention over the newest frame of
 * each view (FlashDrive technical summary, Methodology 1, "Algorithmic
 * Shortcut": a window step encodes only each camera's newest frame and reuses
 * the rest). For view v, token t of its frame attends to every token of the
 * same frame -- bidirectional, nothing of other views, no rotation (the pages
 * name no encoder internals; plain softmax attention is the reading taken),
 * scores scaled by 1/sqrt(d), query head h reading kv head h / (H/Hkv).
 *   Q [views * tok_per_frame][H][d] bf16, K and V [views * tok_per_frame][Hkv][d]
 *   bf16 (token t of view v at row v * tok_per_frame + t, device);
 *   out [views * tok_per_frame][H][d] fp32. views and tok_per_frame are the
 *   handle's; H, Hkv, d are the encoder's (H % Hkv == 0, 128 % (H/Hkv) == 0,
 *   d in {64, 128}). The handle supplies the stream and the error word only;
 *   its cache is not touched and its state does not matter.
 * Range: |V| <= 65504 (V is converted to fp16 for P V); checked, reported by
 * fs_stream_sync as FS_ERR_RANGE.
 * Errors: FS_ERR_ARG, FS_ERR_CUDA.
 */
int fs_frame_attend(fs_stream_t s, const void* Q, const void* K, const void* V, int H, int Hkv, int d, void* out);

/*
 * fs_stream_step_host -- one insert + attend with HOST buffers: copies K_new,
 * V_new and Q (bf16) to the device (staging buffers owned by the handle), runs
 * fs_stream_insert and fs_stream_attend on the handle's stream, and copies out
 * back. The uploads run on a copy stream of the handle (after the previous
 * call's kernels have read the staging buffer) and the download on a second
 * one, so consecutive calls on different handles overlap uploads, kernels and
 * downloads. Sizes follow the current state exactly as for fs_stream_insert /
 * fs_stream_attend; out_h receives fp32. The staging buffers and copy streams
 * are created on the first call (buffers grown if a later call needs more), so
 * make the first call outside any stream capture. With pinned host memory the
 * call is asynchronous; out_h is complete once fs_stream_sync(s) returns.
 * Errors: as fs_stream_insert and fs_stream_attend.
 */
int fs_stream_step_host(fs_stream_t s, const void* K_new_h, const void* V_new_h,
                        const void* Q_h, void* out_h);

/* Block until the handle's enqueued work (its stream and host-path copy streams)
 * is done. Returns FS_ERR_DEVICE_TIMEOUT if a kernel of this handle gave up on a
 * bounded wait since the last check, FS_ERR_RANGE if an input was outside the
 * supported range (see the conventions above; the flags are cleared), FS_ERR_CUDA
 * on an asynchronous CUDA error. */
int fs_stream_sync(fs_stream_t s);

/* Sizes and state. */
int fs_stream_info(fs_stream_t s, fs_stream_info_t* info);

/*
 * fs_stream_debug_export -- synchronous copy of the physical cache to HOST
 * buffers for tests: K_phys, V_phys [Hkv][rows][d] bf16 with rows =
 * views*frames*tok_per_frame + text_len + tail_tokens (ring rows, text rows,
 * decode-tail rows: the device layout above), pos_phys[rows] = each row's
 * current window position as the attention kernel computes it (from the
 * device-resident ring head), frame_id_phys[rows] = the insertion counter of
 * the frame a ring row belongs to (frames of the prefill are 0..frames-1, the
 * k-th step inserts frame frames-1+k; -1 for text and tail rows). Any pointer
 * may be NULL to skip that output. State: not EXPECT_PREFILL.
 */
int fs_stream_debug_export(fs_stream_t s, void* K_phys, void* V_phys,
                           int32_t* pos_phys, int32_t* frame_id_phys);

/*
 * fs_stream_debug_wait_probe -- launches one kernel that waits on a device
 * barrier nothing will ever complete, with the given limit in microseconds
 * (1..10^6). The wait must give up, record the timeout and return; the call then
 * synchronises and returns FS_ERR_DEVICE_TIMEOUT. Used by tests of the
 * bounded-wait path; it never hangs the GPU.
 */
int fs_stream_debug_wait_probe(fs_stream_t s, int limit_us);

/* Message of the handle's last failure ("" if none). Valid until the next call on s. */
const char* fs_stream_last_error(fs_stream_t s);

/* Message of the calling thread's last failure, including failures without a handle. */
const char* fs_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* FS_STREAM_H */
