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

/* Stream states. */
#define FS_STATE_EXPECT_PREFILL 0 /* after create/reset: insert takes the whole window     */
#define FS_STATE_PREFILLED      1 /* window inserted, attend takes all L queries (causal)  */
#define FS_STATE_STREAMING      2 /* insert takes one new frame per view plus the text     */

/* Largest drafted block fs_stream_attend_ext accepts. */
#define FS_MAX_VERIFY_TOKENS 256

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
    long long cache_bytes; /* device bytes owned by the handle                           */
    long long launches;  /* kernels this handle has launched since create                 */
} fs_stream_info_t;

/*
 * fs_stream_create -- allocate one layer's static KV cache (FlashDrive README,
 * "System optimizations": static KV cache) and its RoPE table on the current
 * CUDA device.
 *   views, frames, tok_per_frame >= 1; text_len >= 0; H, Hkv >= 1 with H % Hkv == 0
 *   and 128 % (H/Hkv) == 0; d in {64, 128}; rope_base > 0 (10000 in the
 *   synthetic workloads). L + FS_MAX_VERIFY_TOKENS must be <= 262144 (2048 key tiles
 *   of 128 rows per kv head).
 * Device layout of the cache (owned by the handle, zero-initialised):
 *   K_cache, V_cache [Hkv][R][d] bf16 with R = L + FS_MAX_VERIFY_TOKENS rows per
 *   kv head: rows [0, views*frames*tok_per_frame) are the per-view rings
 *   (view v, slot s, token i at row (v*frames + s)*tok_per_frame + i), then
 *   text_len text rows, then scratch rows for a drafted block.
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
 * fs_stream_attend_ext -- verify a drafted block of n_x tokens in one forward
 * (FlashDrive README, "Speculative reasoning (DFlash)"; technical summary,
 * Methodology 2). The block's tokens sit at positions L .. L+n_x-1, after the
 * text; each sees the whole cached window plus, causally, the block.
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
 * fs_stream_step_host -- one insert + attend with HOST buffers: copies K_new,
 * V_new and Q (bf16) to the device (staging buffers owned by the handle), runs
 * fs_stream_insert and fs_stream_attend, and copies out back, all enqueued on
 * the handle's stream. Sizes follow the current state exactly as for
 * fs_stream_insert / fs_stream_attend; out_h receives fp32. The staging
 * buffers are allocated on the first call (and grown if a later call needs
 * more), so make the first call outside any stream capture. With pinned host
 * memory the call is
 * asynchronous; the caller synchronises (fs_stream_sync) before reading out_h.
 * Errors: as fs_stream_insert and fs_stream_attend.
 */
int fs_stream_step_host(fs_stream_t s, const void* K_new_h, const void* V_new_h,
                        const void* Q_h, void* out_h);

/* Block until the handle's enqueued work is done. Returns FS_ERR_DEVICE_TIMEOUT if a
 * kernel of this handle gave up on a bounded wait since the last check (the flag is
 * cleared), FS_ERR_CUDA on an asynchronous CUDA error. */
int fs_stream_sync(fs_stream_t s);

/* Sizes and state. */
int fs_stream_info(fs_stream_t s, fs_stream_info_t* info);

/*
 * fs_stream_debug_export -- synchronous copy of the physical cache to HOST
 * buffers for tests: K_phys, V_phys [Hkv][rows][d] bf16 with rows =
 * views*frames*tok_per_frame + text_len (ring rows then text rows, the device
 * layout above), pos_phys[rows] = each row's current window position as the
 * attention kernel computes it, frame_id_phys[rows] = the insertion counter of
 * the frame a ring row belongs to (frames of the prefill are 0..frames-1, the
 * k-th step inserts frame frames-1+k; -1 for text rows). Any pointer may be
 * NULL to skip that output. State: not EXPECT_PREFILL.
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
