// fs_internal.cuh -- parameters shared by the host side of the library and its
// kernels, and the position arithmetic of the view-major window.
#pragma once
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <utility>
#include <cuda.h>
#include <cuda_runtime.h>

namespace fs {

constexpr int kTileRows = 128;          // query rows (token x head) and keys per tile
constexpr int kMaxKeyTiles = 2048;      // key rows per kv head <= 2048 * 128
constexpr int kMaxVerify = 256;         // scratch rows for a drafted block (FS_MAX_VERIFY_TOKENS)
constexpr int kMaxTail = 1024;          // persisted decode-tail rows (FS_MAX_TAIL_TOKENS)
constexpr int kMaxInsertBatch = 40;     // layers one kv_stream_insert launch covers
constexpr int kMaxVerifySplits = 16;    // key splits per kv head of a verify_attn launch (its cluster size)
constexpr unsigned kErrTimeout = 1u;    // device error word bits
constexpr unsigned kErrBadLaunch = 2u;
constexpr unsigned kErrRange = 4u;      // an fp16 operand would overflow (|x| > 65504) or is NaN
constexpr float kF16Max = 65504.f;

enum QueryMode : int { kQueryPrefill = 0, kQueryStep = 1, kQueryVerify = 2 };

// Shape of the view-major window and the ring head, as the kernels need them.
struct WindowShape {
    int V, T, n, X;     // views, frames per view, tokens per frame, text tokens
    int ring_rows;      // V * T * n
    int head;           // ring slot holding every view's oldest frame
    int tail;           // persisted decode-tail tokens after the text
};

// Ring state kept in device memory, one per handle. kv_stream_insert advances
// it (the last block of the launch writes the new values); every kernel reads
// it after its grid-dependency wait, so no launch parameter changes from one
// window step to the next.
//   head: ring slot holding each view's oldest frame;
//   k:    window steps since the cached keys were last rotated at their plain
//         window positions. A key enters the cache at window position p during
//         step k and is rotated once, at angle index p + k*n; every later step
//         moves it one frame (n positions) towards the start of its view while
//         k grows by one, so p + k*n stays its angle index for as long as it
//         is cached. Queries are rotated at their position + k*n. Scores only
//         depend on angle differences, which equal position differences.
//   done: blocks of the running insert launch that have finished (reset by the
//         last one).
struct RingState {
    int head;
    int k;
    unsigned done;
    int pad;
};

__device__ __forceinline__ int2 load_ring_state(const RingState* st) {
    // L2 (coherence point), never a stale L1 line of an earlier kernel.
    return __ldcg(reinterpret_cast<const int2*>(st));
}

// Window position of physical cache row `row` (per kv head).
// Ring rows: view v, slot s, token i sit at row (v*T + s)*n + i; the slot's
// age in the window is (s - head) mod T (0 = oldest), so the token's position
// in the current view-major window is v*T*n + age*n + i. Text rows (and the
// drafted block after them) keep their row index as position: they follow all
// views. "Keys are stored pre-RoPE and rotated at shifted positions"
// (FlashDrive technical summary, Methodology 1, "Positional Encoding").
__host__ __device__ __forceinline__ int key_pos(const WindowShape& w, int head, int row) {
    if (row >= w.ring_rows) return row;
    const int tn = w.T * w.n;
    const int v = row / tn;
    const int rem = row - v * tn;
    const int s = rem / w.n;
    const int i = rem - s * w.n;
    int age = s - head;
    if (age < 0) age += w.T;
    return v * tn + age * w.n + i;
}
__host__ __device__ __forceinline__ int key_pos(const WindowShape& w, int row) { return key_pos(w, w.head, row); }

// Window position of query token t.
//   prefill: the whole window in order, position t;
//   step: view v's newest frame (the last of its T frames) then the text,
//         "inserted at the end of each view's sequence" (FlashDrive technical
//         summary, Methodology 1, "Token Layout");
//   verify: a drafted block right after the text and the persisted decode tail.
__host__ __device__ __forceinline__ int query_pos(const WindowShape& w, int mode, int t) {
    if (mode == kQueryPrefill) return t;
    if (mode == kQueryVerify) return w.ring_rows + w.X + w.tail + t;
    const int vn = w.V * w.n;
    if (t < vn) {
        const int v = t / w.n;
        const int i = t - v * w.n;
        return v * w.T * w.n + (w.T - 1) * w.n + i;
    }
    return w.ring_rows + (t - vn);
}

struct AttnParams {
    WindowShape w;
    int key_rows;         // valid key rows per kv head for this launch
    int Hkv, G, H, d;     // kv heads, query heads per kv head, query heads, head dim
    int nq;               // query tokens
    int q_mode;           // QueryMode
    int q_tiles;          // ceil(nq * G / 128)
    int splits;           // key splits per (kv head, query tile)
    float q_scale;        // log2(e) / sqrt(d), folded into the rotated queries
    const float2* rope;   // [rope_rows][d/2] (cos, sin) of angle index * theta_i
    int rope_rows;
    const RingState* state;  // head and angle offset k (written by kv_stream_insert)
    float* out;           // [nq][H][d] fp32
    float* part_o;        // [items][splits][128][d] fp32 (splits > 1)
    float2* part_ml;      // [items][splits][128] (running max in log2 units, sum)
    unsigned* err;        // device error word
    unsigned long long wait_limit_ns;
};

// One layer's buffers for kv_stream_insert.
struct InsertLayer {
    const uint16_t* K_src;  // [N][Hkv][d] bf16, pre-RoPE
    const uint16_t* V_src;
    uint16_t* K;            // bf16 cache [Hkv][rows_cap][d]: new rows written, others read on a re-base
    uint16_t* V;
    uint16_t* Kh;           // fp16 rotated key, hi part, same layout as the cache
    uint16_t* Kl;           // fp16 rotated key, lo part
    uint16_t* V16;          // fp16 V
    RingState* state;
    unsigned* err;          // device error word (kErrRange)
};

struct InsertParams {
    WindowShape w;          // window shape (head comes from each layer's state)
    int mode;               // 0: prefill (row = t), 1: window step, 2: rows [row0, row0 + N) after the text,
                            // 3: re-rotate the window from the cache (state already advanced)
    int N;                  // tokens per layer in K_src / V_src
    int row0;               // mode 2: first physical row written
    int Hkv, d, rows_cap;
    int rebase_every;       // R: a window step whose k would reach R re-rotates the whole window (k = 0)
    const float2* rope;     // [rope_rows][d/2] (cos, sin)
    int layers;             // entries of `layer` in use (gridDim.y)
    InsertLayer layer[kMaxInsertBatch];
};

// A drafted block's attention in one launch (kernel verify_attn).
struct VerifyParams {
    WindowShape w;
    int key_rows;           // L + tail + n_x: cached rows, then the block's rows
    int row_block;          // L + tail: physical row (= position) of the block's first token
    int n_x;                // block tokens (n_x * G <= 128)
    int Hkv, G, H, d, rows_cap;
    int splits;             // key splits per kv head = cluster size (grid = Hkv * splits)
    float q_scale;          // log2(e) / sqrt(d)
    const float2* rope;     // [rope_rows][d/2] (cos, sin)
    const RingState* state; // angle offset k * n
    const uint16_t* Q_x;    // [n_x][H][d] bf16
    const uint16_t* K_x;    // [n_x][Hkv][d] bf16
    const uint16_t* V_x;
    float* out;             // [n_x][H][d] fp32
    unsigned* err;
    unsigned long long wait_limit_ns;
};

// Launches `kernel` with programmatic stream serialisation: its launch and set-up
// may overlap the end of the previous kernel on the stream; the kernel itself
// calls grid_dependency_wait() before touching memory that kernel may use.
// FS_PDL=0 in the environment turns the overlap off (ordinary stream order).
inline bool overlapped_launch_enabled() {
    static const bool on = [] {
        const char* e = std::getenv("FS_PDL");
        return !(e && e[0] == '0');
    }();
    return on;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_overlapped(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = overlapped_launch_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// The K/V projection of a step's hidden states fused with the ring insert (kernel kv_proj).
struct ProjParams {
    WindowShape w;          // window shape (head from the ring state)
    int mode;               // 0: prefill (token t -> row t), 1: window step
    int N;                  // tokens (rows of X)
    int d_model;
    int Hkv, d, rows_cap;
    int rebase_every;
    const float2* rope;
    uint16_t* K;            // bf16 cache [Hkv][rows_cap][d]
    uint16_t* V;
    uint16_t* Kh;           // operands, same layout
    uint16_t* Kl;
    uint16_t* V16;
    RingState* state;
    unsigned* err;
    unsigned long long wait_limit_ns;
};

// The vision encoder's attention over each view's newest frame (kernel frame_attn).
struct FrameParams {
    int views, n;           // views, tokens per frame; token t of view v is row v * n + t
    int H, Hkv, G, d;
    int q_tiles;            // ceil(n * G / 128) query tiles per (view, kv head)
    float q_scale;          // log2(e) / sqrt(d)
    const uint16_t* Q;      // [views * n][H][d] bf16
    const uint16_t* K;      // [views * n][Hkv][d] bf16
    const uint16_t* V;
    float* out;             // [views * n][H][d] fp32
    unsigned* err;
    unsigned long long wait_limit_ns;
};

// Raises `Kernel`'s dynamic shared-memory limit to `bytes` once per device (the
// attribute is per device and per function; the first launch on each device
// sets it, later launches skip the call).
template <auto Kernel>
cudaError_t ensure_smem_attr(int bytes) {
    constexpr int kMaxDevices = 64;
    static std::atomic<int> done[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices && done[dev].load(std::memory_order_acquire) >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && dev >= 0 && dev < kMaxDevices) done[dev].store(bytes, std::memory_order_release);
    return e;
}

// Launchers (defined in the .cu files); all enqueue on `stream` and return the
// launch's cudaError_t.
// kv_stream_insert: new K/V into the bf16 cache, and every processed row's rotated
// fp16 K hi / lo and fp16 V.
// One launch covers p.layers layers (blockIdx.y); each block strides over its
// layer's rows.
cudaError_t launch_kv_stream_insert(const InsertParams& p, cudaStream_t stream);
// stream_attn over the rotated operand cache (tkh, tkl, tv16); tq maps the
// call's bf16 queries [nq][H][d] with box {64, G, 128/G} (128-byte swizzle).
cudaError_t launch_stream_attn(const AttnParams& p, const CUtensorMap& tq, const CUtensorMap& tkh,
                               const CUtensorMap& tkl, const CUtensorMap& tv16, cudaStream_t stream);
cudaError_t launch_attn_combine(const AttnParams& p, cudaStream_t stream);
// verify_attn over the operand cache; tkh / tkl: K hi / lo maps with 64-row
// boxes, tv: V map with {64 columns, 128 rows} boxes (128-byte swizzle).
cudaError_t launch_verify_attn(const VerifyParams& p, const CUtensorMap& tkh, const CUtensorMap& tkl,
                               const CUtensorMap& tv, cudaStream_t stream);
cudaError_t launch_frame_attn(const FrameParams& p, cudaStream_t stream);
// kv_proj over X (tensor map tx: [N][d_model] bf16, box {64, 128}) and W (tw:
// [2 Hkv d][d_model], box {64, 128}), both 128-byte swizzled.
cudaError_t launch_kv_proj(const ProjParams& p, const CUtensorMap& tx, const CUtensorMap& tw, cudaStream_t stream);
cudaError_t launch_positions(const WindowShape& w, const RingState* state, int rows, int* pos_out,
                             cudaStream_t stream);
cudaError_t launch_wait_probe(unsigned* err, unsigned long long limit_ns, cudaStream_t stream);
size_t stream_attn_smem_bytes(int d);
// Fixed split-KV scratch in device memory (no allocation): its capacity in
// partial 128-row tiles, and its address on the current device (looked up on
// the first call per device).
int static_split_scratch_tiles();
cudaError_t static_split_scratch(float** part_o, float2** part_ml);

}  // namespace fs
