// kv_stream_insert -- writes a window's (or a step's) pre-RoPE K/V into the
// per-view ring buffers of the static KV cache.
//
// FlashDrive technical summary (gist.science), Methodology 1, "Token Layout":
// with view-major ordering, a new frame's tokens go at the end of its own
// view's run of tokens, not at the global end. Here each view's run is a ring
// of T frame slots: the step's new frame overwrites the slot of that view's
// oldest frame (evict-oldest); the host then advances the head by one slot, so
// the window order is recovered by positions (key_pos), never by moving data.
//
// Work: a pure copy, bound by HBM bandwidth. Each thread moves 16-byte chunks;
// consecutive threads take consecutive chunks of the token-major source, so
// loads are fully coalesced and stores form 256-byte runs (one d=128 vector).
// All index arithmetic is 32-bit (a step moves < 2^31 chunks).
#include "fs_internal.cuh"

namespace fs {

namespace {

constexpr int kInsertThreads = 256;
constexpr int kTokensPerBlock = 4;

__device__ __forceinline__ int dest_row(const InsertParams& p, int t) {
    if (p.mode == 0) return t;                                   // prefill: window order, head = slot 0
    if (p.mode == 2) return p.ring_rows + p.X + t;               // drafted block after the text
    const int vn = p.V * p.n;
    if (t < vn) {
        const int v = t / p.n;
        const int i = t - v * p.n;
        return (v * p.T + p.head) * p.n + i;                     // slot of view v's oldest frame
    }
    return p.ring_rows + (t - vn);                               // fresh text
}

// One block moves kTokensPerBlock tokens: their Hkv x chunks 16-byte chunks of
// K and of V. Source reads are contiguous; each (token, kv head) vector lands
// as one contiguous run of d*2 bytes in its kv head's ring.
__global__ void __launch_bounds__(kInsertThreads) kv_stream_insert_kernel(const InsertParams p) {
    const int per_tok = p.Hkv * p.chunks;
    const int t0 = blockIdx.x * kTokensPerBlock;
    const int nt = min(kTokensPerBlock, p.N - t0);
    const int total = nt * per_tok;
    const size_t src0 = (size_t)t0 * per_tok;
    for (int i = threadIdx.x; i < total; i += kInsertThreads) {
        const int tl = i / per_tok;
        const int hc = i - tl * per_tok;
        const int h = hc / p.chunks;
        const int c = hc - h * p.chunks;
        const uint4 k = __ldcs(p.K_src + src0 + i);  // streamed once: do not keep in L1
        const uint4 v = __ldcs(p.V_src + src0 + i);
        const size_t dst = ((size_t)h * p.rows_cap + dest_row(p, t0 + tl)) * p.chunks + c;
        p.K_cache[dst] = k;
        p.V_cache[dst] = v;
    }
}

}  // namespace

cudaError_t launch_kv_stream_insert(const InsertParams& p, int num_sms, cudaStream_t stream) {
    (void)num_sms;
    if (p.N <= 0) return cudaSuccess;
    const unsigned blocks = unsigned((p.N + kTokensPerBlock - 1) / kTokensPerBlock);
    kv_stream_insert_kernel<<<blocks, kInsertThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace fs
