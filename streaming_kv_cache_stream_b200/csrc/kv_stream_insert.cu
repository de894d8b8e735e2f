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
#include "fs_internal.cuh"

namespace fs {

namespace {

constexpr int kInsertThreads = 256;
constexpr int kInsertUnroll = 4;

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

__global__ void __launch_bounds__(kInsertThreads) kv_stream_insert_kernel(const InsertParams p) {
    const long long total = (long long)p.N * p.Hkv * p.chunks;
    const long long stride = (long long)gridDim.x * kInsertThreads * kInsertUnroll;
    for (long long base = (long long)blockIdx.x * kInsertThreads * kInsertUnroll + threadIdx.x; base < total;
         base += stride) {
        uint4 k[kInsertUnroll], v[kInsertUnroll];
#pragma unroll
        for (int u = 0; u < kInsertUnroll; ++u) {
            const long long idx = base + (long long)u * kInsertThreads;
            if (idx < total) {
                k[u] = __ldcs(p.K_src + idx);   // streamed once: do not keep in L1/L2
                v[u] = __ldcs(p.V_src + idx);
            }
        }
#pragma unroll
        for (int u = 0; u < kInsertUnroll; ++u) {
            const long long idx = base + (long long)u * kInsertThreads;
            if (idx < total) {
                const int c = int(idx % p.chunks);
                const long long th = idx / p.chunks;
                const int h = int(th % p.Hkv);
                const int t = int(th / p.Hkv);
                const long long dst = ((long long)h * p.rows_cap + dest_row(p, t)) * p.chunks + c;
                p.K_cache[dst] = k[u];
                p.V_cache[dst] = v[u];
            }
        }
    }
}

}  // namespace

cudaError_t launch_kv_stream_insert(const InsertParams& p, int num_sms, cudaStream_t stream) {
    const long long total = (long long)p.N * p.Hkv * p.chunks;
    if (total <= 0) return cudaSuccess;
    long long blocks = (total + kInsertThreads * kInsertUnroll - 1) / (kInsertThreads * kInsertUnroll);
    const long long cap = (long long)num_sms * 8;  // 8 resident 256-thread blocks per SM
    if (blocks > cap) blocks = cap;
    kv_stream_insert_kernel<<<(unsigned)blocks, kInsertThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace fs
