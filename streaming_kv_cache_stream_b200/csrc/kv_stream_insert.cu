// kv_stream_insert -- writes a window's (or a step's) pre-RoPE K/V into the
// per-view ring buffers of the static KV cache and, in the same pass, rotates
// every cached key at the position it now holds, producing the attention
// kernel's MMA operands.
//
// FlashDrive technical summary (gist.science), Methodology 1:
//  * "Token Layout": with view-major ordering, a new frame's tokens go at the
//    end of its own view's run of tokens, not at the global end. Here each
//    view's run is a ring of T frame slots: the step's new frame overwrites the
//    slot of that view's oldest frame (evict-oldest); the head then advances by
//    one slot, so the window order is recovered by positions (key_pos), never
//    by moving data.
//  * "Positional Encoding": keys are stored pre-RoPE because absolute positions
//    go stale as the window shifts; rotary embeddings are applied at the
//    shifted positions. After an insert every cached key's position is final
//    until the next one, so the rotation happens here, once per key and step,
//    instead of once per query tile that reads the key inside stream_attn.
//
// One thread takes one pair of 16-byte chunks (c, c + d/16) of one (row, kv
// head) -- the rotate-half partners. A row being written this call takes its
// K/V from the caller's token-major [N][Hkv][d] buffers and stores them into
// the bf16 cache; every other row reads the cache. Both then write the rotated
// key as fp16 hi + fp16 lo (lo = the rounding residual of hi, ~22 bits
// together) and V as fp16, row-major [Hkv][rows_cap][d] like the cache (the
// attention kernel's tensor maps swizzle on load). Rows from the last key to
// the end of its 128-row tile get zeros (the attention kernel masks them by
// position). The rotation runs in fp32 from the bf16 values and the cos/sin
// table (evaluated in double at create).
//
// Work is a streaming pass bound by HBM bandwidth: per (row, kv head) read 4d
// bytes (K, V; from the caller for new rows), write 6d bytes of operands, and
// for new rows 4d bytes of bf16 cache. A warp covers whole rows, so every load
// and store is contiguous and coalesced. Index arithmetic is 32-bit except for
// the final offsets.
#include "fs_internal.cuh"
#include "sm100.cuh"

namespace fs {
namespace {

constexpr int kInsertThreads = 256;

// fp32 pair -> fp16 hi pair + fp16 lo pair.
__device__ __forceinline__ void split_pair(float a, float b, uint32_t& hi, uint32_t& lo) {
    hi = pack_f16x2(a, b);
    const float2 hf = __half22float2(*reinterpret_cast<const __half2*>(&hi));
    lo = pack_f16x2(a - hf.x, b - hf.y);
}

__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 v) {
    return make_uint4(pack_f16x2(bf16lo(v.x), bf16hi(v.x)), pack_f16x2(bf16lo(v.y), bf16hi(v.y)),
                      pack_f16x2(bf16lo(v.z), bf16hi(v.z)), pack_f16x2(bf16lo(v.w), bf16hi(v.w)));
}

// Token of this call's K/V that lands in physical row `row`, or -1 if the row
// keeps its cached content.
__device__ __forceinline__ int source_token(const InsertParams& p, int row) {
    if (p.mode == 0) return row;                                 // prefill: window order, head = slot 0
    if (p.mode == 2) return row - (p.w.ring_rows + p.w.X);       // drafted block after the text
    if (row >= p.w.ring_rows) return p.w.V * p.w.n + (row - p.w.ring_rows);  // fresh text
    const int s = row / p.w.n;
    if (s % p.w.T != p.old_head) return -1;                      // not the slot being overwritten
    return (s / p.w.T) * p.w.n + (row - s * p.w.n);             // view's new frame, token i
}

template <int D>
__global__ void __launch_bounds__(kInsertThreads) kv_stream_insert_kernel(const InsertParams p) {
    grid_dependency_wait();     // the previous kernel (say, an attention reading these operands) is done
    allow_dependents_launch();  // the next kernel may start its set-up
    constexpr int kPairs = D / 16;  // threads per (row, kv head)
    const unsigned gid = blockIdx.x * kInsertThreads + threadIdx.x;
    const unsigned nrows = unsigned(p.row_end - p.row_begin);
    const unsigned rr = gid / kPairs;
    if (rr >= nrows * unsigned(p.Hkv)) return;
    const int c = int(gid % kPairs);
    const int h = int(rr / nrows);
    const int row = p.row_begin + int(rr % nrows);
    const size_t base = ((size_t)h * p.rows_cap + row) * D;
    const size_t oa = base + 8 * c, ob = base + D / 2 + 8 * c;  // element offsets of the two chunks

    uint4 ah = make_uint4(0, 0, 0, 0), al = ah, bh = ah, bl = ah, va16 = ah, vb16 = ah;
    if (row < p.key_rows) {
        uint4 ka, kb, va, vb;
        const int t = source_token(p, row);
        if (t >= 0) {
            const size_t src = ((size_t)t * p.Hkv + h) * D;
            ka = __ldcs(reinterpret_cast<const uint4*>(p.K_src + src + 8 * c));  // read once: do not keep in L1
            kb = __ldcs(reinterpret_cast<const uint4*>(p.K_src + src + D / 2 + 8 * c));
            va = __ldcs(reinterpret_cast<const uint4*>(p.V_src + src + 8 * c));
            vb = __ldcs(reinterpret_cast<const uint4*>(p.V_src + src + D / 2 + 8 * c));
            *reinterpret_cast<uint4*>(p.K + oa) = ka;
            *reinterpret_cast<uint4*>(p.K + ob) = kb;
            *reinterpret_cast<uint4*>(p.V + oa) = va;
            *reinterpret_cast<uint4*>(p.V + ob) = vb;
        } else {
            ka = *reinterpret_cast<const uint4*>(p.K + oa);
            kb = *reinterpret_cast<const uint4*>(p.K + ob);
            va = *reinterpret_cast<const uint4*>(p.V + oa);
            vb = *reinterpret_cast<const uint4*>(p.V + ob);
        }
        // Rotate-half: element i pairs with i + D/2, angle pos * theta_i.
        const float4* t4 = reinterpret_cast<const float4*>(p.rope + (size_t)key_pos(p.w, row) * (D / 2) + 8 * c);
        const float4 tb[4] = {__ldg(t4), __ldg(t4 + 1), __ldg(t4 + 2), __ldg(t4 + 3)};
        const uint32_t aw[4] = {ka.x, ka.y, ka.z, ka.w};
        const uint32_t bw[4] = {kb.x, kb.y, kb.z, kb.w};
        uint32_t rah[4], ral[4], rbh[4], rbl[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float x0 = bf16lo(aw[q]), x1 = bf16hi(aw[q]);
            const float y0 = bf16lo(bw[q]), y1 = bf16hi(bw[q]);
            const float4 tq = tb[q];  // (cos, sin) of elements 8c + 2q and 8c + 2q + 1
            split_pair(x0 * tq.x - y0 * tq.y, x1 * tq.z - y1 * tq.w, rah[q], ral[q]);
            split_pair(y0 * tq.x + x0 * tq.y, y1 * tq.z + x1 * tq.w, rbh[q], rbl[q]);
        }
        ah = make_uint4(rah[0], rah[1], rah[2], rah[3]);
        al = make_uint4(ral[0], ral[1], ral[2], ral[3]);
        bh = make_uint4(rbh[0], rbh[1], rbh[2], rbh[3]);
        bl = make_uint4(rbl[0], rbl[1], rbl[2], rbl[3]);
        va16 = bf16x8_to_f16x8(va);
        vb16 = bf16x8_to_f16x8(vb);
    }
    *reinterpret_cast<uint4*>(p.Kh + oa) = ah;
    *reinterpret_cast<uint4*>(p.Kh + ob) = bh;
    *reinterpret_cast<uint4*>(p.Kl + oa) = al;
    *reinterpret_cast<uint4*>(p.Kl + ob) = bl;
    *reinterpret_cast<uint4*>(p.V16 + oa) = va16;
    *reinterpret_cast<uint4*>(p.V16 + ob) = vb16;
}

template <int D>
cudaError_t launch_d(const InsertParams& p, cudaStream_t stream) {
    const long long threads = (long long)(p.row_end - p.row_begin) * p.Hkv * (D / 16);
    const unsigned blocks = unsigned((threads + kInsertThreads - 1) / kInsertThreads);
    return launch_overlapped(kv_stream_insert_kernel<D>, dim3(blocks), dim3(kInsertThreads), 0, stream, p);
}

}  // namespace

cudaError_t launch_kv_stream_insert(const InsertParams& p, cudaStream_t stream) {
    if (p.row_end <= p.row_begin) return cudaSuccess;
    return p.d == 128 ? launch_d<128>(p, stream) : launch_d<64>(p, stream);
}

}  // namespace fs
