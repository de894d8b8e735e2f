// kv_stream_insert -- writes a window's (or a step's) pre-RoPE K/V into the
// per-view ring buffers of the static KV cache and, in the same pass, rotates
// the written keys for the attention kernel's MMA operands.
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
//    shifted positions. Scores depend only on the difference of the query's
//    and the key's rotation angles, so a key is rotated once, when it enters
//    the cache, at the angle index p + k*n (p its window position, k the ring
//    state's step count): while it stays cached its position drops by n per
//    step and k grows by one, so p + k*n is still its index later, and the
//    queries of a step are rotated at their positions + k*n. Every R-th step
//    (k would reach R) the pass re-rotates the whole window at k = 0, which
//    keeps the angle table finite.
//
// A launch covers one or more layers (blockIdx.y = layer); each block strides
// over its layer's rows: the whole window on a prefill or a re-base step, the
// new rows (each view's new frame and the text) on other steps, and rows
// [row0, row0 + N) for a decode-tail or drafted block, and (mode 3) the whole
// window from the cache after the fused projection wrote a re-base step's rows.
// One thread takes one
// pair of 16-byte chunks (c, c + d/16) of one (row, kv head) -- the
// rotate-half partners. A row being written this call takes its K/V from the
// caller's token-major [N][Hkv][d] buffers and stores them into the bf16
// cache; a re-based row reads the cache. Both then write the rotated key as
// fp16 hi + fp16 lo (lo = the rounding residual of hi, ~22 bits together) and
// V as fp16, row-major [Hkv][rows_cap][d] like the cache (the attention
// kernel's tensor maps swizzle on load). The rotation runs in fp32 from the
// bf16 values and the cos/sin table (evaluated in double at create).
//
// Operands are fp16: a rotated key or V element above 65504 in magnitude (or a
// NaN) cannot be represented; the pass flags it in the handle's error word
// (kErrRange), which fs_stream_sync reports.
//
// The pass is bound by HBM bandwidth: per new (row, kv head) read 4d bytes
// (K, V from the caller) and write 4d bytes of bf16 cache plus 6d bytes of
// operands. A warp covers whole rows, so every load and store is contiguous
// and coalesced. The last block of the launch advances the layer's ring state
// (head, k) in device memory.
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

// Window-step source of physical ring/text row `row`: the token of this call's
// K/V that lands there, or -1 if the row keeps its cached content.
__device__ __forceinline__ int step_source_token(const WindowShape& w, int old_head, int row) {
    if (row >= w.ring_rows) return w.V * w.n + (row - w.ring_rows);  // fresh text
    const int s = row / w.n;
    if (s % w.T != old_head) return -1;                               // not the slot being overwritten
    return (s / w.T) * w.n + (row - s * w.n);                         // view's new frame, token i
}

template <int D>
__global__ void __launch_bounds__(kInsertThreads) kv_stream_insert_kernel(const __grid_constant__ InsertParams p) {
    grid_dependency_wait();     // the previous kernel (say, an attention reading these operands) is done
    allow_dependents_launch();  // the next kernel may start its set-up
    constexpr int kPairs = D / 16;  // threads per (row, kv head)
    const InsertLayer& ly = p.layer[blockIdx.y];
    const int2 st = load_ring_state(ly.state);  // (head, k) before this insert
    WindowShape w = p.w;
    const int L = w.ring_rows + w.X;
    int new_k = st.y;
    bool all_rows = false;
    if (p.mode == 0) {
        w.head = 0;
        new_k = 0;
        all_rows = true;
    } else if (p.mode == 1) {
        w.head = st.x + 1 == w.T ? 0 : st.x + 1;
        new_k = st.y + 1 >= p.rebase_every ? 0 : st.y + 1;
        all_rows = new_k == 0;
    } else if (p.mode == 3) {
        w.head = st.x;  // already advanced by the kernel that wrote the step's rows
        all_rows = true;
    } else {
        w.head = st.x;
    }
    const int old_head = st.x;
    const int rows = all_rows ? L : (p.mode == 1 ? w.V * w.n + w.X : p.N);
    const int angle_off = new_k * w.n;
    const unsigned items = unsigned(rows) * unsigned(p.Hkv) * kPairs;

    for (unsigned it = blockIdx.x * kInsertThreads + threadIdx.x; it < items; it += gridDim.x * kInsertThreads) {
        const int c = int(it % kPairs);
        const unsigned rr = it / kPairs;
        const int h = int(rr / unsigned(rows));
        const int ri = int(rr % unsigned(rows));
        int row, t;
        if (p.mode == 0) {
            row = ri;
            t = ri;
        } else if (p.mode == 3) {
            row = ri;
            t = -1;
        } else if (p.mode == 1) {
            if (all_rows) {
                row = ri;
                t = step_source_token(w, old_head, ri);
            } else {
                const int vn = w.V * w.n;
                row = ri < vn ? ((ri / w.n) * w.T + old_head) * w.n + ri % w.n : w.ring_rows + (ri - vn);
                t = ri;
            }
        } else {
            row = p.row0 + ri;
            t = ri;
        }
        const size_t base = ((size_t)h * p.rows_cap + row) * D;
        const size_t oa = base + 8 * c, ob = base + D / 2 + 8 * c;  // element offsets of the two chunks
        uint4 ka, kb, va, vb;
        if (t >= 0) {
            const size_t src = ((size_t)t * p.Hkv + h) * D;
            ka = __ldcs(reinterpret_cast<const uint4*>(ly.K_src + src + 8 * c));  // read once: do not keep in L1
            kb = __ldcs(reinterpret_cast<const uint4*>(ly.K_src + src + D / 2 + 8 * c));
            va = __ldcs(reinterpret_cast<const uint4*>(ly.V_src + src + 8 * c));
            vb = __ldcs(reinterpret_cast<const uint4*>(ly.V_src + src + D / 2 + 8 * c));
            *reinterpret_cast<uint4*>(ly.K + oa) = ka;
            *reinterpret_cast<uint4*>(ly.K + ob) = kb;
            *reinterpret_cast<uint4*>(ly.V + oa) = va;
            *reinterpret_cast<uint4*>(ly.V + ob) = vb;
        } else {
            ka = *reinterpret_cast<const uint4*>(ly.K + oa);
            kb = *reinterpret_cast<const uint4*>(ly.K + ob);
            va = *reinterpret_cast<const uint4*>(ly.V + oa);
            vb = *reinterpret_cast<const uint4*>(ly.V + ob);
        }
        // Rotate-half: element i pairs with i + D/2, angle (pos + k*n) * theta_i.
        const float4* t4 =
            reinterpret_cast<const float4*>(p.rope + (size_t)(key_pos(w, row) + angle_off) * (D / 2) + 8 * c);
        const float4 tb[4] = {__ldg(t4), __ldg(t4 + 1), __ldg(t4 + 2), __ldg(t4 + 3)};
        const uint32_t aw[4] = {ka.x, ka.y, ka.z, ka.w};
        const uint32_t bw[4] = {kb.x, kb.y, kb.z, kb.w};
        uint32_t rah[4], ral[4], rbh[4], rbl[4];
        // Every element converted to fp16 must be finite and at most 65504 in
        // magnitude (a NaN fails the comparison too).
        bool in_range = true;
        const uint32_t vw[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
#pragma unroll
        for (int q = 0; q < 8; ++q)
            in_range = in_range && fabsf(bf16lo(vw[q])) <= kF16Max && fabsf(bf16hi(vw[q])) <= kF16Max;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float x0 = bf16lo(aw[q]), x1 = bf16hi(aw[q]);
            const float y0 = bf16lo(bw[q]), y1 = bf16hi(bw[q]);
            const float4 tq = tb[q];  // (cos, sin) of elements 8c + 2q and 8c + 2q + 1
            const float r0 = x0 * tq.x - y0 * tq.y, r1 = x1 * tq.z - y1 * tq.w;
            const float s0 = y0 * tq.x + x0 * tq.y, s1 = y1 * tq.z + x1 * tq.w;
            in_range = in_range && fabsf(r0) <= kF16Max && fabsf(r1) <= kF16Max && fabsf(s0) <= kF16Max &&
                       fabsf(s1) <= kF16Max;
            split_pair(r0, r1, rah[q], ral[q]);
            split_pair(s0, s1, rbh[q], rbl[q]);
        }
        if (!in_range) atomicOr(ly.err, kErrRange);
        *reinterpret_cast<uint4*>(ly.Kh + oa) = make_uint4(rah[0], rah[1], rah[2], rah[3]);
        *reinterpret_cast<uint4*>(ly.Kh + ob) = make_uint4(rbh[0], rbh[1], rbh[2], rbh[3]);
        *reinterpret_cast<uint4*>(ly.Kl + oa) = make_uint4(ral[0], ral[1], ral[2], ral[3]);
        *reinterpret_cast<uint4*>(ly.Kl + ob) = make_uint4(rbl[0], rbl[1], rbl[2], rbl[3]);
        *reinterpret_cast<uint4*>(ly.V16 + oa) = bf16x8_to_f16x8(va);
        *reinterpret_cast<uint4*>(ly.V16 + ob) = bf16x8_to_f16x8(vb);
    }

    if (p.mode == 0 || p.mode == 1) {
        // Every block read the old state above, before it arrives here; the last
        // block to arrive publishes the new one (the next kernel on the stream
        // starts reading it only after this grid has completed).
        __syncthreads();
        if (threadIdx.x == 0) {
            const unsigned prev = atomicAdd(&ly.state->done, 1u);
            if (prev == gridDim.x - 1) {
                ly.state->head = w.head;
                ly.state->k = new_k;
                ly.state->done = 0u;
            }
        }
    }
}

template <int D>
cudaError_t launch_d(const InsertParams& p, cudaStream_t stream) {
    // Blocks per layer: enough for the rows of an ordinary call (a re-base
    // step loops over the whole window with the same grid).
    const int rows = p.mode == 0 || p.mode == 3 ? p.w.ring_rows + p.w.X : (p.mode == 1 ? p.w.V * p.w.n + p.w.X : p.N);
    const long long threads = (long long)rows * p.Hkv * (D / 16);
    const unsigned blocks = unsigned((threads + kInsertThreads - 1) / kInsertThreads);
    return launch_overlapped(kv_stream_insert_kernel<D>, dim3(blocks, unsigned(p.layers)), dim3(kInsertThreads), 0,
                             stream, p);
}

}  // namespace

cudaError_t launch_kv_stream_insert(const InsertParams& p, cudaStream_t stream) {
    if (p.layers <= 0) return cudaSuccess;
    return p.d == 128 ? launch_d<128>(p, stream) : launch_d<64>(p, stream);
}

}  // namespace fs
