// frame_attn -- the vision encoder's attention over each view's newest frame.
//
// FlashDrive technical summary (gist.science), Methodology 1, "Algorithmic
// Shortcut": instead of re-encoding every frame of the sliding window, a window
// step encodes only the newest frame of each camera and reuses the rest. Inside
// the encoder, the newest frame's tokens attend to each other; this kernel is
// that attention: for view v, query token t of the frame sees every token of
// the same frame (bidirectional, no mask inside the frame, nothing of other
// views), no positional rotation, scores scaled by 1/sqrt(d), query head h
// reading kv head h / (H/Hkv).
//
// CTA (view v, kv head h, query tile q) holds 128 query rows (128/G tokens x
// the G query heads of h) and walks the frame's key tiles of 128 tokens. The
// inputs are bf16 and are not rotated, so S = Q K^T is one bf16 tcgen05 MMA
// chain per tile (products exact in the fp32 accumulator in TMEM). Each thread
// owns one query row (TMEM lane) and runs the online softmax over all keys of
// the tile (exact row max, keys past the frame masked); P goes to TMEM as fp16
// and O += P V with V converted to fp16 in shared memory. Operands are loaded
// with coalesced 16-byte loads into the 128-byte swizzled layouts the MMA
// reads; the output is staged in shared memory and written row by row.
#include <cfloat>

#include "fs_internal.cuh"
#include "sm100.cuh"

namespace fs {
namespace {

constexpr int kFThreads = 128;
constexpr uint32_t kFTmemCols = 256;  // S [0, 128), O [128, 128 + D)
constexpr int kFCtrlBytes = 1024;

enum : int { kFBarS = 0, kFBarO, kFBarDrain, kFNumBars };

struct FCtrl {
    uint64_t bars[kFNumBars];
    uint32_t tmem_base;
};
static_assert(sizeof(FCtrl) <= kFCtrlBytes, "control block too large");

// Q (bf16), K (bf16), V (fp16): each 128 rows x D in 128-byte swizzled
// 64-column regions (chunk c of row r at c ^ (r & 7)); the output staging
// reuses Q and K.
template <int D>
struct FLayout {
    static constexpr int kRegion = 128 * 128;
    static constexpr int kOp = 128 * D * 2;
    static constexpr int kQ = 0, kK = kOp, kV = 2 * kOp;
    static constexpr int kSmemBytes = kFCtrlBytes + 3 * kOp;
    static_assert(128 * D * 4 <= 2 * kOp, "output staging does not fit");
};

// Byte offset of 16-byte chunk c (8 elements) of row r in a 128-row operand.
template <int D>
__device__ __forceinline__ int chunk_off(int r, int c) {
    return (c >> 3) * FLayout<D>::kRegion + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}

__device__ __forceinline__ uint4 bf16x8_to_f16x8f(uint4 v, bool& in_range) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q)
        in_range = in_range && fabsf(bf16lo(w[q])) <= kF16Max && fabsf(bf16hi(w[q])) <= kF16Max;
    return make_uint4(pack_f16x2(bf16lo(v.x), bf16hi(v.x)), pack_f16x2(bf16lo(v.y), bf16hi(v.y)),
                      pack_f16x2(bf16lo(v.z), bf16hi(v.z)), pack_f16x2(bf16lo(v.w), bf16hi(v.w)));
}

template <int D>
__global__ void __launch_bounds__(kFThreads, 1) frame_attn_kernel(const __grid_constant__ FrameParams p) {
    using L = FLayout<D>;
    constexpr int kChunks = D / 8;
    constexpr int kC4 = D / 4;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    FCtrl& ctrl = *reinterpret_cast<FCtrl*>(smem_raw);
    uint8_t* smem = smem_raw + kFCtrlBytes;
    {
        uint32_t dyn;
        asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
        if ((smem_u32(smem) & 1023u) != 0 || dyn < uint32_t(L::kSmemBytes)) {
            if (threadIdx.x == 0) atomicOr(p.err, kErrBadLaunch);
            return;
        }
    }
    grid_dependency_wait();  // the previous kernel (say, the projection writing Q, K, V) is done
    allow_dependents_launch();
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int qt = blockIdx.x % p.q_tiles;
    const int kvh = (blockIdx.x / p.q_tiles) % p.Hkv;
    const int v = blockIdx.x / (p.q_tiles * p.Hkv);
    const int tpt = kTileRows / p.G;     // tokens per query tile
    const int tok0 = qt * tpt;           // first query token of the tile (in the frame)
    const size_t frame0 = (size_t)v * p.n;  // the view's first token row in Q, K, V, out
    const BoundedWait wait{p.err, p.wait_limit_ns, kErrTimeout};
    auto bar = [&](int i) { return smem_u32(&ctrl.bars[i]); };

    if (tid == 0) {
        for (int i = 0; i < kFNumBars; ++i) mbar_init(bar(i), 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&ctrl.tmem_base), kFTmemCols);
        tmem_relinquish();
    }
    // Query tile: row r = (token tok0 + r / G, head kvh * G + r % G); rows past
    // the frame are zero.
    for (int i = tid; i < kTileRows * kChunks; i += kFThreads) {
        const int r = i / kChunks, c = i % kChunks;
        const int t = tok0 + r / p.G;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (t < p.n)
            val = __ldg(reinterpret_cast<const uint4*>(p.Q + ((frame0 + t) * p.H + kvh * p.G + r % p.G) * D + 8 * c));
        *reinterpret_cast<uint4*>(smem + L::kQ + chunk_off<D>(r, c)) = val;
    }
    // Keys and values of frame tokens [128 j, 128 j + 128) of this kv head.
    bool in_range = true;
    auto load_kv = [&](int j) {
        for (int i = tid; i < kTileRows * kChunks; i += kFThreads) {
            const int r = i / kChunks, c = i % kChunks;
            const int t = j * kTileRows + r;
            uint4 kk = make_uint4(0, 0, 0, 0), vv = kk;
            if (t < p.n) {
                const size_t src = ((frame0 + t) * p.Hkv + kvh) * D + 8 * c;
                kk = __ldg(reinterpret_cast<const uint4*>(p.K + src));
                vv = bf16x8_to_f16x8f(__ldg(reinterpret_cast<const uint4*>(p.V + src)), in_range);
            }
            *reinterpret_cast<uint4*>(smem + L::kK + chunk_off<D>(r, c)) = kk;
            *reinterpret_cast<uint4*>(smem + L::kV + chunk_off<D>(r, c)) = vv;
        }
        fence_proxy_async_smem();  // generic stores -> read by the tensor core
    };
    load_kv(0);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctrl.tmem_base;
    const uint32_t lane_off = uint32_t(32 * warp) << 16;
    const uint32_t t_s = tmem, t_o = tmem + 128;
    constexpr uint32_t idesc_qk = idesc_f16(128, 128, true, true, false, false);  // bf16 x bf16
    constexpr uint32_t idesc_pv = idesc_f16(128, D, false, false, false, true);   // fp16 P x fp16 V
    const float c2 = p.q_scale;  // log2(e) / sqrt(d)
    const int n_kt = (p.n + kTileRows - 1) / kTileRows;
    float m_run = -INFINITY, l_run = 0.f;  // running max of the raw scores, sum
    bool ok = true;                         // once a wait gives up, later waits are skipped
    for (int j = 0; j < n_kt; ++j) {
        if (j > 0) {
            load_kv(j);  // after the previous tile's P V (waited below)
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
        }
        if (tid == 0) {
            const uint64_t dq = sw128_desc(smem_u32(smem + L::kQ), 16, 1024);
            const uint64_t dk = sw128_desc(smem_u32(smem + L::kK), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t o = ((kk >> 2) * L::kRegion + (kk & 3) * 32) >> 4;
                mma_ss(t_s, dq + o, dk + o, idesc_qk, kk > 0);
            }
            tc_commit(bar(kFBarS));
        }
        if (ok) ok = wait(bar(kFBarS), j & 1);
        tc_fence_after();
        // Online softmax of this row over the tile's keys (keys past the frame masked).
        uint32_t sr[4][32];
#pragma unroll
        for (int h = 0; h < 4; ++h) tmem_ld32(t_s + lane_off + 32 * h, sr[h]);
        tmem_wait_ld();
        const int klim = p.n - j * kTileRows;  // keys of this tile inside the frame
        if (klim < kTileRows) {
#pragma unroll
            for (int h = 0; h < 4; ++h)
#pragma unroll
                for (int c = 0; c < 32; ++c)
                    if (32 * h + c >= klim) sr[h][c] = __float_as_uint(-INFINITY);
        }
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int h = 0; h < 4; ++h)
#pragma unroll
            for (int c = 0; c < 32; c += 2)
                m4[h] = fmax3(m4[h], __uint_as_float(sr[h][c]), __uint_as_float(sr[h][c + 1]));
        const float m_new = fmaxf(m_run, fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])));
        const float nb = m_new == -INFINITY ? 0.f : -m_new * c2;  // P = 2^(s c2 - m c2) <= 1
        const float alpha = m_run == -INFINITY ? 0.f : ex2_approx((m_run - m_new) * c2);
        float rsum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            uint32_t pk[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const float p0 = ex2_approx(fmaf(__uint_as_float(sr[h][2 * q]), c2, nb));
                const float p1 = ex2_approx(fmaf(__uint_as_float(sr[h][2 * q + 1]), c2, nb));
                rsum[q & 3] += p0 + p1;
                pk[q] = pack_f16x2(p0, p1);
            }
            tmem_st16(t_s + lane_off + 16 * h, pk);
        }
        l_run = l_run * alpha + ((rsum[0] + rsum[1]) + (rsum[2] + rsum[3]));
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
            // O holds the earlier tiles' P V (complete: waited before this tile's loads).
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t o[32];
                tmem_ld32(t_o + lane_off + 32 * cc, o);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                tmem_st32(t_o + lane_off + 32 * cc, o);
            }
        }
        m_run = m_new;
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();  // P of every row is in TMEM
        if (tid == 0) {
            tc_fence_after();
            const uint64_t dv = smem_desc(smem_u32(smem + L::kV), L::kRegion, 1024, 2);
#pragma unroll
            for (int kk = 0; kk < kTileRows / 16; ++kk)
                mma_ts(t_o, t_s + kk * 8, dv + ((kk * 16 * 128) >> 4), idesc_pv, (j > 0 || kk > 0));
            tc_commit(bar(kFBarO));
        }
        // P V done before S is overwritten, K / V reloaded, or O read.
        if (ok) ok = wait(bar(kFBarO), j & 1);
        tc_fence_after();
    }
    if (!in_range) atomicOr(p.err, kErrRange);
    // ---- epilogue: out = O / l, staged over the (free) Q and K tiles, then
    // written as contiguous row segments.
    float4* stg4 = reinterpret_cast<float4*>(smem + L::kQ);
    {
        const int r = tid;
        const float sc = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(t_o + lane_off + 32 * cc, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; e += 4)
                stg4[r * kC4 + (((32 * cc + e) >> 2) ^ (r & 7))] =
                    make_float4(__uint_as_float(o[e]) * sc, __uint_as_float(o[e + 1]) * sc,
                                __uint_as_float(o[e + 2]) * sc, __uint_as_float(o[e + 3]) * sc);
        }
    }
    if (tid == 0) {
        tc_commit(bar(kFBarDrain));  // every MMA complete before TMEM is released
        wait(bar(kFBarDrain), 0);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kFTmemCols);
    }
    const int rows_valid = min(kTileRows, (p.n - tok0) * p.G);
    for (int i = tid; i < rows_valid * kC4; i += kFThreads) {
        const int r = i / kC4, c = i % kC4;
        float* dst = p.out + ((frame0 + tok0 + r / p.G) * p.H + kvh * p.G + r % p.G) * D;
        reinterpret_cast<float4*>(dst)[c] = stg4[r * kC4 + (c ^ (r & 7))];
    }
}

template <int D>
cudaError_t launch_d(const FrameParams& p, cudaStream_t stream) {
    const size_t smem = size_t(FLayout<D>::kSmemBytes);
    cudaError_t e = ensure_smem_attr<frame_attn_kernel<D>>(int(smem));
    if (e != cudaSuccess) return e;
    return launch_overlapped(frame_attn_kernel<D>, dim3(unsigned(p.views * p.Hkv * p.q_tiles)), dim3(kFThreads), smem,
                             stream, p);
}

}  // namespace

cudaError_t launch_frame_attn(const FrameParams& p, cudaStream_t stream) {
    return p.d == 128 ? launch_d<128>(p, stream) : launch_d<64>(p, stream);
}

}  // namespace fs
