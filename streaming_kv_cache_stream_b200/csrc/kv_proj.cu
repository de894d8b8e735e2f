// kv_proj_insert -- the K/V projection of a window step's hidden states, fused
// with the ring insert.
//
// FlashDrive README (z-lab/flashdrive), "System optimizations", and technical
// summary, System Optimizations, "Kernel Fusion": the projections are merged
// into single kernels. Here the step's hidden states X [N][d_model] (each
// view's new-frame tokens, then the text; the whole window on a prefill) are
// multiplied by the stacked K/V weight W [2*Hkv*d][d_model] (K rows first), and
// the epilogue writes the results straight where fs_stream_insert would: each
// output element rounded once to bf16 into the token's ring slot (the view's
// oldest frame is overwritten, "inserted at the end of each view's sequence",
// technical summary, Methodology 1, "Token Layout"), plus the attention
// operands (key rotated once at angle index position + k*n, as fp16 hi + lo;
// V as fp16). There is no separate insert pass over K and V.
//
// Work split: a cluster of two CTAs owns a 128 x 256 tile of X W^T (128
// tokens, 256 output columns) and splits d_model between them (split-K): each
// CTA streams its half of the 64-column blocks of X and W through a 3-stage
// TMA ring (128-byte swizzle) and one thread issues bf16 tcgen05 MMAs of
// M = 128, N = 256 (the shape that keeps the tensor pipe busiest on one SM)
// into an fp32 accumulator in TMEM. Then each CTA stores the partial sums of
// the peer's 128 columns into a receive buffer in the peer's shared memory
// (distributed shared memory, signalled through the peer's mbarrier), adds the
// peer's partial to its own 128 columns, and finishes them. Thread (g, r) of
// the two warpgroups holds token m0 + r and 64 of the columns, chosen so that
// the rotate-half partners (i, i + d/2) of a key are in the same thread.
// Results are staged in shared memory and written out as whole contiguous
// cache rows. The last CTA to finish advances the ring state (head, k) as
// kv_stream_insert does.
#include "fs_internal.cuh"
#include "sm100.cuh"

namespace fs {
namespace {

constexpr int kPThreads = 256;
constexpr int kPStages = 3;
constexpr int kPBK = 64;                      // d_model columns per stage
constexpr int kPXTile = 128 * kPBK * 2;       // 128 tokens x 64 columns, bf16: 16 KB
constexpr int kPWTile = 256 * kPBK * 2;       // 256 weight rows x 64 columns: 32 KB
constexpr int kPStage = kPXTile + kPWTile;
constexpr int kPCtrlBytes = 1024;
constexpr uint32_t kPTmemCols = 256;
// The receive buffer for the peer's partial sums (128 rows x 128 fp32) lies
// past the stage buffers, so the peer may fill it while this CTA's main loop
// still runs; after the main loop the stage buffers hold the finished rows.
constexpr int kPPartBytes = 128 * 128 * 4;
constexpr int kPRecv = kPStages * kPStage;
constexpr int kPOut = 0;                       // up to 3 arrays x 128 rows x 128 bf16/fp16
constexpr int kPOutBytes = 3 * 128 * 128 * 2;
static_assert(kPOut + kPOutBytes <= kPRecv, "staged rows exceed the stage buffers");
constexpr int kPBuf = kPRecv + kPPartBytes;

enum : int { kPFull0 = 0, kPEmpty0 = kPFull0 + kPStages, kPDone = kPEmpty0 + kPStages, kPRecvBar, kPNumBars };

struct PCtrl {
    uint64_t bars[kPNumBars];
    uint32_t tmem_base;
    int prow[128];  // cache row of each token of the tile
};
static_assert(sizeof(PCtrl) <= kPCtrlBytes, "control block too large");
constexpr int kPSmemBytes = kPCtrlBytes + kPBuf;
static_assert(kPSmemBytes <= 227 * 1024, "shared memory over the per-CTA limit");

__device__ __forceinline__ void split_pair_p(float a, float b, uint32_t& hi, uint32_t& lo) {
    hi = pack_f16x2(a, b);
    const float2 hf = __half22float2(*reinterpret_cast<const __half2*>(&hi));
    lo = pack_f16x2(a - hf.x, b - hf.y);
}

// Staged output row layout: row r of one head in one array is D*2 bytes, 16-byte
// chunk c stored at position c ^ (r mod chunks) so that a warp's row-per-thread
// stores and its row-contiguous reads both spread over the banks.
template <int D>
__device__ __forceinline__ uint32_t stage_off(int r, int c) {
    constexpr int kChunks = D / 8;
    return uint32_t(r * (D * 2) + ((c ^ (r & (kChunks - 1))) << 4));
}

// Columns a0 + j and a0 + D/2 + j (j < 32) of one head of token r's projection
// (fp32 ya[j], yb[j]): rounded to bf16 (the cache row, array 0); for a key
// also rotated with cs[i] = (cos, sin) of elements a0 + 2i, a0 + 2i + 1
// (element i pairs with i + D/2)
// into fp16 hi (array 1) and lo (array 2); for a value converted to fp16
// (array 1). Arrays are `array_bytes` apart from `out`. Returns false if an
// operand element would not fit fp16.
template <int D>
__device__ __forceinline__ bool stage_pairs(const float (&ya)[32], const float (&yb)[32], int a0, bool is_key,
                                            const float4 (&cs)[16], uint8_t* out, int array_bytes, int r,
                                            bool operands) {
    uint32_t ba[16], bb[16];  // bf16 pairs
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        ba[i] = pack_bf16x2(ya[2 * i], ya[2 * i + 1]);
        bb[i] = pack_bf16x2(yb[2 * i], yb[2 * i + 1]);
    }
    const int ca = a0 / 8, cb = (a0 + D / 2) / 8;  // first 16-byte chunk of each part
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        *reinterpret_cast<uint4*>(out + stage_off<D>(r, ca + c)) =
            make_uint4(ba[4 * c], ba[4 * c + 1], ba[4 * c + 2], ba[4 * c + 3]);
        *reinterpret_cast<uint4*>(out + stage_off<D>(r, cb + c)) =
            make_uint4(bb[4 * c], bb[4 * c + 1], bb[4 * c + 2], bb[4 * c + 3]);
    }
    if (!operands) return true;
    bool in_range = true;
    uint8_t* o1 = out + array_bytes;
    if (is_key) {
        uint8_t* o2 = out + 2 * array_bytes;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint32_t ah[4], al[4], bh[4], bl[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 tq = cs[4 * c + q];
                const uint32_t wa = ba[4 * c + q], wb = bb[4 * c + q];
                const float x0 = bf16lo(wa), x1 = bf16hi(wa);
                const float y0 = bf16lo(wb), y1 = bf16hi(wb);
                const float r0 = x0 * tq.x - y0 * tq.y, r1 = x1 * tq.z - y1 * tq.w;
                const float s0 = y0 * tq.x + x0 * tq.y, s1 = y1 * tq.z + x1 * tq.w;
                in_range = in_range && fabsf(r0) <= kF16Max && fabsf(r1) <= kF16Max && fabsf(s0) <= kF16Max &&
                           fabsf(s1) <= kF16Max;
                split_pair_p(r0, r1, ah[q], al[q]);
                split_pair_p(s0, s1, bh[q], bl[q]);
            }
            *reinterpret_cast<uint4*>(o1 + stage_off<D>(r, ca + c)) = make_uint4(ah[0], ah[1], ah[2], ah[3]);
            *reinterpret_cast<uint4*>(o1 + stage_off<D>(r, cb + c)) = make_uint4(bh[0], bh[1], bh[2], bh[3]);
            *reinterpret_cast<uint4*>(o2 + stage_off<D>(r, ca + c)) = make_uint4(al[0], al[1], al[2], al[3]);
            *reinterpret_cast<uint4*>(o2 + stage_off<D>(r, cb + c)) = make_uint4(bl[0], bl[1], bl[2], bl[3]);
        }
    } else {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint32_t fa[4], fb[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float x0 = bf16lo(ba[4 * c + q]), x1 = bf16hi(ba[4 * c + q]);
                const float y0 = bf16lo(bb[4 * c + q]), y1 = bf16hi(bb[4 * c + q]);
                in_range = in_range && fabsf(x0) <= kF16Max && fabsf(x1) <= kF16Max && fabsf(y0) <= kF16Max &&
                           fabsf(y1) <= kF16Max;
                fa[q] = pack_f16x2(x0, x1);
                fb[q] = pack_f16x2(y0, y1);
            }
            *reinterpret_cast<uint4*>(o1 + stage_off<D>(r, ca + c)) = make_uint4(fa[0], fa[1], fa[2], fa[3]);
            *reinterpret_cast<uint4*>(o1 + stage_off<D>(r, cb + c)) = make_uint4(fb[0], fb[1], fb[2], fb[3]);
        }
    }
    return in_range;
}

// Receive-buffer position of 16-byte chunk q (fp32 columns 4q .. 4q+3) of row
// r: chunk-major, so the 32 rows of a warp are 512 contiguous bytes, for the
// sender's remote stores and the receiver's reads alike.
__device__ __forceinline__ uint32_t recv_off(int r, int q) { return uint32_t((q * 128 + r) << 4); }

template <int D>
__global__ void __launch_bounds__(kPThreads, 1)
    kv_proj_kernel(const __grid_constant__ ProjParams p, const __grid_constant__ CUtensorMap tx,
                   const __grid_constant__ CUtensorMap tw) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    PCtrl& ctrl = *reinterpret_cast<PCtrl*>(smem_raw);
    uint8_t* smem = smem_raw + kPCtrlBytes;
    {
        // The same for both CTAs of a cluster, so both leave before any cluster barrier.
        uint32_t dyn;
        asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
        if ((smem_u32(smem) & 1023u) != 0 || dyn < uint32_t(kPSmemBytes)) {
            if (threadIdx.x == 0) atomicOr(p.err, kErrBadLaunch);
            return;
        }
    }
    grid_dependency_wait();  // the previous kernel (reading these cache rows, or writing X) is done
    allow_dependents_launch();
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const uint32_t crank = cluster_rank();  // = blockIdx.x & 1
    const int m0 = int(blockIdx.x >> 1) * 128;
    const int n0 = int(blockIdx.y) * 256;
    const int nkb = (p.d_model + kPBK - 1) / kPBK;
    const int kb_half = (nkb + 1) / 2;
    const int kb0 = crank ? kb_half : 0;
    const int kb1 = crank ? nkb : kb_half;
    const bool has_acc = kb1 > kb0;  // a CTA with no column blocks contributes zeros
    const BoundedWait wait{p.err, p.wait_limit_ns, kErrTimeout};
    auto bar = [&](int i) { return smem_u32(&ctrl.bars[i]); };

    if (tid == 0) {
        for (int s = 0; s < kPStages; ++s) {
            mbar_init(bar(kPFull0 + s), 1);
            mbar_init(bar(kPEmpty0 + s), 1);
        }
        mbar_init(bar(kPDone), 1);
        mbar_init(bar(kPRecvBar), kPThreads);  // every thread of the peer arrives once
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&ctrl.tmem_base), kPTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctrl.tmem_base;
    // Both CTAs of the cluster have started and initialised their mbarriers once
    // this barrier completes; its wait comes just before the first access to
    // the peer's shared memory, after the main loop.
    cluster_arrive();

    // Lane 0 of warp 0 produces and lane 0 of warp 1 issues the MMAs; the other
    // lanes of those warps wait for them at __syncwarp (not spinning on an
    // mbarrier, which would take issue slots from the working lane).
    if (warp == 0) {
        if ((tid & 31) == 0) {
            // ---- TMA producer: X rows [m0, m0 + 128) and W rows [n0, n0 + 256)
            // of column block kb (rows past the end read as zero).
            tma_prefetch_desc(&tx);
            tma_prefetch_desc(&tw);
            for (int kb = kb0; kb < kb1; ++kb) {
                const int i = kb - kb0, s = i % kPStages;
                if (!wait(bar(kPEmpty0 + s), ((i / kPStages) & 1) ^ 1)) break;
                mbar_arrive_expect_tx(bar(kPFull0 + s), kPStage);
                uint8_t* st_x = smem + s * kPStage;
                tma_load_3d(smem_u32(st_x), &tx, kb * kPBK, m0, 0, bar(kPFull0 + s));
                tma_load_3d(smem_u32(st_x + kPXTile), &tw, kb * kPBK, n0, 0, bar(kPFull0 + s));
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if ((tid & 31) == 0) {
            // ---- MMA issuer: D[128 x 256] (+)= X_tile W_tile^T, bf16 in, fp32 in TMEM.
            constexpr uint32_t idesc = idesc_f16(128, 256, true, true, false, false);
            bool ok = true;
            for (int kb = kb0; kb < kb1 && ok; ++kb) {
                const int i = kb - kb0, s = i % kPStages;
                if (!(ok = wait(bar(kPFull0 + s), (i / kPStages) & 1))) break;
                tc_fence_after();
                const uint64_t da = sw128_desc(smem_u32(smem + s * kPStage), 16, 1024);
                const uint64_t db = sw128_desc(smem_u32(smem + s * kPStage + kPXTile), 16, 1024);
#pragma unroll
                for (int kk = 0; kk < kPBK / 16; ++kk)
                    mma_ss(tmem, da + uint32_t(kk * 2), db + uint32_t(kk * 2), idesc, (i > 0 || kk > 0));
                tc_commit(bar(kPEmpty0 + s));  // the stage is free once these MMAs have read it
            }
            tc_commit(bar(kPDone));  // every MMA above (issued or not) complete
        }
        __syncwarp();
    }

    // Ring state before this insert and after it (as kv_stream_insert), read
    // while the main loop runs.
    const int2 st = load_ring_state(p.state);
    WindowShape w = p.w;
    int new_k;
    if (p.mode == 0) {
        w.head = 0;
        new_k = 0;
    } else {
        w.head = st.x + 1 == w.T ? 0 : st.x + 1;
        new_k = st.y + 1 >= p.rebase_every ? 0 : st.y + 1;
    }
    const int old_head = st.x;
    // On a re-base step a full pass over the window follows and writes every
    // operand; this kernel then only writes the bf16 cache rows.
    const bool operands = !(p.mode == 1 && new_k == 0);

    // Token rows of the tile and their cache rows.
    const int g = warp >> 2;                // warpgroup: which 64 of the CTA's 128 columns
    const int r = 32 * (warp & 3) + (tid & 31);  // TMEM lane = tile row = token m0 + r
    const uint32_t lane_off = uint32_t(32 * (warp & 3)) << 16;
    const int t = m0 + r;
    const bool valid = t < p.N;
    const int vn = w.V * w.n;
    int row = 0;
    if (valid) {
        if (p.mode == 0) {
            row = t;
        } else {
            row = t < vn ? ((t / w.n) * w.T + old_head) * w.n + t % w.n : w.ring_rows + (t - vn);
        }
    }
    if (g == 0) ctrl.prow[r] = row;
    constexpr int kArrayBytes = 128 * 128 * 2;  // one staged output array of the tile: 32 KB
    const int hh = D == 128 ? 0 : g;             // head within the CTA's 128 columns
    const int a0 = D == 128 ? 32 * g : 0;        // this thread's first head-local column
    const int col0 = n0 + 128 * int(crank);      // first weight row of the CTA's columns
    const int head = (col0 + hh * D) / D;        // in [0, 2 Hkv): K heads, then V heads
    const bool rotate = valid && operands && head < p.Hkv;
    // (cos, sin) of elements a0 .. a0 + 31 at the key's angle index, fetched
    // while the main loop runs.
    float4 tq[16];
    {
        const float4* cs4 =
            reinterpret_cast<const float4*>(p.rope + (size_t)(key_pos(w, row) + new_k * w.n) * (D / 2) + a0);
#pragma unroll
        for (int i = 0; i < 16; ++i) tq[i] = rotate ? __ldg(cs4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    }

    const bool done = __all_sync(0xffffffffu, wait(bar(kPDone), 0));
    tc_fence_after();

    // ---- split-K exchange: the partial sums of the peer's 128 columns go
    // into the peer's receive buffer; warpgroup g sends columns
    // [64 g, 64 g + 64) of them for row r, then arrives on the peer's mbarrier.
    cluster_wait();
    {
        const uint32_t peer = crank ^ 1u;
        const uint32_t peer_cols = 128u * peer + 64u * uint32_t(g);
        const uint32_t remote = map_to_rank(smem_u32(smem + kPRecv), peer);
#pragma unroll 1
        for (int cc = 0; cc < 2; ++cc) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_off + peer_cols + uint32_t(32 * cc), o);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint4 v = has_acc && done ? make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3])
                                                : make_uint4(0u, 0u, 0u, 0u);
                st_dsmem_u4(remote + recv_off(r, 16 * g + 8 * cc + j), v);
            }
        }
        mbar_arrive_remote(map_to_rank(bar(kPRecvBar), peer));
    }
    // The peer's partial has arrived once all its threads have arrived here
    // (so nothing writes into this CTA's shared memory after this wait).
    const bool recvd = __all_sync(0xffffffffu, wait.wait<true>(bar(kPRecvBar), 0));

    // ---- epilogue: this CTA's 128 columns [n0 + 128 crank, + 128), own partial
    // + the peer's. Thread (g, r) takes head-local columns a0 + j and
    // a0 + D/2 + j (j < 32) of head hh.
    const uint8_t* recv = smem + kPRecv;
    uint8_t* out = smem + kPOut;
    {
        float ya[32], yb[32];
        const uint32_t ca = uint32_t(128 * crank + hh * D + a0), cb = ca + D / 2;  // accumulator columns
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + ca, o);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 q = *reinterpret_cast<const float4*>(recv + recv_off(r, (hh * D + a0) / 4 + j));
            ya[4 * j + 0] = (has_acc ? __uint_as_float(o[4 * j + 0]) : 0.f) + q.x;
            ya[4 * j + 1] = (has_acc ? __uint_as_float(o[4 * j + 1]) : 0.f) + q.y;
            ya[4 * j + 2] = (has_acc ? __uint_as_float(o[4 * j + 2]) : 0.f) + q.z;
            ya[4 * j + 3] = (has_acc ? __uint_as_float(o[4 * j + 3]) : 0.f) + q.w;
        }
        tmem_ld32(tmem + lane_off + cb, o);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 q = *reinterpret_cast<const float4*>(recv + recv_off(r, (hh * D + a0 + D / 2) / 4 + j));
            yb[4 * j + 0] = (has_acc ? __uint_as_float(o[4 * j + 0]) : 0.f) + q.x;
            yb[4 * j + 1] = (has_acc ? __uint_as_float(o[4 * j + 1]) : 0.f) + q.y;
            yb[4 * j + 2] = (has_acc ? __uint_as_float(o[4 * j + 2]) : 0.f) + q.z;
            yb[4 * j + 3] = (has_acc ? __uint_as_float(o[4 * j + 3]) : 0.f) + q.w;
        }
        if (valid && done && recvd && head < 2 * p.Hkv &&
            !stage_pairs<D>(ya, yb, a0, head < p.Hkv, tq, out + hh * 128 * D * 2, kArrayBytes, r, operands))
            atomicOr(p.err, kErrRange);
    }
    __syncthreads();  // the staged rows are complete

    // ---- copy-out: whole cache rows, 16 bytes per thread, consecutive threads
    // on consecutive chunks of a row.
    if (done && recvd) {
        constexpr int kChunks = D / 8;
        const int rows = p.N - m0 < 128 ? p.N - m0 : 128;
#pragma unroll 1
        for (int h2 = 0; h2 < 128 / D; ++h2) {
            const int hd = (col0 + h2 * D) / D;
            if (hd >= 2 * p.Hkv) break;
            const bool is_key = hd < p.Hkv;
            const int kvh = is_key ? hd : hd - p.Hkv;
            const int arrays = operands ? (is_key ? 3 : 2) : 1;
#pragma unroll 1
            for (int a = 0; a < arrays; ++a) {
                uint16_t* dst = (a == 0 ? (is_key ? p.K : p.V) : (a == 1 ? (is_key ? p.Kh : p.V16) : p.Kl)) +
                                (size_t)kvh * p.rows_cap * D;
                const uint8_t* src = out + a * kArrayBytes + h2 * 128 * D * 2;
#pragma unroll 4
                for (int it = tid; it < rows * kChunks; it += kPThreads) {
                    const int rr = it / kChunks, c = it % kChunks;
                    const uint4 v = *reinterpret_cast<const uint4*>(src + stage_off<D>(rr, c));
                    *reinterpret_cast<uint4*>(dst + (size_t)ctrl.prow[rr] * D + 8 * c) = v;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kPTmemCols);
    }
    // The last CTA to finish publishes the new ring state.
    if (tid == 0) {
        const unsigned prev = atomicAdd(&p.state->done, 1u);
        if (prev == gridDim.x * gridDim.y - 1) {
            p.state->head = w.head;
            p.state->k = new_k;
            p.state->done = 0u;
        }
    }
}

template <int D>
cudaError_t launch_d(const ProjParams& p, const CUtensorMap& tx, const CUtensorMap& tw, cudaStream_t stream) {
    cudaError_t e = ensure_smem_attr<kv_proj_kernel<D>>(kPSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(2 * ((p.N + 127) / 128)), unsigned((2 * p.Hkv * D + 255) / 256));
    cfg.blockDim = dim3(kPThreads);
    cfg.dynamicSmemBytes = size_t(kPSmemBytes);
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = overlapped_launch_enabled() ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, kv_proj_kernel<D>, p, tx, tw);
}

}  // namespace

cudaError_t launch_kv_proj(const ProjParams& p, const CUtensorMap& tx, const CUtensorMap& tw, cudaStream_t stream) {
    return p.d == 128 ? launch_d<128>(p, tx, tw, stream) : launch_d<64>(p, tx, tw, stream);
}

}  // namespace fs
