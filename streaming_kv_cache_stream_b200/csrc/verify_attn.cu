// verify_attn -- attention of a short drafted block (speculative reasoning)
// against the streaming KV cache, in one launch.
//
// FlashDrive README (z-lab/flashdrive), "Speculative reasoning (DFlash)", and
// technical summary (gist.science), Methodology 2: the drafter proposes a
// block of 8 tokens that the target verifies in one forward. The block's n_x
// tokens sit after the text and the persisted decode tail, at window positions
// L + tail + t; each sees every cached key (window and tail) and, causally, the
// block itself. Cached keys were rotated once, at angle index position + k*n
// (k: the ring state's step count), so the block's queries and keys are
// rotated here at (L + tail + t) + k*n.
//
// A block is small (8 tokens x G heads = 32 query rows per kv head), so the
// work is split over the keys. The C CTAs of one kv head form a thread-block
// cluster; CTA s (cluster rank) takes one 128-row query tile (the block's rows
// of the kv head; rows past the block are zero) and key tiles
// [s * nkt / C, (s + 1) * nkt / C). Per key tile: TMA loads the rotated K
// (fp16 hi and lo) and V (fp16) from the handle's operand cache, one thread
// issues S = Q_hi K_hi + Q_hi K_lo + Q_lo K_hi (tcgen05, M = 128, N = 128,
// fp32 in TMEM), the 128 threads each own one query row (TMEM lane) and run the
// online softmax over all 128 keys (exact row max, no exchange), P goes to TMEM
// as fp16 and O += P V (tcgen05, P from TMEM). The tile holding the block's
// own key rows is loaded like the others and the block's rows, rotated, are
// written over its stale rows in shared memory. At the end every CTA
// stages its unnormalised O and (m, l) in shared memory and the cluster merges
// them through distributed shared memory: each CTA combines a share of the
// output rows' columns from all C partials and writes them. No global scratch,
// no second launch.
//
// Every mbarrier wait is bounded (BoundedWait): a CTA that gives up sets the
// error word and carries on to the exit path; nothing spins forever.
#include <cfloat>
#include <climits>

#include "fs_internal.cuh"
#include "sm100.cuh"

namespace fs {
namespace {

constexpr int kVThreads = 128;
constexpr uint32_t kVTmemCols = 256;  // S [0, 128), O [128, 128 + D)
constexpr int kVCtrlBytes = 1024;

enum : int { kVBarK = 0, kVBarV, kVBarS, kVBarO, kVBarDrain, kVNumBars };

struct VCtrl {
    uint64_t bars[kVNumBars];
    uint32_t tmem_base;
};
static_assert(sizeof(VCtrl) <= kVCtrlBytes, "control block too large");

// Shared memory after the control block (1024-byte aligned): Q hi, Q lo, K hi,
// K lo, V; each 128 rows x D fp16 in 128-byte swizzled 64-column regions
// (16 KB each) -- K-major for Q and K, MN-major (keys x columns) for V; then
// the block's pre-RoPE bf16 query rows as loaded. The epilogue reuses the Q
// tiles for the partial O (fp32) and the K hi tile for (m, l).
template <int D>
struct VLayout {
    static constexpr int kRegion = 128 * 128;
    static constexpr int kOp = 128 * D * 2;
    static constexpr int kQh = 0, kQl = kOp, kKh = 2 * kOp, kKl = 3 * kOp, kV = 4 * kOp;
    static constexpr int kQs = 5 * kOp;
    static constexpr int kSmemBytes = kVCtrlBytes + 6 * kOp;
    static_assert(128 * D * 4 <= 2 * kOp, "partial O staging does not fit the Q tiles");
};

__device__ __forceinline__ void split2v(float a, float b, uint32_t& hi, uint32_t& lo) {
    hi = pack_f16x2(a, b);
    const float2 hf = __half22float2(*reinterpret_cast<const __half2*>(&hi));
    lo = pack_f16x2(a - hf.x, b - hf.y);
}

// Rotate-half RoPE of one 16-byte chunk pair (a: elements 8c .. 8c+7, b: the
// partners D/2 + 8c ..) by the angles in tab (cos, sin per element pair), times
// `scale`, as fp16 hi / lo. Returns false if an element is above 65504 in
// magnitude or not finite.
__device__ __forceinline__ bool rotate_chunk(uint4 a, uint4 b, const float4 (&tab)[4], float scale, uint4& ha,
                                             uint4& la, uint4& hb, uint4& lb) {
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
    const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
    uint32_t ah[4], al[4], bh[4], bl[4];
    bool in_range = true;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 tq = tab[q];  // (cos, sin) of elements 2q and 2q + 1 of the chunk
        const float x0 = bf16lo(aw[q]), x1 = bf16hi(aw[q]);
        const float y0 = bf16lo(bw[q]), y1 = bf16hi(bw[q]);
        const float r0 = (x0 * tq.x - y0 * tq.y) * scale, r1 = (x1 * tq.z - y1 * tq.w) * scale;
        const float s0 = (y0 * tq.x + x0 * tq.y) * scale, s1 = (y1 * tq.z + x1 * tq.w) * scale;
        in_range = in_range && fabsf(r0) <= kF16Max && fabsf(r1) <= kF16Max && fabsf(s0) <= kF16Max &&
                   fabsf(s1) <= kF16Max;
        split2v(r0, r1, ah[q], al[q]);
        split2v(s0, s1, bh[q], bl[q]);
    }
    ha = make_uint4(ah[0], ah[1], ah[2], ah[3]);
    la = make_uint4(al[0], al[1], al[2], al[3]);
    hb = make_uint4(bh[0], bh[1], bh[2], bh[3]);
    lb = make_uint4(bl[0], bl[1], bl[2], bl[3]);
    return in_range;
}

__device__ __forceinline__ uint4 bf16x8_to_f16x8v(uint4 v) {
    return make_uint4(pack_f16x2(bf16lo(v.x), bf16hi(v.x)), pack_f16x2(bf16lo(v.y), bf16hi(v.y)),
                      pack_f16x2(bf16lo(v.z), bf16hi(v.z)), pack_f16x2(bf16lo(v.w), bf16hi(v.w)));
}

__device__ __forceinline__ bool bf16x8_in_range(uint4 v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    bool ok = true;
#pragma unroll
    for (int q = 0; q < 4; ++q) ok = ok && fabsf(bf16lo(w[q])) <= kF16Max && fabsf(bf16hi(w[q])) <= kF16Max;
    return ok;
}

template <int D>
__global__ void __launch_bounds__(kVThreads, 1)
    verify_attn_kernel(const __grid_constant__ VerifyParams p, const __grid_constant__ CUtensorMap tkh,
                       const __grid_constant__ CUtensorMap tkl, const __grid_constant__ CUtensorMap tv) {
    using L = VLayout<D>;
    constexpr int kPairs = D / 16;  // rotate-half chunk pairs per row
    constexpr int kChunks = D / 8;  // 16-byte bf16 chunks per row
    constexpr int kC4 = D / 4;      // 16-byte fp32 chunks per output row
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    VCtrl& ctrl = *reinterpret_cast<VCtrl*>(smem_raw);
    uint8_t* smem = smem_raw + kVCtrlBytes;
    {
        // Every CTA of a cluster sees the same layout, so all leave here together.
        uint32_t dyn;
        asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
        if ((smem_u32(smem) & 1023u) != 0 || dyn < uint32_t(L::kSmemBytes)) {
            if (threadIdx.x == 0) atomicOr(p.err, kErrBadLaunch);
            return;
        }
    }
    grid_dependency_wait();  // the previous kernel (an insert or attention on these operands) is done
    allow_dependents_launch();
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int C = p.splits;  // CTAs per kv head = cluster size
    const int kvh = blockIdx.x / C;
    const int split = int(cluster_rank());
    const int n_ktiles = (p.key_rows + kTileRows - 1) / kTileRows;
    const int kt0 = split * n_ktiles / C;
    const int kt1 = (split + 1) * n_ktiles / C;
    const int rows = min(p.n_x * p.G, kTileRows);  // valid query rows of this kv head
    const int angle_off = load_ring_state(p.state).y * p.w.n;
    const BoundedWait wait{p.err, p.wait_limit_ns, kErrTimeout};
    auto bar = [&](int i) { return smem_u32(&ctrl.bars[i]); };

    if (tid == 0) {
        for (int i = 0; i < kVNumBars; ++i) mbar_init(bar(i), 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&ctrl.tmem_base), kVTmemCols);
        tmem_relinquish();
    }

    constexpr uint32_t idesc_qk = idesc_f16(128, 128, false, false, false, false);
    constexpr uint32_t idesc_pv = idesc_f16(128, D, false, false, false, true);
    auto load_k = [&](int j) {
        mbar_arrive_expect_tx(bar(kVBarK), 2 * L::kOp);
#pragma unroll
        for (int g = 0; g < D / 64; ++g)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                tma_load_3d(smem_u32(smem + L::kKh + g * L::kRegion + h * (L::kRegion / 2)), &tkh, 64 * g,
                            j * kTileRows + 64 * h, kvh, bar(kVBarK));
                tma_load_3d(smem_u32(smem + L::kKl + g * L::kRegion + h * (L::kRegion / 2)), &tkl, 64 * g,
                            j * kTileRows + 64 * h, kvh, bar(kVBarK));
            }
    };
    auto load_v = [&](int j) {
        mbar_arrive_expect_tx(bar(kVBarV), L::kOp);
#pragma unroll
        for (int g = 0; g < D / 64; ++g)
            tma_load_3d(smem_u32(smem + L::kV + g * L::kRegion), &tv, 64 * g, j * kTileRows, kvh, bar(kVBarV));
    };
    // The first tile's loads start right away (a tile holding block rows gets
    // them written over its stale rows once it has landed, below).
    if (tid == 0 && kt0 < kt1) {
        tma_prefetch_desc(&tkh);
        tma_prefetch_desc(&tkl);
        tma_prefetch_desc(&tv);
        load_k(kt0);
        load_v(kt0);
    }

    // The block's key rows that fall in this CTA's key tiles, rotated now (one
    // (row, chunk pair) item per thread when they fit) so that only the stores
    // into the landed tiles remain for later.
    const int b0 = max(p.row_block, kt0 * kTileRows), b1 = min(p.key_rows, kt1 * kTileRows);
    const int b_items = b1 > b0 ? (b1 - b0) * kPairs : 0;
    const bool b_pre = b_items <= kVThreads;
    uint4 bha = make_uint4(0, 0, 0, 0), bla = bha, bhb = bha, blb = bha, bva = bha, bvb = bha;
    auto block_item = [&](int i, uint4& ha, uint4& la, uint4& hb, uint4& lb, uint4& va16, uint4& vb16) {
        const int row = b0 + i / kPairs, c = i % kPairs;
        const size_t src = ((size_t)(row - p.row_block) * p.Hkv + kvh) * D;
        float4 tab[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            tab[q] = __ldg(reinterpret_cast<const float4*>(p.rope + (size_t)(row + angle_off) * (D / 2) + 8 * c) + q);
        const uint4 ka = __ldg(reinterpret_cast<const uint4*>(p.K_x + src + 8 * c));
        const uint4 kb = __ldg(reinterpret_cast<const uint4*>(p.K_x + src + D / 2 + 8 * c));
        const uint4 va = __ldg(reinterpret_cast<const uint4*>(p.V_x + src + 8 * c));
        const uint4 vb = __ldg(reinterpret_cast<const uint4*>(p.V_x + src + D / 2 + 8 * c));
        bool in_range = rotate_chunk(ka, kb, tab, 1.f, ha, la, hb, lb);
        in_range = in_range && bf16x8_in_range(va) && bf16x8_in_range(vb);
        if (!in_range) atomicOr(p.err, kErrRange);
        va16 = bf16x8_to_f16x8v(va);
        vb16 = bf16x8_to_f16x8v(vb);
    };
    // Stores one item into the K hi, K lo and V tiles of key tile j (the same
    // 128-byte swizzled key-row layout for all three).
    auto put_block_item = [&](int i, int j, uint4 ha, uint4 la, uint4 hb, uint4 lb, uint4 va16, uint4 vb16) {
        const int row = b0 + i / kPairs, c = i % kPairs;
        const int kr = row - j * kTileRows, sw = kr & 7;
        const int oa = kr * 128 + ((c ^ sw) << 4);
        const int ob = D == 128 ? oa + L::kRegion : kr * 128 + (((c + 4) ^ sw) << 4);
        *reinterpret_cast<uint4*>(smem + L::kKh + oa) = ha;
        *reinterpret_cast<uint4*>(smem + L::kKh + ob) = hb;
        *reinterpret_cast<uint4*>(smem + L::kKl + oa) = la;
        *reinterpret_cast<uint4*>(smem + L::kKl + ob) = lb;
        *reinterpret_cast<uint4*>(smem + L::kV + oa) = va16;
        *reinterpret_cast<uint4*>(smem + L::kV + ob) = vb16;
    };
    if (b_pre && tid < b_items) block_item(tid, bha, bla, bhb, blb, bva, bvb);

    // Query tile: row r = (block token r / G, head kvh * G + r % G). The rows of
    // one token are contiguous in Q_x: the kv head's rows are loaded with
    // coalesced 16-byte loads into shared memory (chunks swizzled by row), then
    // all threads rotate (row, chunk pair) items into the fp16 hi / lo tiles.
    uint8_t* qs = smem + L::kQs;
    for (int i = tid; i < rows * kChunks; i += kVThreads) {
        const int row = i / kChunks, c = i % kChunks;
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(
            p.Q_x + ((size_t)(row / p.G) * p.H + kvh * p.G + row % p.G) * D + 8 * c));
        *reinterpret_cast<uint4*>(qs + row * (D * 2) + ((c ^ (row & 7)) << 4)) = v;
    }
    __syncthreads();
    {
        uint8_t* qh = smem + L::kQh;
        uint8_t* ql = smem + L::kQl;
        auto put = [&](int row, int c, uint4 ha, uint4 la, uint4 hb, uint4 lb) {
            const int sw = row & 7;
            const int oa = row * 128 + ((c ^ sw) << 4);
            const int ob = D == 128 ? oa + L::kRegion : row * 128 + (((c + 4) ^ sw) << 4);
            *reinterpret_cast<uint4*>(qh + oa) = ha;
            *reinterpret_cast<uint4*>(qh + ob) = hb;
            *reinterpret_cast<uint4*>(ql + oa) = la;
            *reinterpret_cast<uint4*>(ql + ob) = lb;
        };
        // Rows past the block: zeros.
        const uint4 z = make_uint4(0, 0, 0, 0);
        for (int it = rows * kPairs + tid; it < kTileRows * kPairs; it += kVThreads) put(it / kPairs, it % kPairs, z, z, z, z);
        // The block's rows: two (row, chunk pair) items per thread per round, all
        // of a round's loads issued before its arithmetic.
        const int items = rows * kPairs;
        for (int i0 = tid; i0 < items; i0 += 2 * kVThreads) {
            float4 tab[2][4];
            uint4 a[2], b[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int it = min(i0 + u * kVThreads, items - 1);
                const int row = it / kPairs, c = it % kPairs, sw = row & 7;
                const float4* t4 = reinterpret_cast<const float4*>(
                    p.rope + (size_t)(p.row_block + row / p.G + angle_off) * (D / 2) + 8 * c);
#pragma unroll
                for (int q = 0; q < 4; ++q) tab[u][q] = __ldg(t4 + q);
                a[u] = *reinterpret_cast<const uint4*>(qs + row * (D * 2) + ((c ^ sw) << 4));
                b[u] = *reinterpret_cast<const uint4*>(qs + row * (D * 2) + (((c + kPairs) ^ sw) << 4));
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int it = i0 + u * kVThreads;
                if (it >= items) break;
                uint4 ha, la, hb, lb;
                if (!rotate_chunk(a[u], b[u], tab[u], p.q_scale, ha, la, hb, lb)) atomicOr(p.err, kErrRange);
                put(it / kPairs, it % kPairs, ha, la, hb, lb);
            }
        }
        fence_proxy_async_smem();  // generic stores -> read by the tensor core
    }
    tc_fence_before();
    __syncthreads();  // query tiles rotated
    tc_fence_after();
    const uint32_t tmem = ctrl.tmem_base;
    const uint32_t lane_off = uint32_t(32 * warp) << 16;
    const uint32_t t_s = tmem, t_o = tmem + 128;
    const int r = tid;       // query row = TMEM lane
    const int tq = r / p.G;  // its block token
    // Rows past the block are zero queries: their scores stay 0 and their P and
    // O are never read, so warps holding only such rows skip the softmax.
    const bool warp_rows = warp * 32 < rows;

    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;  // once a wait gives up, later waits are skipped
    for (int j = kt0; j < kt1; ++j) {
        const int it = j - kt0;
        const int kr0 = j * kTileRows;
        const int t0 = max(b0, kr0), t1 = min(b1, kr0 + kTileRows);  // block rows in this tile
        if (t1 > t0) {
            // Once K and V have landed, the block's rows go over the tile's stale rows.
            if (ok) ok = wait(bar(kVBarK), it & 1);
            if (ok) ok = wait(bar(kVBarV), it & 1);
            const int i0 = (t0 - b0) * kPairs, i1 = (t1 - b0) * kPairs;
            if (b_pre) {
                if (tid >= i0 && tid < i1) put_block_item(tid, j, bha, bla, bhb, blb, bva, bvb);
            } else {
                for (int i = i0 + tid; i < i1; i += kVThreads) {
                    uint4 ha, la, hb, lb, va16, vb16;
                    block_item(i, ha, la, hb, lb, va16, vb16);
                    put_block_item(i, j, ha, la, hb, lb, va16, vb16);
                }
            }
            fence_proxy_async_smem();  // generic stores -> read by the tensor core
            __syncthreads();
        }
        if (tid == 0) {
            // S = Q K^T over the three hi/lo products; K tile j landed.
            if (ok) ok = wait(bar(kVBarK), it & 1);
            tc_fence_after();
            const uint64_t dqh = sw128_desc(smem_u32(smem + L::kQh), 16, 1024);
            const uint64_t dql = sw128_desc(smem_u32(smem + L::kQl), 16, 1024);
            const uint64_t dkh = sw128_desc(smem_u32(smem + L::kKh), 16, 1024);
            const uint64_t dkl = sw128_desc(smem_u32(smem + L::kKl), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t o = ((kk >> 2) * L::kRegion + (kk & 3) * 32) >> 4;
                mma_ss(t_s, dqh + o, dkh + o, idesc_qk, kk > 0);
                mma_ss(t_s, dqh + o, dkl + o, idesc_qk, 1);
                mma_ss(t_s, dql + o, dkh + o, idesc_qk, 1);
            }
            tc_commit(bar(kVBarS));
        }
        if (ok) ok = wait(bar(kVBarS), it & 1);
        tc_fence_after();
        if (tid == 0 && j + 1 < kt1) load_k(j + 1);  // the QK has read this K tile
        if (warp_rows) {
        // Online softmax of row r over the tile's 128 keys. Key row c of the
        // tile is visible iff it is cached (before the block) or a block token
        // at or before this row's token.
        const int qlim = p.row_block + tq;  // last visible key row
        uint32_t sr[4][32];
#pragma unroll
        for (int h = 0; h < 4; ++h) tmem_ld32(t_s + lane_off + 32 * h, sr[h]);
        tmem_wait_ld();
        if (kr0 + kTileRows > p.row_block) {  // only tiles reaching the block need the mask
#pragma unroll
            for (int h = 0; h < 4; ++h)
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const int kr = kr0 + 32 * h + c;
                    if (kr >= p.key_rows || kr > qlim) sr[h][c] = __float_as_uint(-INFINITY);
                }
        }
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int h = 0; h < 4; ++h)
#pragma unroll
            for (int c = 0; c < 32; c += 2)
                m4[h] = fmax3(m4[h], __uint_as_float(sr[h][c]), __uint_as_float(sr[h][c + 1]));
        const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        const float m_new = fmaxf(m_run, mx);
        const float base = m_new == -INFINITY ? 0.f : m_new;
        const float alpha = m_run == -INFINITY ? 0.f : ex2_approx(m_run - base);
        float rsum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            uint32_t pk[16];
#pragma unroll
            for (int c2 = 0; c2 < 16; ++c2) {
                const float p0 = ex2_approx(__uint_as_float(sr[h][2 * c2]) - base);
                const float p1 = ex2_approx(__uint_as_float(sr[h][2 * c2 + 1]) - base);
                rsum[c2 & 3] += p0 + p1;
                pk[c2] = pack_f16x2(p0, p1);
            }
            tmem_st16(t_s + lane_off + 16 * h, pk);
        }
        l_run = l_run * alpha + ((rsum[0] + rsum[1]) + (rsum[2] + rsum[3]));
        if (it > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
            // O holds the earlier tiles' P V (complete: this tile's QK was issued after it).
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
        }  // warps without block rows leave their (zero-query) rows of P as the zero scores
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();  // P of every row is in TMEM
        if (tid == 0) {
            tc_fence_after();
            if (ok) ok = wait(bar(kVBarV), it & 1);
            tc_fence_after();
            const uint64_t dv = smem_desc(smem_u32(smem + L::kV), L::kRegion, 1024, 2);
#pragma unroll
            for (int kk = 0; kk < kTileRows / 16; ++kk)
                mma_ts(t_o, t_s + kk * 8, dv + ((kk * 16 * 128) >> 4), idesc_pv, (it > 0 || kk > 0));
            tc_commit(bar(kVBarO));
        }
        // P V done before S is overwritten by the next QK, before O is read, and
        // before V is reloaded.
        if (ok) ok = wait(bar(kVBarO), it & 1);
        tc_fence_after();
        if (tid == 0 && j + 1 < kt1) load_v(j + 1);
    }

    // ---- epilogue. Each CTA stages its unnormalised O (fp32, chunk c of row r
    // at c ^ (r & 7): conflict-free) over its free Q tiles and (m, l) over its
    // free K hi tile; after a cluster barrier, CTA s combines the s-th of C
    // contiguous slices of the (row, column chunk) list from all C partials
    // through distributed shared memory:
    //   out = sum_q 2^(m_q - M) O_q / sum_q 2^(m_q - M) l_q,  M = max_q m_q.
    float4* stg4 = reinterpret_cast<float4*>(smem + L::kQh);
    float2* sml = reinterpret_cast<float2*>(smem + L::kKh);
    if (kt0 < kt1 && warp_rows) {
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(t_o + lane_off + 32 * cc, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; e += 4)
                stg4[r * kC4 + (((32 * cc + e) >> 2) ^ (r & 7))] =
                    make_float4(__uint_as_float(o[e]), __uint_as_float(o[e + 1]), __uint_as_float(o[e + 2]),
                                __uint_as_float(o[e + 3]));
        }
    } else if (warp_rows) {
        for (int c = 0; c < kC4; ++c) stg4[r * kC4 + c] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    sml[r] = make_float2(m_run, l_run);
    if (tid == 0 && kt0 < kt1) {
        // Every MMA issued above is complete before TMEM is released (after a
        // wait that gave up too).
        tc_commit(bar(kVBarDrain));
        wait(bar(kVBarDrain), 0);
    }
    tc_fence_before();
    cluster_sync();  // every partial of this kv head is staged
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kVTmemCols);
    }
    const uint32_t stg_addr = smem_u32(stg4), sml_addr = smem_u32(sml);
    const int n_items = rows * kC4;
    const int i_end = (split + 1) * n_items / C;
    for (int i = split * n_items / C + tid; i < i_end; i += kVThreads) {
        const int row = i / kC4, c = i % kC4;
        const uint32_t ml_off = sml_addr + uint32_t(row) * 8u;
        const uint32_t o_off = stg_addr + uint32_t(row * kC4 + (c ^ (row & 7))) * 16u;
        // Every partial's (m, l) and O chunk requested at once.
        float2 ml[kMaxVerifySplits];
        float4 v[kMaxVerifySplits];
#pragma unroll
        for (int q = 0; q < kMaxVerifySplits; ++q) {
            if (q < C) {
                ml[q] = ld_dsmem_f2(map_to_rank(ml_off, uint32_t(q)));
                v[q] = ld_dsmem_f4(map_to_rank(o_off, uint32_t(q)));
            }
        }
        float M = -INFINITY;
#pragma unroll
        for (int q = 0; q < kMaxVerifySplits; ++q)
            if (q < C) M = fmaxf(M, ml[q].x);
        float lsum = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int q = 0; q < kMaxVerifySplits; ++q) {
            if (q < C && ml[q].x != -INFINITY) {
                const float wgt = ex2_approx(ml[q].x - M);
                lsum += wgt * ml[q].y;
                acc.x += wgt * v[q].x;
                acc.y += wgt * v[q].y;
                acc.z += wgt * v[q].z;
                acc.w += wgt * v[q].w;
            }
        }
        const float sc = lsum > 0.f ? 1.f / lsum : 0.f;
        float* dst = p.out + ((size_t)(row / p.G) * p.H + kvh * p.G + row % p.G) * D;
        reinterpret_cast<float4*>(dst)[c] = make_float4(acc.x * sc, acc.y * sc, acc.z * sc, acc.w * sc);
    }
    cluster_sync();  // no CTA leaves while others still read its shared memory
}

template <int D>
cudaError_t launch_d(const VerifyParams& p, const CUtensorMap& tkh, const CUtensorMap& tkl, const CUtensorMap& tv,
                     cudaStream_t stream) {
    const size_t smem = size_t(VLayout<D>::kSmemBytes);
    cudaError_t e = ensure_smem_attr<verify_attn_kernel<D>>(int(smem));
    if (e != cudaSuccess) return e;
    if (p.splits > 8) {
        // Clusters above the portable 8 CTAs (up to 16 on B200) must be allowed per function.
        e = cudaFuncSetAttribute(verify_attn_kernel<D>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(p.Hkv * p.splits));
    cfg.blockDim = dim3(kVThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = unsigned(p.splits);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = overlapped_launch_enabled() ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, verify_attn_kernel<D>, p, tkh, tkl, tv);
}

}  // namespace

cudaError_t launch_verify_attn(const VerifyParams& p, const CUtensorMap& tkh, const CUtensorMap& tkl,
                               const CUtensorMap& tv, cudaStream_t stream) {
    if (p.splits < 1 || p.splits > kMaxVerifySplits) return cudaErrorInvalidValue;
    cudaError_t e = p.d == 128 ? launch_d<128>(p, tkh, tkl, tv, stream) : launch_d<64>(p, tkh, tkl, tv, stream);
    if (e != cudaSuccess && p.splits > 8) {
        // A cluster above the portable size could not be formed: fall back to 8 CTAs.
        cudaGetLastError();
        VerifyParams q = p;
        q.splits = 8;
        e = p.d == 128 ? launch_d<128>(q, tkh, tkl, tv, stream) : launch_d<64>(q, tkh, tkl, tv, stream);
    }
    return e;
}

}  // namespace fs
