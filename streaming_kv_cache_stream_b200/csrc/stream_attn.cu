// stream_attn -- attention of a window's new tokens against the streaming KV
// cache, on B200 tensor cores (tcgen05, accumulators in TMEM, TMA-staged tiles).
//
// Method (FlashDrive, arXiv 2608.12932; technical summary on gist.science,
// Methodology 1): keys are cached pre-RoPE in a view-major layout and rotated
// on the fly at the position they hold in the current (shifted) window; the
// new-frame and text queries attend under the streaming mask "query p sees key
// q iff pos(q) <= pos(p)".
//
// Work unit: a pair of CTAs on two SMs (a cluster of 2, tcgen05 cta_group::2)
// takes four 128-row query tiles of one kv head, as two query groups a and b
// of M = 256 rows (each CTA holds 128 rows of each group). Every key tile is
// staged once per pair (each CTA holds half of it: 64 of the 128 keys, D/2 of
// the V columns) and multiplied against both groups, so the pair reads 96 KB
// of operands per 512 query rows: on B200 the tensor pipes of all SMs would
// otherwise need more from L2 than it delivers. A query tile packs 128/G
// tokens x the G query heads of one kv group (GQA). The keys were rotated once
// by kv_stream_insert (fp16 hi + lo at angle index position + k*n, k the ring
// state's step count; V as fp16); this kernel rotates its query rows at their
// positions + k*n, read from the device-resident ring state.
//
// Warp roles per CTA (12 warps):
//   warps 0-3   prologue: classify the key tiles against the unit's and each
//               group's query range; then
//   warp 0      TMA producer: this CTA's halves of K hi/lo and V, 2 + 2 stages;
//   warp 1      TMEM allocation; in the even CTA, the single MMA issuer;
//   warps 4-11  prologue: RoPE of the query rows (group a: 4-7, group b: 8-11)
//               from a TMA-loaded bf16 tile, in place in shared memory; then
//               the online softmax of every S tile of both groups, warpgroup w
//               on key columns [64 w, 64 w + 64); then the epilogue, warpgroup
//               w finishing group w.
// TMEM per CTA: S_a, S_b (fp32 scores, 128 columns each; P as fp16 over the
// first 64 columns of its S) and O_a, O_b (fp32, D columns each).
// The kernel is launched with programmatic stream serialisation: it waits for
// the previous kernel on the stream (the insert that wrote its operands) at
// entry, and lets the next one start launching.
// MMA issue order for key tile k: QK_a(k), PV_b(k-1), QK_b(k), PV_a(k). A QK
// into S_g waits for the previous PV_g (it reads P_g from the same columns),
// and that wait always has other work queued on the tensor pipe; while one
// group's softmax runs, the tensor pipe works for the other group. A commit
// of S_g(k) also orders the preceding PV_g(k-1), so the softmax may rescale
// O_g in place before it hands over P_g(k).
// Key tiles are walked in physical ring order; positions come from key_pos(),
// so the ring never moves. Tiles whose every key is after the pair's last
// query are skipped; per group, tiles entirely visible to it skip the
// elementwise mask.
//
// Precision. Rotation happens in fp32 from the bf16 inputs and a table of
// fp32 cos/sin evaluated in double. The rotated Q (pre-scaled by log2(e)/sqrt(d))
// and K are each split into fp16 hi + lo parts and the scores are accumulated
// in fp32 as Q_hi K_hi + Q_hi K_lo + Q_lo K_hi: a single fp16 rounding of the
// rotated operands (2^-12 relative) moves the softmax weights of competing
// large-norm keys by ~1e-2 at the 1%-outlier-key workload, the split brings
// the scores to ~2^-22 relative. P is fp16 (V is fp16 to match), O
// accumulates in fp32, and the output is stored in fp32.
//
// Shared-memory tiles use the swizzled layouts TMA writes and tcgen05 reads:
// 128-byte rows with 16-byte chunk c of row r at chunk position c ^ (r & 7)
// (head dims 64..127 in a second region), or 64-byte rows for V at D = 64.
#include <cfloat>
#include <climits>
#include <mutex>

#include "fs_internal.cuh"
#include "sm100.cuh"

namespace fs {
namespace {

constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;
// Rescale O only when the running max grows by more than 2^14: P = 2^(s - m)
// then stays below 2^14 (fp16 holds up to 65504), so most tiles skip it.
constexpr float kRescaleLog2 = 14.0f;
constexpr int kKStages = 2;  // K hi/lo stages per CTA
constexpr int kVStages = 2;  // V stages per CTA

__device__ __forceinline__ constexpr uint32_t col_s(int grp) { return grp ? 128u : 0u; }
__device__ __forceinline__ constexpr uint32_t col_o(int grp) { return grp ? 384u : 256u; }

enum : int {
    kBarQReady0 = 0,                        // per group
    kBarKFull0 = kBarQReady0 + 2,           // per K stage
    kBarKEmpty0 = kBarKFull0 + kKStages,
    kBarVFull0 = kBarKEmpty0 + kKStages,    // per V stage
    kBarVEmpty0 = kBarVFull0 + kVStages,
    kBarSFull0 = kBarVEmpty0 + kVStages,    // per group: QK done
    kBarPFull0 = kBarSFull0 + 2,            // per group: P stored (and O rescaled)
    kBarPVDone0 = kBarPFull0 + 2,           // per group: PV done (S free again)
    kBarMmaDone = kBarPVDone0 + 2,
    kBarQLoad,                              // this CTA's bf16 query tiles landed (TMA)
    kNumBars
};

constexpr int kMaskWords = kMaxKeyTiles / 32;

struct Ctrl {
    uint64_t bars[kNumBars];
    alignas(16) int kpos[kTileRows];     // key positions of the tile being masked
    uint16_t red_m[2][2][kTileRows];     // [group][column half][row]: partial row max, 16 bits at a time
    uint32_t vis[kMaskWords];            // key tile visible to some query of the pair
    uint32_t part[2][kMaskWords];        // per group: tile needs the elementwise mask
    uint32_t tmem_base;
    int j_begin;                         // first visible tile of this key split
    int nt;                              // visible tiles in this key split
};
constexpr int kCtrlBytes = 3072;
static_assert(sizeof(Ctrl) <= kCtrlBytes, "control block too large");

// Per-CTA shared memory after the control block (1024-byte aligned): the
// CTA's 128 query rows of group a and of group b as fp16 hi and lo (128-byte
// swizzle, head dims 64..127 in a second region), then the K stages (this
// CTA's 64 keys of a tile, K hi then K lo), then the V stages (all 128 keys,
// this CTA's D/2 columns; 128-byte swizzle at D = 128, 64-byte at D = 64).
// At D = 128: 128 KB + 64 KB + 32 KB + 3 KB = 227 KB, all of a CTA's limit.
template <int D>
struct Layout {
    static constexpr int kQRegion = 128 * 128;                // 128 rows x 128 bytes
    static constexpr int kQHalf = 128 * D * 2;                // Q hi or Q lo of one group
    static constexpr int kKRegion = 64 * 128;                 // 64 key rows x 128 bytes
    static constexpr int kKHalf = 64 * D * 2;                 // K hi or K lo of a stage
    static constexpr int kKStage = 2 * kKHalf;
    static constexpr int kVRow = D;                           // bytes per key row of the V half
    static constexpr int kVStage = kTileRows * kVRow;
    static constexpr uint32_t kVLayout = D == 128 ? 2u : 4u;  // 128- or 64-byte swizzle
    static constexpr int kQ = 0;                              // [group][hi, lo]
    static constexpr int kK0 = 4 * kQHalf;
    static constexpr int kV0 = kK0 + kKStages * kKStage;
    static constexpr int kTiles = kV0 + kVStages * kVStage;
    static constexpr int kSmemBytes = kCtrlBytes + kTiles;    // dynamic shared memory per CTA
};

// Lowest and highest window position among physical key rows [r0, r1). Rows of
// one ring slot (or the text) are consecutive positions, so walking slot-sized
// runs is exact.
__device__ __forceinline__ void key_bounds(const WindowShape& w, int head, int r0, int r1, int& lo, int& hi) {
    lo = INT_MAX;
    hi = INT_MIN;
    int r = r0;
    while (r < r1) {
        int end = r1;
        if (r < w.ring_rows) {
            const int slot_end = (r / w.n + 1) * w.n;
            end = slot_end < r1 ? slot_end : r1;
        }
        const int a = key_pos(w, head, r);
        const int b = a + (end - 1 - r);
        lo = a < lo ? a : lo;
        hi = b > hi ? b : hi;
        r = end;
    }
}

// fp32 pair -> fp16 hi pair + fp16 lo pair (lo = the rounding residual of hi).
__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
    hi = pack_f16x2(a, b);
    const float2 hf = __half22float2(*reinterpret_cast<const __half2*>(&hi));
    lo = pack_f16x2(a - hf.x, b - hf.y);
}

// Rotates one query row (pre-RoPE bf16 in global memory) by the angles in
// `cs`, scales it by `scale`, and writes it as fp16 hi / lo into row `row` of
// the swizzled Q tiles `qhi` / `qlo` (the K-major A operand of the QK MMA).
// Pair (i, i + D/2): for D = 128 chunk c of region 0 pairs with chunk c of
// region 1; for D = 64 chunk c pairs with chunk c + 4.
template <int D, typename Ready>
__device__ __forceinline__ bool rope_query_row(const float2* __restrict__ cs, float scale, uint8_t* qhi, uint8_t* qlo,
                                               int row, Ready ready) {
    constexpr int kPairs = D / 16;  // 16-byte chunk pairs (c, c + D/16) of the row
    constexpr int kHalf = kPairs / 2;
    const int sw = row & 7;
    // The first half of the row's cos/sin is in flight while the query tile lands.
    float4 t[kHalf][4];
#pragma unroll
    for (int u = 0; u < kHalf; ++u)
#pragma unroll
        for (int q = 0; q < 4; ++q) t[u][q] = __ldg(reinterpret_cast<const float4*>(cs + 8 * u) + q);
    const bool ok = ready();  // on a timeout the rows rotate whatever is there; the error is reported
    (void)ok;
    // Read the whole bf16 row before overwriting its lo half in place.
    bool in_range = true;  // every element finite and at most 65504 in magnitude (NaN fails too)
    uint4 a[kPairs], b[kPairs];
#pragma unroll
    for (int c = 0; c < kPairs; ++c) {
        const int oa = row * 128 + ((c ^ sw) << 4);
        const int ob = D == 128 ? oa + Layout<D>::kQRegion : row * 128 + (((c + 4) ^ sw) << 4);
        a[c] = *reinterpret_cast<const uint4*>(qlo + oa);
        b[c] = *reinterpret_cast<const uint4*>(qlo + ob);
    }
#pragma unroll
    for (int c = 0; c < kPairs; ++c) {
        const int u = c % kHalf;
        if (c == kHalf) {
#pragma unroll
            for (int v = 0; v < kHalf; ++v)
#pragma unroll
                for (int q = 0; q < 4; ++q) t[v][q] = __ldg(reinterpret_cast<const float4*>(cs + 8 * (kHalf + v)) + q);
        }
        const int oa = row * 128 + ((c ^ sw) << 4);
        const int ob = D == 128 ? oa + Layout<D>::kQRegion : row * 128 + (((c + 4) ^ sw) << 4);
        const uint32_t aw[4] = {a[c].x, a[c].y, a[c].z, a[c].w};
        const uint32_t bw[4] = {b[c].x, b[c].y, b[c].z, b[c].w};
        uint32_t ah[4], al[4], bh[4], bl[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 tq = t[u][q];  // (cos, sin) of elements 8c + 2q and 8c + 2q + 1
            const float x0 = bf16lo(aw[q]), x1 = bf16hi(aw[q]);
            const float y0 = bf16lo(bw[q]), y1 = bf16hi(bw[q]);
            const float r0 = (x0 * tq.x - y0 * tq.y) * scale, r1 = (x1 * tq.z - y1 * tq.w) * scale;
            const float s0 = (y0 * tq.x + x0 * tq.y) * scale, s1 = (y1 * tq.z + x1 * tq.w) * scale;
            in_range = in_range && fabsf(r0) <= kF16Max && fabsf(r1) <= kF16Max && fabsf(s0) <= kF16Max &&
                       fabsf(s1) <= kF16Max;
            split2(r0, r1, ah[q], al[q]);
            split2(s0, s1, bh[q], bl[q]);
        }
        *reinterpret_cast<uint4*>(qhi + oa) = make_uint4(ah[0], ah[1], ah[2], ah[3]);
        *reinterpret_cast<uint4*>(qhi + ob) = make_uint4(bh[0], bh[1], bh[2], bh[3]);
        *reinterpret_cast<uint4*>(qlo + oa) = make_uint4(al[0], al[1], al[2], al[3]);
        *reinterpret_cast<uint4*>(qlo + ob) = make_uint4(bl[0], bl[1], bl[2], bl[3]);
    }
    return in_range;
}

// Uniform decision over `threads` threads at named barrier `id`: true iff all pass `ok`.
__device__ __forceinline__ bool vote_all_ok(uint32_t id, uint32_t threads, bool ok) {
    uint32_t res;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %3, 0;\n\t"
        "barrier.red.and.pred q, %1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(res)
        : "r"(id), "r"(threads), "r"(uint32_t(ok))
        : "memory");
    return res != 0;
}

// Smallest visible key tile index >= j (the caller knows one exists).
__device__ __forceinline__ int next_visible(const uint32_t* vis, int j) {
    int w = j >> 5;
    uint32_t bits = vis[w] & (0xFFFFFFFFu << (j & 31));
    while (bits == 0 && w + 1 < kMaskWords) bits = vis[++w];
    return bits ? (w << 5) + __ffs(bits) - 1 : j;
}

__device__ __forceinline__ bool test_bit(const uint32_t* m, int j) { return (m[j >> 5] >> (j & 31)) & 1u; }

// bf16 of x rounded toward +inf (-inf stays -inf), as raw bits.
__device__ __forceinline__ uint16_t bf16_round_up(float x) {
    uint32_t u = __float_as_uint(x);
    if (x > 0.f) u += 0xFFFFu;
    return uint16_t(u >> 16);
}
__device__ __forceinline__ float bf16_to_float(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }

template <int D>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    stream_attn_kernel(const __grid_constant__ AttnParams p, const __grid_constant__ CUtensorMap tq,
                       const __grid_constant__ CUtensorMap tkh, const __grid_constant__ CUtensorMap tkl,
                       const __grid_constant__ CUtensorMap tv16) {
    using L = Layout<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    Ctrl& ctrl = *reinterpret_cast<Ctrl*>(smem_raw);
    uint8_t* smem = smem_raw + kCtrlBytes;  // operand tiles
    {
        // Both CTAs of a pair see the same layout, so both leave here together.
        uint32_t dyn;
        asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
        if ((smem_u32(smem) & 1023u) != 0 || dyn < uint32_t(L::kSmemBytes)) {
            if (threadIdx.x == 0) atomicOr(p.err, kErrBadLaunch);
            return;
        }
    }
    grid_dependency_wait();     // the insert that wrote this call's operands is done
    allow_dependents_launch();  // the next kernel may start its set-up
    // Ring head and angle offset as the last insert left them (the window shape
    // itself stays in the parameter space).
    const WindowShape& w = p.w;
    int head, angle_off;
    {
        const int2 rs = load_ring_state(p.state);
        head = rs.x;
        angle_off = rs.y * w.n;
    }
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const uint32_t rank = cluster_rank();  // 0: leader (issues the pair's MMAs), 1: peer
    const bool leader = rank == 0;

    // ---- work item: four query tiles 4u .. 4u+3 of one kv head (group a: 4u, 4u+1;
    // group b: 4u+2, 4u+3; this CTA holds 4u + 2 grp + rank); heavy units first.
    const int pair_id = blockIdx.x >> 1;
    const int split = pair_id % p.splits;
    const int item = pair_id / p.splits;
    const int units = (p.q_tiles + 3) >> 2;
    const int u = units - 1 - item / p.Hkv;
    const int kvh = item % p.Hkv;
    const int tpt = kTileRows / p.G;  // tokens per query tile
    const int unit_t0 = 4 * u * tpt;
    const int unit_t1 = min(unit_t0 + 4 * tpt, p.nq);
    const int unit_qmax = query_pos(w, p.q_mode, unit_t1 - 1);
    const BoundedWait wait{p.err, p.wait_limit_ns, kErrTimeout};

    auto bar = [&](int i) { return smem_u32(&ctrl.bars[i]); };
    auto lbar = [&](int i) { return map_to_rank(smem_u32(&ctrl.bars[i]), 0); };  // the leader's copy

    if (tid == 0) {
        for (int g = 0; g < 2; ++g) {
            mbar_init(bar(kBarQReady0 + g), 8);  // one arrival per RoPE warp of the group, both CTAs
            mbar_init(bar(kBarSFull0 + g), 1);
            mbar_init(bar(kBarPFull0 + g), 16);  // one arrival per softmax warp (8 per CTA), both CTAs
            mbar_init(bar(kBarPVDone0 + g), 1);
        }
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(bar(kBarKFull0 + s), 1);
            mbar_init(bar(kBarKEmpty0 + s), 1);
        }
        for (int s = 0; s < kVStages; ++s) {
            mbar_init(bar(kBarVFull0 + s), 1);
            mbar_init(bar(kBarVEmpty0 + s), 1);
        }
        mbar_init(bar(kBarMmaDone), 1);
        mbar_init(bar(kBarQLoad), 1);
        fence_mbar_init();
        // This CTA's rows of both query groups, bf16, into the Q lo regions (the
        // layout the rotation reads and overwrites in place); rows past the last
        // token read as zero.
        mbar_arrive_expect_tx(bar(kBarQLoad), 2 * L::kQHalf);
#pragma unroll
        for (int g = 0; g < 2; ++g)
#pragma unroll
            for (int reg = 0; reg < D / 64; ++reg)
                tma_load_3d(smem_u32(smem + L::kQ + (2 * g + 1) * L::kQHalf + reg * L::kQRegion), &tq, 64 * reg,
                            kvh * p.G, (4 * u + 2 * g + int(rank)) * tpt, bar(kBarQLoad));
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(&ctrl.tmem_base), kTmemCols);
        tmem_relinquish_pair();
    }
    __syncthreads();  // barriers initialised before anyone waits on them
    cluster_arrive();  // pairs with cluster_wait before the first cross-CTA operation

    // ---- prologue, split by warpgroup (each runs under its own register limit):
    // warps 0-3 classify the key tiles against the unit's and each group's query
    // range and place this split's share; warps 4-7 (group a) and 8-11 (group b)
    // meanwhile rotate their query rows into shared memory.
    // Register split, one setmaxnreg per warpgroup at the head of its region:
    // 128 x (96 + 200 + 200) <= 384 x 168, the registers allocated at launch.
    uint32_t tmem = 0;
    int nt = 0, j_begin = 0;
    const uint32_t lane_off = uint32_t(32 * (warp & 3)) << 16;  // TMEM lanes of this warp
    // The control block and the TMEM base are complete before anyone reads them
    // (warps 0-3 publish them at named barrier 4 without waiting for the query
    // rotation); both CTAs' barriers exist before any cross-CTA arrive or commit.
    auto prologue_sync = [&](bool publisher) {
        tc_fence_before();
        if (publisher) asm volatile("bar.arrive 4, 384;" ::: "memory");
        else named_bar_sync(4, 384);
        cluster_wait();
        tc_fence_after();
        tmem = ctrl.tmem_base;
        nt = ctrl.nt;
        j_begin = ctrl.j_begin;
    };
    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 96;");
        const int n_ktiles = (p.key_rows + kTileRows - 1) / kTileRows;
        {
            int gmin[2], gmax[2];
            bool gpresent[2];
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                const int t0 = unit_t0 + 2 * g * tpt;
                const int t1 = min(t0 + 2 * tpt, p.nq);
                gpresent[g] = t0 < t1;
                gmin[g] = gpresent[g] ? query_pos(w, p.q_mode, t0) : 0;
                gmax[g] = gpresent[g] ? query_pos(w, p.q_mode, t1 - 1) : 0;
            }
            const int words = (n_ktiles + 31) >> 5;
            for (int wd = warp; wd < words; wd += 4) {
                const int j = wd * 32 + lane;
                bool v = false, pa = true, pb = true;
                if (j < n_ktiles) {
                    const int r0 = j * kTileRows;
                    const int r1 = min(r0 + kTileRows, p.key_rows);
                    int lo, hi;
                    key_bounds(w, head, r0, r1, lo, hi);
                    v = lo <= unit_qmax;
                    const bool full_tile = r1 - r0 == kTileRows;
                    pa = !(gpresent[0] && hi <= gmin[0] && full_tile);
                    pb = !(gpresent[1] && hi <= gmin[1] && full_tile);
                }
                const uint32_t bv = __ballot_sync(0xffffffffu, v);
                const uint32_t ba = __ballot_sync(0xffffffffu, pa);
                const uint32_t bb = __ballot_sync(0xffffffffu, pb);
                if (lane == 0) {
                    ctrl.vis[wd] = bv;
                    ctrl.part[0][wd] = ba;
                    ctrl.part[1][wd] = bb;
                }
            }
            (void)gmax;
        }
        named_bar_sync(3, 128);  // warps 0-3: the masks are complete
        if (tid == 0) {
            // This split's share of the visible tiles: [kbeg, kend) in visible order.
            const int words = (n_ktiles + 31) >> 5;
            int nvis = 0;
            for (int wd = 0; wd < words; ++wd) nvis += __popc(ctrl.vis[wd]);
            const int kbeg = int((long long)split * nvis / p.splits);
            const int kend = int((long long)(split + 1) * nvis / p.splits);
            int j = 0, seen = 0;
            for (int wd = 0; wd < words; ++wd) {
                const int c = __popc(ctrl.vis[wd]);
                if (seen + c > kbeg) {
                    uint32_t bits = ctrl.vis[wd];
                    for (int skip = kbeg - seen; skip > 0; --skip) bits &= bits - 1;
                    j = wd * 32 + __ffs(bits) - 1;
                    break;
                }
                seen += c;
            }
            ctrl.j_begin = j;
            ctrl.nt = kend - kbeg;
        }
        named_bar_sync(3, 128);  // warps 0-3: the split is placed
        prologue_sync(true);
        if (warp == 0) {
            // ============================================= TMA producer (both CTAs)
            // Each CTA loads its half of every operand tile: keys [64 r, 64 r + 64)
            // of K hi/lo, columns [D/2 r, D/2 r + D/2) of V; the leader's full
            // barriers count the bytes of both CTAs.
            if (lane == 0 && nt > 0) {
                tma_prefetch_desc(&tkh);
                tma_prefetch_desc(&tkl);
                tma_prefetch_desc(&tv16);
                int j = j_begin;
                for (int k = 0; k < nt; ++k) {
                    if (k > 0) j = next_visible(ctrl.vis, j + 1);
                    const int ks = k % kKStages;
                    if (!wait(bar(kBarKEmpty0 + ks), ((k / kKStages) & 1) ^ 1)) break;
                    if (leader) mbar_arrive_expect_tx(bar(kBarKFull0 + ks), 2 * L::kKStage);
                    const uint32_t kd = smem_u32(smem + L::kK0 + ks * L::kKStage);
#pragma unroll
                    for (int r = 0; r < D / 64; ++r) {
                        tma_load_3d_pair(kd + r * L::kKRegion, &tkh, r * 64, j * kTileRows + 64 * int(rank), kvh,
                                         lbar(kBarKFull0 + ks));
                        tma_load_3d_pair(kd + L::kKHalf + r * L::kKRegion, &tkl, r * 64,
                                         j * kTileRows + 64 * int(rank), kvh, lbar(kBarKFull0 + ks));
                    }
                    const int vs = k % kVStages;
                    if (!wait(bar(kBarVEmpty0 + vs), ((k / kVStages) & 1) ^ 1)) break;
                    if (leader) mbar_arrive_expect_tx(bar(kBarVFull0 + vs), 2 * L::kVStage);
                    tma_load_3d_pair(smem_u32(smem + L::kV0 + vs * L::kVStage), &tv16, (D / 2) * int(rank),
                                     j * kTileRows, kvh, lbar(kBarVFull0 + vs));
                }
            }
        } else if (warp == 1) {
            // ============================================= MMA issuer (leader CTA only)
            if (leader && lane == 0 && nt > 0) {
                constexpr uint32_t idesc_qk = idesc_f16(256, 128, false, false, false, false);
                constexpr uint32_t idesc_pv = idesc_f16(256, D, false, false, false, true);
                // Descriptors are formed once; a K step advances the start-address
                // field (bits 0-13, in 16-byte units) by the step's offset.
                const uint64_t dq0 = sw128_desc(smem_u32(smem + L::kQ), 16, 1024);
                const uint64_t dk0 = sw128_desc(smem_u32(smem + L::kK0), 16, 1024);
                const uint64_t dv0 = smem_desc(smem_u32(smem + L::kV0), L::kVStage, 8 * L::kVRow, L::kVLayout);
                // S_g = Q_g K^T over the three hi/lo products.
                auto issue_qk = [&](int grp, int ks) {
                    const uint64_t dqh = dq0 + uint32_t((2 * grp * L::kQHalf) >> 4);
                    const uint64_t dql = dqh + uint32_t(L::kQHalf >> 4);
                    const uint64_t dkh = dk0 + uint32_t((ks * L::kKStage) >> 4);
                    const uint64_t dkl = dkh + uint32_t(L::kKHalf >> 4);
                    const uint32_t d_s = tmem + col_s(grp);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t qo = ((kk >> 2) * L::kQRegion + (kk & 3) * 32) >> 4;
                        const uint32_t ko = ((kk >> 2) * L::kKRegion + (kk & 3) * 32) >> 4;
                        mma_ss_pair(d_s, dqh + qo, dkh + ko, idesc_qk, kk > 0);
                        mma_ss_pair(d_s, dqh + qo, dkl + ko, idesc_qk, 1);
                        mma_ss_pair(d_s, dql + qo, dkh + ko, idesc_qk, 1);
                    }
                };
                // O_g (+)= P_g V, P_g (fp16) from the first 64 columns of S_g.
                auto issue_pv = [&](int grp, int vs, bool first) {
                    const uint64_t dv = dv0 + uint32_t((vs * L::kVStage) >> 4);
#pragma unroll
                    for (int kk = 0; kk < kTileRows / 16; ++kk)
                        mma_ts_pair(tmem + col_o(grp), tmem + col_s(grp) + kk * 8, dv + ((kk * 16 * L::kVRow) >> 4),
                                    idesc_pv, (!first || kk > 0));
                };
                bool ok = wait(bar(kBarQReady0 + 0), 0) && wait(bar(kBarQReady0 + 1), 0);
                for (int k = 0; ok && k <= nt; ++k) {
                    const int ks = k % kKStages;
                    if (k < nt) {
                        if (!(ok = wait(bar(kBarKFull0 + ks), (k / kKStages) & 1))) break;
                        if (k > 0 && !(ok = wait(bar(kBarPVDone0 + 0), (k - 1) & 1))) break;
                        tc_fence_after();
                        issue_qk(0, ks);
                        tc_commit_pair(bar(kBarSFull0 + 0));
                    }
                    if (k > 0) {
                        const int kp = k - 1;
                        const int vs = kp % kVStages;
                        if (!(ok = wait(bar(kBarPFull0 + 1), kp & 1))) break;
                        tc_fence_after();
                        issue_pv(1, vs, kp == 0);
                        tc_commit_pair(bar(kBarPVDone0 + 1));
                        tc_commit_pair(bar(kBarVEmpty0 + vs));
                    }
                    if (k < nt) {
                        if (k > 0 && !(ok = wait(bar(kBarPVDone0 + 1), (k - 1) & 1))) break;
                        tc_fence_after();
                        issue_qk(1, ks);
                        tc_commit_pair(bar(kBarSFull0 + 1));
                        tc_commit_pair(bar(kBarKEmpty0 + ks));
                        const int vs = k % kVStages;
                        if (!(ok = wait(bar(kBarPFull0 + 0), k & 1))) break;
                        if (!(ok = wait(bar(kBarVFull0 + vs), (k / kVStages) & 1))) break;
                        tc_fence_after();
                        issue_pv(0, vs, k == 0);
                        tc_commit_pair(bar(kBarPVDone0 + 0));
                    }
                }
                // Drain: every MMA issued above completes before TMEM is read or released.
                tc_commit_pair(bar(kBarMmaDone));
                wait(bar(kBarMmaDone), 0);
            }
        }
    } else {
        // ================================================= query groups: RoPE, softmax, epilogue
        asm volatile("setmaxnreg.inc.sync.aligned.u32 200;");
        const int grp = warp >= 8 ? 1 : 0;
        const int r = (tid - 128) & 127;  // row = TMEM lane
        const int qt = 4 * u + 2 * grp + int(rank);
        const bool tile_valid = qt < p.q_tiles;
        const int t = qt * tpt + r / p.G;
        {
            // Rotate this group's query rows (landed by TMA) in shared memory while
            // warps 0-3 classify the key tiles; rows past the last token rotate
            // zeros and are never stored.
            const int qp0 = query_pos(w, p.q_mode, (tile_valid && t < p.nq) ? t : unit_t0);
            uint8_t* qg = smem + L::kQ + 2 * grp * L::kQHalf;
            const bool in_range =
                rope_query_row<D>(p.rope + (size_t)(qp0 + angle_off) * (D / 2), p.q_scale, qg, qg + L::kQHalf, r,
                                  [&] { return wait(bar(kBarQLoad), 0); });
            if (!in_range && tile_valid && t < p.nq) atomicOr(p.err, kErrRange);
            fence_proxy_async_smem();  // generic stores -> read by the tensor core
        }
        prologue_sync(false);
        if (nt > 0 && lane == 0) mbar_arrive_cluster(lbar(kBarQReady0 + grp));  // rows rotated in the prologue

        // ---- softmax: both warpgroups on every S tile of both groups; warpgroup
        // hw takes columns [64 hw, 64 hw + 64) of the 128 keys (two warps per SM
        // sub-partition on each tile). The halves agree on the row max through
        // shared memory (see the exchange below: both compute the same base, at
        // or above the true max, so P <= 1), keep their own partial row sums,
        // and rescale their own D/2 columns of O.
        const int hw = grp;                // column half (the warpgroup)
        int qpos[2];                       // this row's query position in group g (-1: no query)
        bool rvalid[2];
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            const int qtg = 4 * u + 2 * g + int(rank);
            const int tg = qtg * tpt + r / p.G;
            rvalid[g] = qtg < p.q_tiles && tg < p.nq;
            qpos[g] = rvalid[g] ? query_pos(w, p.q_mode, tg) : -1;
        }
        float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
        bool ok = true;
        int j = j_begin;
        for (int k = 0; ok && k < nt; ++k) {
            if (k > 0) j = next_visible(ctrl.vis, j + 1);
            const bool pa = test_bit(ctrl.part[0], j), pb = test_bit(ctrl.part[1], j);
            if (pa || pb) {
                // Key position of every column of the tile, for the elementwise
                // streaming mask (the same key tile serves both groups).
                if (hw == 0) {
                    const int row = j * kTileRows + r;
                    ctrl.kpos[r] = row < p.key_rows ? key_pos(w, head, row) : INT_MAX;
                }
                named_bar_sync(5, 256);
            }
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                const uint32_t s_col = tmem + col_s(g) + lane_off + 64 * hw;
                const bool w_ok = wait(bar(kBarSFull0 + g), k & 1);
                tc_fence_after();
                uint32_t sr[2][32];
                tmem_ld32(s_col, sr[0]);
                tmem_ld32(s_col + 32, sr[1]);
                tmem_wait_ld();
                if (g == 0 ? pa : pb) {
                    const int qp = qpos[g];
#pragma unroll
                    for (int c4 = 0; c4 < 16; ++c4) {
                        const int4 k4 = *reinterpret_cast<const int4*>(ctrl.kpos + 64 * hw + 4 * c4);
                        const uint32_t ninf = __float_as_uint(-INFINITY);
                        uint32_t* q4 = &sr[c4 >> 3][(c4 & 7) * 4];
                        if (k4.x > qp) q4[0] = ninf;
                        if (k4.y > qp) q4[1] = ninf;
                        if (k4.z > qp) q4[2] = ninf;
                        if (k4.w > qp) q4[3] = ninf;
                    }
                }
                // Partial row max of this half: three-input max into 8 independent maxima.
                float mx[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) mx[i] = __uint_as_float(sr[0][i]);
#pragma unroll
                for (int c = 8; c < 64; c += 2)
                    mx[(c >> 1) & 7] = fmax3(mx[(c >> 1) & 7], __uint_as_float(sr[c >> 5][c & 31]),
                                             __uint_as_float(sr[c >> 5][(c + 1) & 31]));
                const float mh = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
                // Row max over both halves, exchanged through shared memory: each
                // half stores its maximum rounded up to bf16 and both take the
                // larger, so they agree on one base at or above the true row max
                // (P <= 1). Rounding up by at most 2^-8 of the value keeps the base
                // within 1 of the true max while |max| < 256 (log2 units); beyond
                // that the base could overshoot enough to flush every P to zero,
                // so such rows exchange their exact fp32 maxima, 16 bits at a time.
                ctrl.red_m[g][hw][r] = bf16_round_up(mh);
                // Exchange point, and the uniform decision: a failed wait anywhere
                // ends the loop for all 256 threads together.
                if (!vote_all_ok(6, 256, w_ok && ok)) {
                    ok = false;
                    break;
                }
                float mt = fmaxf(bf16_to_float(ctrl.red_m[g][0][r]), bf16_to_float(ctrl.red_m[g][1][r]));
                // The two halves of these 32 rows are warps (warp & 3) and (warp & 3) + 4
                // of the two warpgroups; both see the same stored values, so they
                // take this branch together and meet at their own named barrier.
                if (__any_sync(0xffffffffu, !(fabsf(mt) < 256.f) && mt != -INFINITY)) {
                    const uint32_t pair_bar = 7u + uint32_t(warp & 3);
                    const uint32_t bits = __float_as_uint(mh);
                    named_bar_sync(pair_bar, 64);  // both halves have read the rounded values
                    ctrl.red_m[g][hw][r] = uint16_t(bits >> 16);
                    named_bar_sync(pair_bar, 64);
                    const uint32_t hi = ctrl.red_m[g][hw ^ 1][r];
                    named_bar_sync(pair_bar, 64);
                    ctrl.red_m[g][hw][r] = uint16_t(bits & 0xFFFFu);
                    named_bar_sync(pair_bar, 64);
                    const uint32_t lo = ctrl.red_m[g][hw ^ 1][r];
                    mt = fmaxf(mh, __uint_as_float((hi << 16) | lo));  // same value in both halves
                }
                const float m_new = fmaxf(m_run[g], mt);
                const bool resc = m_new > m_run[g] + kRescaleLog2;
                const float m_use = resc ? m_new : m_run[g];
                const float alpha = resc ? ex2_approx(m_run[g] - m_use) : 1.f;
                const float base = (m_use == -INFINITY) ? 0.f : m_use;
                const uint64_t base2 = f2pack(base, base);
                uint64_t acc[4] = {0, 0, 0, 0};  // paired partial row sums
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t pk[16];
#pragma unroll
                    for (int c2 = 0; c2 < 16; ++c2) {
                        float d0, d1;
                        f2unpack(sub2(f2pack(__uint_as_float(sr[h][2 * c2]), __uint_as_float(sr[h][2 * c2 + 1])),
                                      base2),
                                 d0, d1);
                        const float p0 = ex2_approx(d0);
                        const float p1 = ex2_approx(d1);
                        acc[c2 & 3] = add2(acc[c2 & 3], f2pack(p0, p1));
                        pk[c2] = pack_f16x2(p0, p1);
                    }
                    // P (fp16 pairs): keys 64 hw + 32 h .. + 31 -> packed columns 32 hw + 16 h ..
                    tmem_st16(tmem + col_s(g) + lane_off + 32 * hw + 16 * h, pk);
                }
                float rs;
                {
                    const uint64_t a01 = add2(acc[0], acc[1]), a23 = add2(acc[2], acc[3]);
                    float x0, x1;
                    f2unpack(add2(a01, a23), x0, x1);
                    rs = x0 + x1;
                }
                l_run[g] = l_run[g] * alpha + rs;
                if (k > 0 && __any_sync(0xffffffffu, resc)) {
                    // O_g holds the group's earlier PVs, the last of which completed
                    // before QK_g(k) was issued; rescale this half's columns in TMEM.
                    const uint32_t o_col = tmem + col_o(g) + lane_off + uint32_t(hw) * (D / 2);
#pragma unroll 1
                    for (int cc = 0; cc < D / 64; ++cc) {
                        uint32_t o[32];
                        tmem_ld32(o_col + 32 * cc, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st32(o_col + 32 * cc, o);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(lbar(kBarPFull0 + g));
                m_run[g] = m_use;
            }
        }
        // ---- epilogue: warpgroup hw finishes group hw: O / l in fp32 (or the
        // unnormalised split partial with (m, l)), l being the sum of the two
        // halves' partial sums, exchanged through the (now free) K stages.
        const int g = hw;  // qt, tile_valid above are this group's
        const size_t part_row = (((size_t)qt * p.Hkv + kvh) * p.splits + split) * kTileRows + r;
        if (ok && nt > 0) {
            const bool mma_ok = wait(bar(kBarMmaDone), 0);  // single phase: after the last PV
            float* red_l = reinterpret_cast<float*>(smem + L::kK0);  // [group][half][row]
            red_l[(0 * 2 + hw) * kTileRows + r] = l_run[0];
            red_l[(1 * 2 + hw) * kTileRows + r] = l_run[1];
            if (vote_all_ok(6, 256, mma_ok)) {
                tc_fence_after();
                const float l_tot = red_l[(g * 2 + 0) * kTileRows + r] + red_l[(g * 2 + 1) * kTileRows + r];
                const float sc = p.splits == 1 ? (l_tot > 0.f ? 1.f / l_tot : 0.f) : 1.f;
                const uint32_t o_col = tmem + col_o(g) + lane_off;
                uint8_t* stg = smem + L::kQ + 2 * g * L::kQHalf;
                constexpr int kRowBytes = D * 4;
#pragma unroll 1
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t o[32];
                    tmem_ld32(o_col + 32 * cc, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const int c = 8 * cc + q;
                        *reinterpret_cast<float4*>(stg + r * kRowBytes + ((c ^ (r & 7)) << 4)) =
                            make_float4(__uint_as_float(o[4 * q]) * sc, __uint_as_float(o[4 * q + 1]) * sc,
                                        __uint_as_float(o[4 * q + 2]) * sc, __uint_as_float(o[4 * q + 3]) * sc);
                    }
                }
                if (p.splits > 1 && tile_valid) p.part_ml[part_row] = make_float2(m_run[g], l_tot);
                // Warp w of the warpgroup copies rows 32 w .. 32 w + 31; lane i works
                // out the destination of row 32 w + i once and the copy loop
                // broadcasts it.
                const int row0 = (warp & 3) * 32;
                float* dmy = nullptr;
                {
                    const int rr = row0 + lane;
                    const int t2 = qt * tpt + rr / p.G;
                    if (tile_valid && (p.splits > 1 || t2 < p.nq))
                        dmy = p.splits == 1 ? p.out + ((size_t)t2 * p.H + kvh * p.G + rr % p.G) * D
                                            : p.part_o + (part_row - r + rr) * D;
                }
                named_bar_sync(1 + hw, 128);
                constexpr int kChunks = D / 4;              // 16-byte chunks per row
                constexpr int kRowsPerInstr = 32 / kChunks;  // rows one warp instruction covers
                const int c = lane % kChunks;
#pragma unroll 8
                for (int i = 0; i < 32; i += kRowsPerInstr) {
                    const int il = i + lane / kChunks;
                    float* drow = reinterpret_cast<float*>(
                        __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(dmy), il));
                    const int rr = row0 + il;
                    const float4 v = *reinterpret_cast<const float4*>(stg + rr * kRowBytes + ((c ^ (rr & 7)) << 4));
                    if (drow) reinterpret_cast<float4*>(drow)[c] = v;
                }
            }
        } else if (nt == 0 && p.splits > 1 && tile_valid) {
            p.part_ml[part_row] = make_float2(-INFINITY, 0.f);
        }
        (void)rvalid;
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // neither CTA releases TMEM or exits while the pair's MMAs could touch it
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

// Merge key splits: out = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s, M = max_s m_s.
template <int D>
__global__ void __launch_bounds__(128) attn_combine_kernel(const AttnParams p) {
    const int warp_global = (blockIdx.x * 128 + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int rows = p.Hkv * p.q_tiles * kTileRows;
    if (warp_global >= rows) return;
    const int item_id = warp_global / kTileRows;
    const int r = warp_global % kTileRows;
    const int qt = item_id / p.Hkv;
    const int kvh = item_id % p.Hkv;
    const int t = qt * (kTileRows / p.G) + r / p.G;
    const int g = r % p.G;
    if (t >= p.nq) return;
    float M = -INFINITY;
    for (int s = 0; s < p.splits; ++s) M = fmaxf(M, p.part_ml[((size_t)item_id * p.splits + s) * kTileRows + r].x);
    constexpr int kPer = D / 32;
    float acc[kPer];
#pragma unroll
    for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
    float lsum = 0.f;
    for (int s = 0; s < p.splits; ++s) {
        const size_t row = ((size_t)item_id * p.splits + s) * kTileRows + r;
        const float2 ml = p.part_ml[row];
        if (ml.x == -INFINITY) continue;
        const float wgt = ex2_approx(ml.x - M);
        lsum += wgt * ml.y;
#pragma unroll
        for (int e = 0; e < kPer; ++e) acc[e] += wgt * p.part_o[row * D + lane * kPer + e];
    }
    const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
    float* dst = p.out + ((size_t)t * p.H + kvh * p.G + g) * D + lane * kPer;
#pragma unroll
    for (int e = 0; e < kPer; ++e) dst[e] = acc[e] * inv;
}

// Window positions of physical rows [0, rows) as the attention kernel derives
// them (same function, head read from the device-resident ring state).
__global__ void positions_kernel(const WindowShape w0, const RingState* state, int rows, int* pos) {
    WindowShape w = w0;
    w.head = load_ring_state(state).x;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < rows) pos[i] = key_pos(w, i);
}

// Waits on a barrier that nothing completes; the bounded wait gives up and records it.
__global__ void wait_probe_kernel(unsigned* err, unsigned long long limit_ns) {
    __shared__ uint64_t b;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&b), 1);
        fence_mbar_init();
        const BoundedWait wait{err, limit_ns, kErrTimeout};
        wait(smem_u32(&b), 0);
    }
}

template <int D>
cudaError_t launch_d(const AttnParams& p, const CUtensorMap& tq, const CUtensorMap& tkh, const CUtensorMap& tkl,
                     const CUtensorMap& tv16, cudaStream_t stream) {
    const size_t smem = stream_attn_smem_bytes(D);
    cudaError_t e = ensure_smem_attr<stream_attn_kernel<D>>(int(smem));
    if (e != cudaSuccess) return e;
    const int units = (p.q_tiles + 3) / 4;
    const unsigned grid = unsigned(2 * units * p.Hkv * p.splits);
    return launch_overlapped(stream_attn_kernel<D>, dim3(grid), dim3(kThreads), smem, stream, p, tq, tkh, tkl, tv16);
}

}  // namespace

size_t stream_attn_smem_bytes(int d) {
    const size_t need = size_t(d == 128 ? Layout<128>::kSmemBytes : Layout<64>::kSmemBytes);
    // At least half the SM's shared memory, so two CTAs never compete for TMEM.
    return need < 120 * 1024 ? 120 * 1024 : need;
}

cudaError_t launch_stream_attn(const AttnParams& p, const CUtensorMap& tq, const CUtensorMap& tkh,
                               const CUtensorMap& tkl, const CUtensorMap& tv16, cudaStream_t stream) {
    return p.d == 128 ? launch_d<128>(p, tq, tkh, tkl, tv16, stream) : launch_d<64>(p, tq, tkh, tkl, tv16, stream);
}

cudaError_t launch_attn_combine(const AttnParams& p, cudaStream_t stream) {
    const int rows = p.Hkv * p.q_tiles * kTileRows;
    const unsigned grid = unsigned((rows * 32 + 127) / 128);
    if (p.d == 128) attn_combine_kernel<128><<<grid, 128, 0, stream>>>(p);
    else attn_combine_kernel<64><<<grid, 128, 0, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_positions(const WindowShape& w, const RingState* state, int rows, int* pos_out,
                             cudaStream_t stream) {
    if (rows <= 0) return cudaSuccess;
    positions_kernel<<<(rows + 255) / 256, 256, 0, stream>>>(w, state, rows, pos_out);
    return cudaGetLastError();
}

cudaError_t launch_wait_probe(unsigned* err, unsigned long long limit_ns, cudaStream_t stream) {
    wait_probe_kernel<<<1, 32, 0, stream>>>(err, limit_ns);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Split-KV scratch that needs no allocation (used by fs_stream_attend_ext_static).
//
// The split-KV path of stream_attn writes one partial (O, m, l) per query tile
// and key split, then attn_combine merges them. fs_stream_attend_ext takes
// that scratch from its handle (allocated at create and sized for the largest
// call). This array serves callers that may not allocate device memory on a
// per-call path: a drafting / verification loop with a device-memory budget
// fixed at start-up, where a cudaMalloc or cudaFree (which can synchronise the
// device and take unbounded time) would break the per-step latency budget.
//
// The array is file-scope device memory of fixed size (kStaticPartTiles
// partial tiles of 128 rows: 64 x 128 x 128 x 4 B = 4 MiB of O plus 64 KiB of
// (m, l) pairs). It is shared by every call on a device and keeps the last
// call's contents; nothing in it has to start at zero, because every partial
// row that attn_combine reads is written by the same call's stream_attn launch
// first (including the (m = -inf, l = 0) rows of key splits with no visible
// tile). Calls that overlap on the GPU (two streams, two handles) race on it.
constexpr int kStaticPartTiles = 64;
constexpr size_t kStaticPartOBytes = size_t(kStaticPartTiles) * kTileRows * 128 * sizeof(float);
constexpr size_t kStaticPartMLBytes = size_t(kStaticPartTiles) * kTileRows * sizeof(float2);
static __device__ __align__(256) unsigned char g_split_scratch[kStaticPartOBytes + kStaticPartMLBytes];

int static_split_scratch_tiles() { return kStaticPartTiles; }

cudaError_t static_split_scratch(float** part_o, float2** part_ml) {
    // One symbol lookup per device, done by the first call on that device with
    // the device current; later calls reuse the address.
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static void* addr[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_split_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = ptr;
    }
    unsigned char* base = static_cast<unsigned char*>(addr[dev]);
    *part_o = reinterpret_cast<float*>(base);
    *part_ml = reinterpret_cast<float2*>(base + kStaticPartOBytes);
    return cudaSuccess;
}

}  // namespace fs
