// stream_attn -- attention of a window's new tokens against the streaming KV
// cache, on B200 tensor cores (tcgen05, accumulators in TMEM, TMA-staged tiles).
//
// Method (FlashDrive, arXiv 2608.12932; technical summary on gist.science,
// Methodology 1): keys are cached pre-RoPE in a view-major layout and rotated
// on the fly at the position they hold in the current (shifted) window; the
// new-frame and text queries attend under the streaming mask "query p sees key
// q iff pos(q) <= pos(p)".
//
// One CTA = one (kv head, 128-row query tile[, key split]). A query tile packs
// 128/G tokens x the G query heads that share the kv head, so every key tile
// is loaded once for all G heads (GQA). The keys were rotated once for this
// step by kv_stream_rope (RoPE in shared memory at their shifted positions,
// written as fp16 hi + lo, V as fp16); this kernel rotates its query rows.
// Warp roles, 12 warps:
//   warp 0      TMA producer: K hi + K lo tile and V tile, two stages each;
//   warp 1      TMEM allocator and tcgen05.mma issuer (one thread);
//   warps 4-7   softmax: one query row per thread; S read from TMEM, streaming
//               mask, online softmax in fp32 with exp2, P written back into
//               TMEM over S, lazy rescale of O in TMEM, epilogue;
//   warps 8-11  RoPE of the query rows at their window positions, written into
//               TMEM as the A operand (fp16 hi + lo), once per CTA.
// Pipeline per key tile j (S double-buffered in TMEM):
//   TMA K_j, V_j -> MMA S_j = Q K_j^T -> softmax(S_j) -> P_j -> MMA O += P_j V_j;
//   QK_{j+1} is issued before PV_j, so the tensor core works on the next tile
//   while the softmax warps run.
// Key tiles are walked in physical ring order; positions come from key_pos(),
// so the ring never moves. Tiles whose every key is after the tile's last
// query are skipped; tiles that are entirely visible skip the elementwise mask.
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
// Shared-memory tiles use the 128-byte swizzle that TMA writes and tcgen05
// reads: rows of 128 bytes, 16-byte chunk c of row r at chunk position
// c ^ (r & 7); head dims 64..127 live in a second 16 KB region.
#include <cfloat>
#include <climits>

#include "fs_internal.cuh"
#include "sm100.cuh"

namespace fs {
namespace {

constexpr int kThreads = 384;
constexpr int kRegion = 16384;           // 128 rows x 128 bytes
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;          // O: 256 .. 256+D
constexpr uint32_t kColQ = 384;          // Q hi: 384 .. 384+D/2, Q lo: 384+D/2 .. 384+D
constexpr float kRescaleLog2 = 8.0f;     // rescale O only when the max grows by > 2^8

__device__ __forceinline__ constexpr uint32_t col_s(int s) { return s ? 128u : 0u; }

enum : int {
    kBarQReady = 0, kBarKFull0, kBarKFull1, kBarKEmpty0, kBarKEmpty1, kBarVFull0, kBarVFull1,
    kBarVEmpty0, kBarVEmpty1, kBarSFull0, kBarSFull1, kBarPFull0, kBarPFull1, kBarSFree0, kBarSFree1,
    kBarOFull, kBarMmaDone, kNumBars
};

constexpr uint8_t kSkip = 0, kFull = 1, kPartial = 2;

struct Ctrl {
    alignas(16) int kpos[2][kTileRows];
    uint64_t bars[kNumBars];
    uint32_t tmem_base;
    int nvis;
    uint16_t list[kMaxKeyTiles];  // visible tiles: bits 0-12 tile index, bit 15 partial
    uint8_t cls[kMaxKeyTiles];
};

template <int D>
struct Layout {
    static constexpr int kTileBytes = kTileRows * D * 2;   // one [128 x D] 16-bit tile
    static constexpr int kK0 = 0;                          // K stage s: hi tile then lo tile
    static constexpr int kKStage = 2 * kTileBytes;
    static constexpr int kV0 = 2 * kKStage;                // V stage s
    static constexpr int kCtrl = kV0 + 2 * kTileBytes;
    static constexpr int kBytes = kCtrl + int(sizeof(Ctrl));
};

// Lowest and highest window position among physical key rows [r0, r1). Rows of
// one ring slot (or the text) are consecutive positions, so walking slot-sized
// runs is exact.
__device__ __forceinline__ void key_bounds(const WindowShape& w, int r0, int r1, int& lo, int& hi) {
    lo = INT_MAX;
    hi = INT_MIN;
    int r = r0;
    while (r < r1) {
        int end = r1;
        if (r < w.ring_rows) {
            const int slot_end = (r / w.n + 1) * w.n;
            end = slot_end < r1 ? slot_end : r1;
        }
        const int a = key_pos(w, r);
        const int b = a + (end - 1 - r);
        lo = a < lo ? a : lo;
        hi = b > hi ? b : hi;
        r = end;
    }
}

// fp32 -> fp16 hi + fp16 lo (lo = the rounding residual), packed in pairs.
__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
    hi = pack_f16x2(a, b);
    const __half2 h = *reinterpret_cast<const __half2*>(&hi);
    const float2 hf = __half22float2(h);
    lo = pack_f16x2(a - hf.x, b - hf.y);
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}

// Rotates this thread's query row (loaded from global memory, pre-RoPE bf16),
// scales it by q_scale, and writes fp16 hi / lo parts into TMEM (K-major A
// operand: element i of the row at column i/2, two fp16 per column).
template <int D>
__device__ __forceinline__ void rope_query_row(const uint16_t* __restrict__ qrow, const float2* __restrict__ cs,
                                               float scale, uint32_t t_hi, uint32_t t_lo) {
    constexpr int kHalf = D / 2;
    constexpr int kM = kHalf / 16;  // 16-element blocks per half
#pragma unroll
    for (int m0 = 0; m0 < kM; m0 += 2) {
        // Issue every load of two blocks before any arithmetic: one round trip per pair.
        uint4 qa[2][2], qb[2][2];
        float4 tt[2][8];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int m = m0 + u;
            if (m < kM) {
                const uint4* pa = reinterpret_cast<const uint4*>(qrow + 16 * m);
                const uint4* pb = reinterpret_cast<const uint4*>(qrow + kHalf + 16 * m);
                qa[u][0] = __ldg(pa);
                qa[u][1] = __ldg(pa + 1);
                qb[u][0] = __ldg(pb);
                qb[u][1] = __ldg(pb + 1);
                const float4* t4 = reinterpret_cast<const float4*>(cs + 16 * m);
#pragma unroll
                for (int q = 0; q < 8; ++q) tt[u][q] = __ldg(t4 + q);
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int m = m0 + u;
            if (m >= kM) break;
            const uint32_t aw[8] = {qa[u][0].x, qa[u][0].y, qa[u][0].z, qa[u][0].w,
                                    qa[u][1].x, qa[u][1].y, qa[u][1].z, qa[u][1].w};
            const uint32_t bw[8] = {qb[u][0].x, qb[u][0].y, qb[u][0].z, qb[u][0].w,
                                    qb[u][1].x, qb[u][1].y, qb[u][1].z, qb[u][1].w};
            uint32_t ah[8], al[8], bh[8], bl[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 t = tt[u][q];  // (cos, sin) of elements 16m + 2q, 16m + 2q + 1
                const float x0 = bf16lo(aw[q]), x1 = bf16hi(aw[q]);
                const float y0 = bf16lo(bw[q]), y1 = bf16hi(bw[q]);
                split2((x0 * t.x - y0 * t.y) * scale, (x1 * t.z - y1 * t.w) * scale, ah[q], al[q]);
                split2((y0 * t.x + x0 * t.y) * scale, (y1 * t.z + x1 * t.w) * scale, bh[q], bl[q]);
            }
            tmem_st8(t_hi + 8 * m, ah);
            tmem_st8(t_hi + kHalf / 2 + 8 * m, bh);
            tmem_st8(t_lo + 8 * m, al);
            tmem_st8(t_lo + kHalf / 2 + 8 * m, bl);
        }
    }
}

__device__ __forceinline__ bool vote_all_ok_wg(bool ok) {
    // Uniform decision over the 128 softmax threads (named barrier 1).
    uint32_t res;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.red.and.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(res)
        : "r"(uint32_t(ok))
        : "memory");
    return res != 0;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    stream_attn_kernel(const __grid_constant__ AttnParams p, const uint16_t* __restrict__ Q,
                       const __grid_constant__ CUtensorMap tkh, const __grid_constant__ CUtensorMap tkl,
                       const __grid_constant__ CUtensorMap tv16) {
    using L = Layout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ctrl& ctrl = *reinterpret_cast<Ctrl*>(smem + L::kCtrl);
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    // ---- work item: heavy query tiles (later tokens see more keys) first
    const int split = blockIdx.x % p.splits;
    const int item = blockIdx.x / p.splits;
    const int qt = p.q_tiles - 1 - item / p.Hkv;
    const int kvh = item % p.Hkv;
    const int item_id = qt * p.Hkv + kvh;
    const int tok_per_tile = kTileRows / p.G;
    const int t0 = qt * tok_per_tile;
    const int t_end = min(t0 + tok_per_tile, p.nq);
    const int qmin = query_pos(p.w, p.q_mode, t0);
    const int qmax = query_pos(p.w, p.q_mode, t_end - 1);
    const BoundedWait wait{p.err, p.wait_limit_ns, kErrTimeout};

    auto bar = [&](int i) { return smem_u32(&ctrl.bars[i]); };

    if (tid == 0) {
        mbar_init(bar(kBarQReady), 128);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(kBarKFull0 + s), 1);
            mbar_init(bar(kBarKEmpty0 + s), 1);
            mbar_init(bar(kBarVFull0 + s), 1);
            mbar_init(bar(kBarVEmpty0 + s), 1);
            mbar_init(bar(kBarSFull0 + s), 1);
            mbar_init(bar(kBarPFull0 + s), 128);
            mbar_init(bar(kBarSFree0 + s), 1);
        }
        mbar_init(bar(kBarOFull), 1);
        mbar_init(bar(kBarMmaDone), 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&ctrl.tmem_base), kTmemCols);
        tmem_relinquish();
    }

    // ---- classify key tiles against this query tile, then list the visible ones
    const int n_ktiles = (p.key_rows + kTileRows - 1) / kTileRows;
    for (int j = tid; j < n_ktiles; j += kThreads) {
        const int r0 = j * kTileRows;
        const int r1 = min(r0 + kTileRows, p.key_rows);
        int lo, hi;
        key_bounds(p.w, r0, r1, lo, hi);
        uint8_t c = kPartial;
        if (lo > qmax) c = kSkip;
        else if (hi <= qmin && r1 - r0 == kTileRows) c = kFull;
        ctrl.cls[j] = c;
    }
    __syncthreads();
    if (warp == 0) {
        int count = 0;
        for (int base = 0; base < n_ktiles; base += 32) {
            const int j = base + lane;
            const uint8_t c = j < n_ktiles ? ctrl.cls[j] : kSkip;
            const unsigned vis = __ballot_sync(0xffffffffu, c != kSkip);
            if (c != kSkip) {
                const int slot = count + __popc(vis & ((1u << lane) - 1u));
                ctrl.list[slot] = uint16_t(j | (c == kPartial ? 0x8000 : 0));
            }
            count += __popc(vis);
        }
        if (lane == 0) ctrl.nvis = count;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctrl.tmem_base;
    const int nvis = ctrl.nvis;
    const int kbeg = int((long long)split * nvis / p.splits);
    const int kend = int((long long)(split + 1) * nvis / p.splits);
    const int nt = kend - kbeg;
    const uint32_t lane_off = uint32_t(32 * (warp & 3)) << 16;  // TMEM lanes of this warp

    // Register split, one setmaxnreg per warpgroup at the head of its region: the
    // softmax warpgroup holds a 128-column S row per thread.
    // 128 x (80 + 232 + 192) <= 384 x 168, the registers allocated at launch.
    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 80;");
        if (warp == 0) {
            // ============================================= TMA producer
            if (lane == 0 && nt > 0) {
                tma_prefetch_desc(&tkh);
                tma_prefetch_desc(&tkl);
                tma_prefetch_desc(&tv16);
                for (int k = 0; k < nt; ++k) {
                    const int s = k & 1;
                    const uint32_t par = ((k >> 1) & 1) ^ 1;
                    const int j = ctrl.list[kbeg + k] & 0x1FFF;
                    if (!wait(bar(kBarKEmpty0 + s), par)) break;
                    mbar_arrive_expect_tx(bar(kBarKFull0 + s), 2 * L::kTileBytes);
                    const uint32_t kd = smem_u32(smem + L::kK0 + s * L::kKStage);
#pragma unroll
                    for (int r = 0; r < D / 64; ++r) {
                        tma_load_3d(kd + r * kRegion, &tkh, r * 64, j * kTileRows, kvh, bar(kBarKFull0 + s));
                        tma_load_3d(kd + L::kTileBytes + r * kRegion, &tkl, r * 64, j * kTileRows, kvh,
                                    bar(kBarKFull0 + s));
                    }
                    if (!wait(bar(kBarVEmpty0 + s), par)) break;
                    mbar_arrive_expect_tx(bar(kBarVFull0 + s), L::kTileBytes);
                    const uint32_t vd = smem_u32(smem + L::kV0 + s * L::kTileBytes);
#pragma unroll
                    for (int r = 0; r < D / 64; ++r)
                        tma_load_3d(vd + r * kRegion, &tv16, r * 64, j * kTileRows, kvh, bar(kBarVFull0 + s));
                }
            }
        } else if (warp == 1) {
            // ============================================= MMA issuer
            if (lane == 0 && nt > 0) {
                constexpr uint32_t idesc_qk = idesc_f16(128, 128, false, false, false, false);
                constexpr uint32_t idesc_pv = idesc_f16(128, D, false, false, false, true);
                const uint32_t q_hi = tmem + kColQ, q_lo = tmem + kColQ + D / 2;
                bool ok = wait(bar(kBarQReady), 0);
                for (int k = 0; ok && k <= nt; ++k) {
                    if (k < nt) {
                        const int s = k & 1;
                        if (!(ok = wait(bar(kBarKFull0 + s), (k >> 1) & 1))) break;
                        if (k >= 2 && !(ok = wait(bar(kBarSFree0 + s), ((k - 2) >> 1) & 1))) break;
                        tc_fence_after();
                        const uint32_t kh = smem_u32(smem + L::kK0 + s * L::kKStage);
                        const uint32_t kl = kh + L::kTileBytes;
                        const uint32_t d_s = tmem + col_s(s);
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint32_t off = (kk >> 2) * kRegion + (kk & 3) * 32;
                            const uint64_t dh = sw128_desc(kh + off, 16, 1024);
                            const uint64_t dl = sw128_desc(kl + off, 16, 1024);
                            mma_ts(d_s, q_hi + 8 * kk, dh, idesc_qk, kk > 0);
                            mma_ts(d_s, q_hi + 8 * kk, dl, idesc_qk, 1);
                            mma_ts(d_s, q_lo + 8 * kk, dh, idesc_qk, 1);
                        }
                        tc_commit(bar(kBarSFull0 + s));
                        tc_commit(bar(kBarKEmpty0 + s));
                    }
                    if (k >= 1) {
                        const int kp = k - 1;
                        const int s = kp & 1;
                        const uint32_t par = (kp >> 1) & 1;
                        if (!(ok = wait(bar(kBarPFull0 + s), par))) break;
                        if (!(ok = wait(bar(kBarVFull0 + s), par))) break;
                        tc_fence_after();
                        const uint32_t vs = smem_u32(smem + L::kV0 + s * L::kTileBytes);
#pragma unroll
                        for (int kk = 0; kk < kTileRows / 16; ++kk)
                            mma_ts(tmem + kColO, tmem + col_s(s) + kk * 8, sw128_desc(vs + kk * 2048, kRegion, 1024),
                                   idesc_pv, (kp > 0 || kk > 0));
                        tc_commit(bar(kBarVEmpty0 + s));
                        tc_commit(bar(kBarSFree0 + s));
                        tc_commit(bar(kBarOFull));
                    }
                }
                // Drain: every MMA issued above completes before TMEM is released.
                tc_commit(bar(kBarMmaDone));
                wait(bar(kBarMmaDone), 0);
            }
        }
    } else if (warp < 8) {
        // ================================================= softmax
        asm volatile("setmaxnreg.inc.sync.aligned.u32 232;");
        const int r = tid - 128;
        const int t = t0 + r / p.G;
        const int g = r % p.G;
        const bool valid = t < t_end;
        const int qp = valid ? query_pos(p.w, p.q_mode, t) : -1;
        float m_run = -INFINITY, l_run = 0.f;
        int npart = 0;
        bool ok = true;
        for (int k = 0; k < nt; ++k) {
            const int s = k & 1;
            // Any failure so far (this wait, or an earlier O wait in any warp) ends
            // the loop for all 128 threads together, so no thread is left waiting
            // at a named barrier.
            const bool w_ok = wait(bar(kBarSFull0 + s), (k >> 1) & 1);
            if (!vote_all_ok_wg(w_ok && ok)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t sr[4][32];
#pragma unroll
            for (int h = 0; h < 4; ++h) tmem_ld32(tmem + col_s(s) + lane_off + 32 * h, sr[h]);
            tmem_wait_ld();
            const uint16_t ent = ctrl.list[kbeg + k];
            if (ent & 0x8000) {
                // Elementwise streaming mask: key position of every column of the tile.
                const int j = ent & 0x1FFF;
                const int row = j * kTileRows + r;
                int* kp = ctrl.kpos[npart & 1];
                kp[r] = row < p.key_rows ? key_pos(p.w, row) : INT_MAX;
                named_bar_sync(1, 128);
#pragma unroll
                for (int c4 = 0; c4 < 32; ++c4) {
                    const int4 k4 = *reinterpret_cast<const int4*>(kp + 4 * c4);
                    const uint32_t ninf = __float_as_uint(-INFINITY);
                    uint32_t* q4 = &sr[c4 >> 3][(c4 & 7) * 4];
                    if (k4.x > qp) q4[0] = ninf;
                    if (k4.y > qp) q4[1] = ninf;
                    if (k4.z > qp) q4[2] = ninf;
                    if (k4.w > qp) q4[3] = ninf;
                }
                ++npart;
            }
            float mt = -INFINITY;
#pragma unroll
            for (int c = 0; c < 128; ++c) mt = fmaxf(mt, __uint_as_float(sr[c >> 5][c & 31]));
            const float m_new = fmaxf(m_run, mt);
            const bool resc = m_new > m_run + kRescaleLog2;
            const float m_use = resc ? m_new : m_run;
            const float alpha = resc ? ex2_approx(m_run - m_use) : 1.f;
            const float base = (m_use == -INFINITY) ? 0.f : m_use;
            float rs = 0.f;
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                uint32_t pk[16];
#pragma unroll
                for (int c2 = 0; c2 < 16; ++c2) {
                    const float p0 = ex2_approx(__uint_as_float(sr[h][2 * c2]) - base);
                    const float p1 = ex2_approx(__uint_as_float(sr[h][2 * c2 + 1]) - base);
                    rs += p0 + p1;
                    pk[c2] = pack_f16x2(p0, p1);
                }
                asm volatile(
                    "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
                    "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(tmem + col_s(s) + lane_off +
                                                                                         16 * h),
                    "r"(pk[0]), "r"(pk[1]), "r"(pk[2]), "r"(pk[3]), "r"(pk[4]), "r"(pk[5]), "r"(pk[6]), "r"(pk[7]),
                    "r"(pk[8]), "r"(pk[9]), "r"(pk[10]), "r"(pk[11]), "r"(pk[12]), "r"(pk[13]), "r"(pk[14]),
                    "r"(pk[15])
                    : "memory");
            }
            l_run = l_run * alpha + rs;
            if (k > 0 && __any_sync(0xffffffffu, resc)) {
                // O holds PV_0..PV_{k-1}; wait for the last of them, then rescale in TMEM.
                bool o_ok = wait(bar(kBarOFull), (k - 1) & 1);
                o_ok = __all_sync(0xffffffffu, o_ok);
                if (o_ok) {
                    tc_fence_after();
#pragma unroll 1
                    for (int cc = 0; cc < D / 32; ++cc) {
                        uint32_t o[32];
                        tmem_ld32(tmem + kColO + lane_off + 32 * cc, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st32(tmem + kColO + lane_off + 32 * cc, o);
                    }
                } else {
                    ok = false;
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(kBarPFull0 + s));
            m_run = m_use;
        }
        // ---- epilogue: O / l in fp32 (or the unnormalised split partials)
        const size_t part_row = ((size_t)item_id * p.splits + split) * kTileRows + r;
        if (ok && nt > 0) {
            bool o_ok = wait(bar(kBarMmaDone), 0);  // single phase: after the last PV
            o_ok = __all_sync(0xffffffffu, o_ok);
            if (o_ok) {
                tc_fence_after();
                const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
                const float sc = p.splits == 1 ? inv_l : 1.f;
                float* dst = p.splits == 1 ? p.out + ((size_t)t * p.H + kvh * p.G + g) * D : p.part_o + part_row * D;
                const bool store = p.splits > 1 || valid;
#pragma unroll 1
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t o[32];
                    tmem_ld32(tmem + kColO + lane_off + 32 * cc, o);
                    tmem_wait_ld();
                    if (store) {
                        float4* d4 = reinterpret_cast<float4*>(dst + 32 * cc);
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            d4[q] = make_float4(__uint_as_float(o[4 * q]) * sc, __uint_as_float(o[4 * q + 1]) * sc,
                                                __uint_as_float(o[4 * q + 2]) * sc, __uint_as_float(o[4 * q + 3]) * sc);
                    }
                }
                if (p.splits > 1) p.part_ml[part_row] = make_float2(m_run, l_run);
            }
        } else if (nt == 0 && p.splits > 1) {
            p.part_ml[part_row] = make_float2(-INFINITY, 0.f);
        }
    } else {
        // ================================================= RoPE on Q (rows into TMEM)
        asm volatile("setmaxnreg.inc.sync.aligned.u32 192;");
        const int r = tid - 256;
        if (nt > 0) {
            const int t = t0 + r / p.G;
            const int h = kvh * p.G + r % p.G;
            // Rows past the last token rotate a valid row (token t0) and are never stored.
            const int tt = t < t_end ? t : t0;
            const int qp = query_pos(p.w, p.q_mode, tt);
            rope_query_row<D>(Q + ((size_t)tt * p.H + h) * D, p.rope + (size_t)qp * (D / 2), p.q_scale,
                              tmem + kColQ + lane_off, tmem + kColQ + D / 2 + lane_off);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(kBarQReady));
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
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

__global__ void positions_kernel(const WindowShape w, int rows, int* pos) {
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
cudaError_t launch_d(const AttnParams& p, const uint16_t* Q, const CUtensorMap& tkh, const CUtensorMap& tkl,
                     const CUtensorMap& tv16, cudaStream_t stream) {
    const size_t smem = stream_attn_smem_bytes(D);
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(stream_attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             int(smem));
        if (e != cudaSuccess) return e;
        attr = true;
    }
    const unsigned grid = unsigned(p.Hkv * p.q_tiles * p.splits);
    stream_attn_kernel<D><<<grid, kThreads, smem, stream>>>(p, Q, tkh, tkl, tv16);
    return cudaGetLastError();
}

}  // namespace

size_t stream_attn_smem_bytes(int d) {
    const size_t need = size_t(d == 128 ? Layout<128>::kBytes : Layout<64>::kBytes) + 1024;
    // At least half the SM's shared memory, so two CTAs never compete for TMEM.
    return need < 120 * 1024 ? 120 * 1024 : need;
}

cudaError_t launch_stream_attn(const AttnParams& p, const uint16_t* Q, const CUtensorMap& tkh,
                               const CUtensorMap& tkl, const CUtensorMap& tv16, cudaStream_t stream) {
    return p.d == 128 ? launch_d<128>(p, Q, tkh, tkl, tv16, stream) : launch_d<64>(p, Q, tkh, tkl, tv16, stream);
}

cudaError_t launch_attn_combine(const AttnParams& p, cudaStream_t stream) {
    const int rows = p.Hkv * p.q_tiles * kTileRows;
    const unsigned grid = unsigned((rows * 32 + 127) / 128);
    if (p.d == 128) attn_combine_kernel<128><<<grid, 128, 0, stream>>>(p);
    else attn_combine_kernel<64><<<grid, 128, 0, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_positions(const WindowShape& w, int rows, int* pos_out, cudaStream_t stream) {
    if (rows <= 0) return cudaSuccess;
    positions_kernel<<<(rows + 255) / 256, 256, 0, stream>>>(w, rows, pos_out);
    return cudaGetLastError();
}

cudaError_t launch_wait_probe(unsigned* err, unsigned long long limit_ns, cudaStream_t stream) {
    wait_probe_kernel<<<1, 32, 0, stream>>>(err, limit_ns);
    return cudaGetLastError();
}

}  // namespace fs
