// kv_stream_rope -- once per window step, rotates every cached pre-RoPE key at
// the position it holds in the current (shifted) window and prepares the MMA
// operands of the attention kernel.
//
// FlashDrive technical summary (gist.science), Methodology 1, "Positional
// Encoding": keys are stored pre-RoPE because absolute positions go stale as
// the window shifts; rotary embeddings are applied on the fly at the shifted
// positions. Every ring row's position moves by one frame each step, so each
// step rotates all of them; doing it here, once per key, instead of inside
// stream_attn, avoids repeating the rotation for every query tile that reads a
// key tile (up to ~50 times per step at the 7-camera window).
//
// One CTA = one (128-row key tile, kv head). TMA stages the bf16 K and V tiles
// in shared memory (128-byte swizzle); the rotation runs there in fp32 with the
// cos/sin table (evaluated in double at create); the rotated key is split into
// fp16 hi + fp16 lo (lo = the rounding residual of hi), V is converted to fp16
// in place, and TMA stores the three fp16 tiles into the handle's operand
// cache in the same swizzled tile format stream_attn loads.
// Work is a streaming copy with arithmetic: read 2 x 256 B, write 3 x 256 B per
// (key row, kv head) at d = 128; bound by HBM bandwidth.
#include <climits>

#include "fs_internal.cuh"
#include "sm100.cuh"

namespace fs {
namespace {

constexpr int kRopeThreads = 128;
constexpr int kRegionBytes = 16384;  // 128 rows x 128 bytes

template <int D>
struct RopeSmem {
    static constexpr int kTile = kTileRows * D * 2;
    static constexpr int kK = 0;          // bf16 K, rotated in place to fp16 hi
    static constexpr int kKlo = kTile;    // fp16 lo
    static constexpr int kV = 2 * kTile;  // bf16 V, converted in place to fp16
    static constexpr int kBar = 3 * kTile;
    static constexpr int kBytes = kBar + 16;
};

// fp32 pair -> fp16 hi pair + fp16 lo pair.
__device__ __forceinline__ void split_pair(float a, float b, uint32_t& hi, uint32_t& lo) {
    hi = pack_f16x2(a, b);
    const float2 hf = __half22float2(*reinterpret_cast<const __half2*>(&hi));
    lo = pack_f16x2(a - hf.x, b - hf.y);
}

template <int D>
__global__ void __launch_bounds__(kRopeThreads) kv_stream_rope_kernel(
    const RopeParams p, const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
    const __grid_constant__ CUtensorMap tkh, const __grid_constant__ CUtensorMap tkl,
    const __grid_constant__ CUtensorMap tv16) {
    using S = RopeSmem<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tile = blockIdx.x;
    const int h = blockIdx.y;
    const int r = threadIdx.x;
    const uint32_t bar = smem_u32(smem + S::kBar);
    if (r == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(bar, 2 * S::kTile);
#pragma unroll
        for (int q = 0; q < D / 64; ++q) {
            tma_load_3d(smem_u32(smem + S::kK + q * kRegionBytes), &tk, q * 64, tile * kTileRows, h, bar);
            tma_load_3d(smem_u32(smem + S::kV + q * kRegionBytes), &tv, q * 64, tile * kTileRows, h, bar);
        }
    }
    __syncthreads();
    const BoundedWait wait{p.err, p.wait_limit_ns, kErrTimeout};
    const bool ok = wait(bar, 0);
    if (ok) {
        const int row = tile * kTileRows + r;
        const int sw = r & 7;
        uint8_t* krow = smem + S::kK + r * 128;
        uint8_t* lrow = smem + S::kKlo + r * 128;
        if (row < p.key_rows) {
            // Rotate-half: pair (i, i + D/2) by the angle pos * theta_i.
            const float2* cs = p.rope + (size_t)key_pos(p.w, row) * (D / 2);
#pragma unroll
            for (int c = 0; c < D / 16; ++c) {
                const int oa = ((c ^ sw) << 4);
                const int ob = D == 128 ? oa + kRegionBytes : (((c + 4) ^ sw) << 4);
                const uint4 a = *reinterpret_cast<const uint4*>(krow + oa);
                const uint4 b = *reinterpret_cast<const uint4*>(krow + ob);
                const float4* t4 = reinterpret_cast<const float4*>(cs + 8 * c);
                const float4 t0 = __ldg(t4), t1 = __ldg(t4 + 1), t2 = __ldg(t4 + 2), t3 = __ldg(t4 + 3);
                const float co[8] = {t0.x, t0.z, t1.x, t1.z, t2.x, t2.z, t3.x, t3.z};
                const float si[8] = {t0.y, t0.w, t1.y, t1.w, t2.y, t2.w, t3.y, t3.w};
                const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
                const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
                uint32_t ah[4], al[4], bh[4], bl[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float x0 = bf16lo(aw[q]), x1 = bf16hi(aw[q]);
                    const float y0 = bf16lo(bw[q]), y1 = bf16hi(bw[q]);
                    const float c0 = co[2 * q], s0 = si[2 * q], c1 = co[2 * q + 1], s1 = si[2 * q + 1];
                    split_pair(x0 * c0 - y0 * s0, x1 * c1 - y1 * s1, ah[q], al[q]);
                    split_pair(y0 * c0 + x0 * s0, y1 * c1 + x1 * s1, bh[q], bl[q]);
                }
                *reinterpret_cast<uint4*>(krow + oa) = make_uint4(ah[0], ah[1], ah[2], ah[3]);
                *reinterpret_cast<uint4*>(krow + ob) = make_uint4(bh[0], bh[1], bh[2], bh[3]);
                *reinterpret_cast<uint4*>(lrow + oa) = make_uint4(al[0], al[1], al[2], al[3]);
                *reinterpret_cast<uint4*>(lrow + ob) = make_uint4(bl[0], bl[1], bl[2], bl[3]);
            }
        } else {
            // Past the last key (masked by position in stream_attn): zeros.
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
                const int o = (c >> 3) * kRegionBytes + ((c & 7) << 4);
                *reinterpret_cast<uint4*>(krow + o) = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4*>(lrow + o) = make_uint4(0, 0, 0, 0);
            }
        }
        // V: bf16 -> fp16 in place (P is fp16, and both MMA operands share one type).
        uint8_t* vrow = smem + S::kV + r * 128;
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
            uint4* q = reinterpret_cast<uint4*>(vrow + (c >> 3) * kRegionBytes + (((c & 7) ^ sw) << 4));
            const uint4 v = *q;
            *q = make_uint4(pack_f16x2(bf16lo(v.x), bf16hi(v.x)), pack_f16x2(bf16lo(v.y), bf16hi(v.y)),
                            pack_f16x2(bf16lo(v.z), bf16hi(v.z)), pack_f16x2(bf16lo(v.w), bf16hi(v.w)));
        }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (r == 0 && ok) {
#pragma unroll
        for (int q = 0; q < D / 64; ++q) {
            tma_store_3d(&tkh, smem_u32(smem + S::kK + q * kRegionBytes), q * 64, tile * kTileRows, h);
            tma_store_3d(&tkl, smem_u32(smem + S::kKlo + q * kRegionBytes), q * 64, tile * kTileRows, h);
            tma_store_3d(&tv16, smem_u32(smem + S::kV + q * kRegionBytes), q * 64, tile * kTileRows, h);
        }
        tma_store_commit();
        tma_store_wait_read();
    }
}

template <int D>
cudaError_t launch_rope_d(const RopeParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                          const CUtensorMap& tkh, const CUtensorMap& tkl, const CUtensorMap& tv16,
                          cudaStream_t stream) {
    const size_t smem = RopeSmem<D>::kBytes + 1024;
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(kv_stream_rope_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             int(smem));
        if (e != cudaSuccess) return e;
        attr = true;
    }
    const dim3 grid(unsigned((p.key_rows + kTileRows - 1) / kTileRows), unsigned(p.Hkv));
    kv_stream_rope_kernel<D><<<grid, kRopeThreads, smem, stream>>>(p, tk, tv, tkh, tkl, tv16);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_kv_stream_rope(const RopeParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                                  const CUtensorMap& tkh, const CUtensorMap& tkl, const CUtensorMap& tv16,
                                  cudaStream_t stream) {
    if (p.key_rows <= 0) return cudaSuccess;
    return p.d == 128 ? launch_rope_d<128>(p, tk, tv, tkh, tkl, tv16, stream)
                      : launch_rope_d<64>(p, tk, tv, tkh, tkl, tv16, stream);
}

}  // namespace fs
