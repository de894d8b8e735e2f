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
// key tile.
//
// Outputs, per kv head and key row (plain row-major [Hkv][rows_cap][d] arrays,
// like the bf16 cache; the attention kernel's tensor maps swizzle on load):
// the rotated key as fp16 hi + fp16 lo (lo = the rounding residual of hi, so
// hi + lo carries ~22 bits), and V converted to fp16. The rotation runs in fp32
// from the bf16 inputs and the cos/sin table (evaluated in double at create).
// Rows from the last key up to the end of its 128-row tile get zero keys (the
// attention kernel masks them by position) and converted V.
//
// Work is a streaming pass: read 2 x 2d bytes, write 3 x 2d bytes per (key row,
// kv head), plus the row's cos/sin (4d bytes, shared by all kv heads, from L2);
// bound by HBM bandwidth. One thread takes one pair of 16-byte chunks (c, c +
// d/16) of a row -- the rotate-half partners -- so a warp reads and writes
// whole rows, contiguous and coalesced, and enough warps are resident to keep
// the loads in flight.
#include "fs_internal.cuh"
#include "sm100.cuh"

namespace fs {
namespace {

constexpr int kRopeThreads = 256;

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

template <int D>
__global__ void __launch_bounds__(kRopeThreads) kv_stream_rope_kernel(const RopeParams p, int rows_do) {
    constexpr int kPairs = D / 16;  // threads per row
    const unsigned gid = blockIdx.x * kRopeThreads + threadIdx.x;
    const unsigned rr = gid / kPairs;
    if (rr >= unsigned(rows_do) * unsigned(p.Hkv)) return;
    const int c = int(gid % kPairs);
    const int h = int(rr / unsigned(rows_do));
    const int row = int(rr % unsigned(rows_do));
    const size_t base = ((size_t)h * p.rows_cap + row) * D;
    const size_t oa = base + 8 * c, ob = base + D / 2 + 8 * c;  // element offsets of the two chunks

    const uint4 va = *reinterpret_cast<const uint4*>(p.V + oa);
    const uint4 vb = *reinterpret_cast<const uint4*>(p.V + ob);
    uint4 ah = make_uint4(0, 0, 0, 0), al = ah, bh = ah, bl = ah;
    if (row < p.key_rows) {
        const uint4 ka = *reinterpret_cast<const uint4*>(p.K + oa);
        const uint4 kb = *reinterpret_cast<const uint4*>(p.K + ob);
        // Rotate-half: element i pairs with i + D/2, angle pos * theta_i.
        const float4* t4 = reinterpret_cast<const float4*>(p.rope + (size_t)key_pos(p.w, row) * (D / 2) + 8 * c);
        const float4 t[4] = {__ldg(t4), __ldg(t4 + 1), __ldg(t4 + 2), __ldg(t4 + 3)};
        const uint32_t aw[4] = {ka.x, ka.y, ka.z, ka.w};
        const uint32_t bw[4] = {kb.x, kb.y, kb.z, kb.w};
        uint32_t rah[4], ral[4], rbh[4], rbl[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float x0 = bf16lo(aw[q]), x1 = bf16hi(aw[q]);
            const float y0 = bf16lo(bw[q]), y1 = bf16hi(bw[q]);
            const float4 tq = t[q];  // (cos, sin) of elements 8c + 2q and 8c + 2q + 1
            split_pair(x0 * tq.x - y0 * tq.y, x1 * tq.z - y1 * tq.w, rah[q], ral[q]);
            split_pair(y0 * tq.x + x0 * tq.y, y1 * tq.z + x1 * tq.w, rbh[q], rbl[q]);
        }
        ah = make_uint4(rah[0], rah[1], rah[2], rah[3]);
        al = make_uint4(ral[0], ral[1], ral[2], ral[3]);
        bh = make_uint4(rbh[0], rbh[1], rbh[2], rbh[3]);
        bl = make_uint4(rbl[0], rbl[1], rbl[2], rbl[3]);
    }
    *reinterpret_cast<uint4*>(p.Kh + oa) = ah;
    *reinterpret_cast<uint4*>(p.Kh + ob) = bh;
    *reinterpret_cast<uint4*>(p.Kl + oa) = al;
    *reinterpret_cast<uint4*>(p.Kl + ob) = bl;
    *reinterpret_cast<uint4*>(p.V16 + oa) = bf16x8_to_f16x8(va);
    *reinterpret_cast<uint4*>(p.V16 + ob) = bf16x8_to_f16x8(vb);
}

template <int D>
cudaError_t launch_rope_d(const RopeParams& p, cudaStream_t stream) {
    // Through the end of the last key's 128-row tile (the attention kernel reads
    // whole tiles), within the allocation.
    int rows_do = (p.key_rows + kTileRows - 1) / kTileRows * kTileRows;
    if (rows_do > p.rows_cap) rows_do = p.rows_cap;
    const long long threads = (long long)rows_do * p.Hkv * (D / 16);
    const unsigned blocks = unsigned((threads + kRopeThreads - 1) / kRopeThreads);
    kv_stream_rope_kernel<D><<<blocks, kRopeThreads, 0, stream>>>(p, rows_do);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_kv_stream_rope(const RopeParams& p, cudaStream_t stream) {
    if (p.key_rows <= 0) return cudaSuccess;
    return p.d == 128 ? launch_rope_d<128>(p, stream) : launch_rope_d<64>(p, stream);
}

}  // namespace fs
