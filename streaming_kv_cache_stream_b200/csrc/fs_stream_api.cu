// fs_stream_api.cu -- host side of the C ABI declared in include/fs_stream.h:
// argument checks, the stream state machine (prefill first, then window
// steps; FlashDrive README, "Library": the first call of a stream only
// prefills), device allocation of the static cache, TMA tensor maps, and
// kernel launches. No compute happens on the host: every step of the path runs
// in the kernels of kv_stream_insert.cu and stream_attn.cu.
// Tensor maps are built once per handle (for the cache); queries are read by
// the kernel with plain loads, so attend encodes nothing per call.
#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include <cudaTypedefs.h>

#include "../../include/fs_stream.h"
#include "fs_internal.cuh"

using fs::AttnParams;
using fs::InsertParams;
using fs::WindowShape;

struct fs_stream {
    int V, T, n, X, H, Hkv, G, d;
    float base;
    int L, ring_rows, step_tokens, rows_cap, rope_rows;
    int rebase_every = 16;  // R: every R-th window step re-rotates the whole window
    int state = FS_STATE_EXPECT_PREFILL;
    int head = 0;           // host mirror of the device ring head (sizes, debug export)
    int tail = 0;           // persisted decode-tail tokens after the text
    int k_host = 0;         // host mirror of the device ring state's step count k
    long long steps = 0;
    std::vector<long long> slot_frame;  // frame id held by each ring slot (same for all views)
    cudaStream_t stream = nullptr;
    int device = 0, num_sms = 148;
    uint16_t* K_cache = nullptr;  // pre-RoPE bf16 ring + text + decode tail + drafted-block rows
    uint16_t* V_cache = nullptr;
    uint16_t* Kh = nullptr;       // attention operands: rotated K fp16 hi / lo, V fp16
    uint16_t* Kl = nullptr;
    uint16_t* V16 = nullptr;
    const float2* rope = nullptr; // shared per (device, d, base, rows); see rope_acquire
    fs::RingState* dstate = nullptr;  // device-resident ring head and angle offset
    unsigned* err = nullptr;
    float* part_o = nullptr;
    float2* part_ml = nullptr;
    int part_rows_cap = 0;  // rows of 128 query rows x d fp32 the split scratch holds
    void* stage = nullptr;  // host-path staging: K, V, Q, out
    size_t stage_bytes = 0;
    cudaStream_t copy_in = nullptr, copy_out = nullptr;         // host-path copy streams
    cudaEvent_t ev_in = nullptr, ev_done = nullptr, ev_out = nullptr;
    CUtensorMap tmap_kh2, tmap_kl2, tmap_v16h;  // fp16 operands, one CTA's half tile (attention loads)
    CUtensorMap tmap_v1;    // fp16 V, {64 columns, 128 rows} boxes (drafted-block verify)
    unsigned long long wait_limit_ns = 2000000000ull;
    long long cache_bytes = 0;
    long long launches = 0;
    std::string last_error;
};

namespace {

thread_local std::string g_last_error;

int fail(fs_stream_t s, int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    if (s) s->last_error = buf;
    return code;
}

#define FS_CUDA(s, call)                                                                       \
    do {                                                                                       \
        cudaError_t e_ = (call);                                                               \
        if (e_ != cudaSuccess)                                                                 \
            return fail((s), FS_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_));     \
    } while (0)

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 3-D 16-bit tensor map, box {b0, b1, b2}, out-of-range reads as zero; 128-byte
// swizzle unless told otherwise.
int make_map(fs_stream_t s, CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
             uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b1, uint32_t b2,
             CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, uint32_t b0 = 64,
             CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
    auto enc = get_encode();
    if (!enc) return fail(s, FS_ERR_CUDA, "cuTensorMapEncodeTiled unavailable from the driver");
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
    cuuint32_t box[3] = {b0, b1, b2};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, dtype, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(s, FS_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
    return FS_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

WindowShape shape_of(const fs_stream* s) {
    WindowShape w;
    w.V = s->V;
    w.T = s->T;
    w.n = s->n;
    w.X = s->X;
    w.ring_rows = s->ring_rows;
    w.head = s->head;
    w.tail = s->tail;
    return w;
}

// ---------------------------------------------------------------- RoPE tables
// cos/sin of (angle index) * base^(-2i/d), evaluated in double, stored as float2
// [rows][d/2]. Handles of the same device, head dim, base and row count share
// one table (a 36-layer stack holds one copy, not 36); reference-counted.
struct RopeEntry {
    int device, d, rows;
    float base;
    float2* ptr;
    int refs;
};
std::mutex g_rope_mu;
std::vector<RopeEntry> g_rope;

const float2* rope_acquire(int device, int d, float base, int rows, cudaError_t* err) {
    std::lock_guard<std::mutex> lock(g_rope_mu);
    for (auto& e : g_rope)
        if (e.device == device && e.d == d && e.rows == rows && e.base == base) {
            ++e.refs;
            return e.ptr;
        }
    const size_t bytes = size_t(rows) * (d / 2) * sizeof(float2);
    std::vector<float2> tab(size_t(rows) * (d / 2));
    for (int i = 0; i < d / 2; ++i) {
        const double theta = std::pow(double(base), -2.0 * i / d);
        for (int a = 0; a < rows; ++a) {
            const double ang = double(a) * theta;
            tab[size_t(a) * (d / 2) + i] = make_float2(float(std::cos(ang)), float(std::sin(ang)));
        }
    }
    float2* ptr = nullptr;
    *err = cudaMalloc(&ptr, bytes);
    if (*err != cudaSuccess) return nullptr;
    *err = cudaMemcpy(ptr, tab.data(), bytes, cudaMemcpyHostToDevice);
    if (*err != cudaSuccess) {
        cudaFree(ptr);
        return nullptr;
    }
    g_rope.push_back(RopeEntry{device, d, rows, base, ptr, 1});
    return ptr;
}

void rope_release(const float2* ptr) {
    if (!ptr) return;
    std::lock_guard<std::mutex> lock(g_rope_mu);
    for (size_t i = 0; i < g_rope.size(); ++i)
        if (g_rope[i].ptr == ptr) {
            if (--g_rope[i].refs == 0) {
                cudaFree(g_rope[i].ptr);
                g_rope.erase(g_rope.begin() + long(i));
            }
            return;
        }
}

void free_all(fs_stream* s) {
    cudaFree(s->K_cache);
    cudaFree(s->V_cache);
    cudaFree(s->Kh);
    cudaFree(s->Kl);
    cudaFree(s->V16);
    rope_release(s->rope);
    cudaFree(s->dstate);
    cudaFree(s->err);
    cudaFree(s->part_o);
    cudaFree(s->part_ml);
    cudaFree(s->stage);
    if (s->copy_in) cudaStreamDestroy(s->copy_in);
    if (s->copy_out) cudaStreamDestroy(s->copy_out);
    if (s->ev_in) cudaEventDestroy(s->ev_in);
    if (s->ev_done) cudaEventDestroy(s->ev_done);
    if (s->ev_out) cudaEventDestroy(s->ev_out);
}

int check_err_word(fs_stream_t s) {
    unsigned h = 0;
    FS_CUDA(s, cudaMemcpy(&h, s->err, sizeof h, cudaMemcpyDeviceToHost));
    if (h) {
        FS_CUDA(s, cudaMemset(s->err, 0, sizeof(unsigned)));
        if (h & fs::kErrTimeout) return fail(s, FS_ERR_DEVICE_TIMEOUT, "a bounded device-side wait gave up");
        if (h & fs::kErrRange)
            return fail(s, FS_ERR_RANGE,
                        "an input was out of range: a rotated key, V or scaled rotated query element above 65504 in "
                        "magnitude, or not finite; outputs since the last check are not valid");
        return fail(s, FS_ERR_CUDA, "device error word 0x%x", h);
    }
    return FS_OK;
}

fs::InsertLayer layer_of(const fs_stream* s, const void* K, const void* V) {
    fs::InsertLayer ly;
    ly.K_src = static_cast<const uint16_t*>(K);
    ly.V_src = static_cast<const uint16_t*>(V);
    ly.K = s->K_cache;
    ly.V = s->V_cache;
    ly.Kh = s->Kh;
    ly.Kl = s->Kl;
    ly.V16 = s->V16;
    ly.state = s->dstate;
    ly.err = s->err;
    return ly;
}

InsertParams insert_params(const fs_stream* s, int mode, int n_tokens, int row0) {
    InsertParams p;
    std::memset(&p, 0, sizeof p);
    p.w = shape_of(s);
    p.mode = mode;
    p.N = n_tokens;
    p.row0 = row0;
    p.Hkv = s->Hkv;
    p.d = s->d;
    p.rows_cap = s->rows_cap;
    p.rebase_every = s->rebase_every;
    p.rope = s->rope;
    p.layers = 0;
    return p;
}

// One pass of kernel kv_stream_insert for one layer: mode 0 = the whole window
// (prefill), 1 = a window step (each view's new frame and the text; the device
// ring state decides whether it is a re-base step that re-rotates the whole
// window), 2 = n_tokens rows from row0 on (decode tail or drafted block).
int do_insert(fs_stream_t s, const void* K, const void* V, int n_tokens, int mode, int row0) {
    InsertParams p = insert_params(s, mode, n_tokens, row0);
    p.layer[0] = layer_of(s, K, V);
    p.layers = 1;
    FS_CUDA(s, fs::launch_kv_stream_insert(p, s->stream));
    s->launches += 1;
    return FS_OK;
}

// Host bookkeeping after a window insert (the device state was advanced by the kernel).
void after_window_insert(fs_stream_t s, bool prefill) {
    s->tail = 0;
    if (prefill) {
        s->head = 0;
        s->k_host = 0;
        s->steps = 0;
        for (int f = 0; f < s->T; ++f) s->slot_frame[f] = f;
        s->state = FS_STATE_PREFILLED;
        return;
    }
    s->slot_frame[s->head] = (long long)s->T + s->steps;  // the k-th step inserts frame T-1+k
    s->head = (s->head + 1) % s->T;
    s->k_host = s->k_host + 1 >= s->rebase_every ? 0 : s->k_host + 1;
    s->steps += 1;
    s->state = FS_STATE_STREAMING;
}

// Splits of the key range per (kv head, unit of four query tiles) so that
// small query sets still fill the SMs (a unit occupies a pair of SMs); capped
// by the scratch (one partial per query tile and split) and by the number of
// key tiles.
int choose_splits(const fs_stream* s, int q_tiles, int key_rows) {
    const int units = ((q_tiles + 3) / 4) * s->Hkv;
    const int slots = s->num_sms / 2;
    if (units >= slots) return 1;
    const int ktiles = (key_rows + fs::kTileRows - 1) / fs::kTileRows;
    int sp = (slots + units - 1) / units;
    if (sp > ktiles / 2) sp = ktiles / 2;
    const int tiles = q_tiles * s->Hkv;
    if (sp > s->part_rows_cap / tiles) sp = s->part_rows_cap / tiles;
    return sp < 1 ? 1 : sp;
}

AttnParams attn_params(const fs_stream* s, int nq, int mode, int key_rows, void* out) {
    AttnParams p;
    std::memset(&p, 0, sizeof p);
    p.w = shape_of(s);
    p.key_rows = key_rows;
    p.Hkv = s->Hkv;
    p.G = s->G;
    p.H = s->H;
    p.d = s->d;
    p.nq = nq;
    p.q_mode = mode;
    p.q_tiles = (nq * s->G + fs::kTileRows - 1) / fs::kTileRows;
    p.splits = 1;
    p.q_scale = float(1.4426950408889634 / std::sqrt(double(s->d)));
    p.rope = s->rope;
    p.rope_rows = s->rope_rows;
    p.state = s->dstate;
    p.out = static_cast<float*>(out);
    p.part_o = s->part_o;
    p.part_ml = s->part_ml;
    p.err = s->err;
    p.wait_limit_ns = s->wait_limit_ns;
    return p;
}

int make_query_map(fs_stream_t s, CUtensorMap* tq, const void* Q, int nq) {
    // One query tile (128/G tokens x G heads) per box.
    return make_map(s, tq, Q, s->d, s->H, nq, uint64_t(s->d) * 2, uint64_t(s->H) * s->d * 2, s->G,
                    fs::kTileRows / s->G);
}

int launch_attention(fs_stream_t s, const AttnParams& p, const CUtensorMap& tq) {
    FS_CUDA(s, fs::launch_stream_attn(p, tq, s->tmap_kh2, s->tmap_kl2, s->tmap_v16h, s->stream));
    s->launches += 1;
    if (p.splits > 1) {
        FS_CUDA(s, fs::launch_attn_combine(p, s->stream));
        s->launches += 1;
    }
    return FS_OK;
}

int do_attend(fs_stream_t s, const void* Q, void* out, int nq, int mode, int key_rows) {
    // Encoded before anything is enqueued, so a failure leaves no partial work.
    CUtensorMap tq;
    const int rcq = make_query_map(s, &tq, Q, nq);
    if (rcq) return rcq;
    AttnParams p = attn_params(s, nq, mode, key_rows, out);
    p.splits = choose_splits(s, p.q_tiles, key_rows);
    return launch_attention(s, p, tq);
}

int check_block_args(fs_stream_t s, const void* Q_x, const void* K_x, const void* V_x, int n_x, const void* out) {
    if (!Q_x || !K_x || !V_x || !out) return fail(s, FS_ERR_ARG, "NULL tensor pointer");
    if (!aligned16(Q_x) || !aligned16(K_x) || !aligned16(V_x) || !aligned16(out))
        return fail(s, FS_ERR_ARG, "pointers must be 16-byte aligned");
    if (n_x < 1 || n_x > FS_MAX_VERIFY_TOKENS) return fail(s, FS_ERR_ARG, "n_x must be in [1, %d]", FS_MAX_VERIFY_TOKENS);
    if (Q_x == out) return fail(s, FS_ERR_ARG, "out must not alias Q_x");
    if (s->state == FS_STATE_EXPECT_PREFILL) return fail(s, FS_ERR_STATE, "verify before the first insert");
    return FS_OK;
}

// A drafted block whose queries fit one 128-row tile per kv head goes through
// verify_attn (one launch: block rotation, split-KV attention, in-kernel
// merge); longer blocks through kv_stream_insert + stream_attn (+ combine).
int verify_small(fs_stream_t s, const void* Q_x, const void* K_x, const void* V_x, int n_x, void* out) {
    fs::VerifyParams p;
    std::memset(&p, 0, sizeof p);
    p.w = shape_of(s);
    p.row_block = s->L + s->tail;
    p.key_rows = p.row_block + n_x;
    p.n_x = n_x;
    p.Hkv = s->Hkv;
    p.G = s->G;
    p.H = s->H;
    p.d = s->d;
    p.rows_cap = s->rows_cap;
    const int nkt = (p.key_rows + fs::kTileRows - 1) / fs::kTileRows;
    p.splits = std::min(fs::kMaxVerifySplits, nkt);
    p.q_scale = float(1.4426950408889634 / std::sqrt(double(s->d)));
    p.rope = s->rope;
    p.state = s->dstate;
    p.Q_x = static_cast<const uint16_t*>(Q_x);
    p.K_x = static_cast<const uint16_t*>(K_x);
    p.V_x = static_cast<const uint16_t*>(V_x);
    p.out = static_cast<float*>(out);
    p.err = s->err;
    p.wait_limit_ns = s->wait_limit_ns;
    FS_CUDA(s, fs::launch_verify_attn(p, s->tmap_kh2, s->tmap_kl2, s->tmap_v1, s->stream));
    s->launches += 1;
    return FS_OK;
}

}  // namespace

extern "C" {

int fs_stream_create(fs_stream_t* out, int views, int frames, int tok_per_frame, int text_len, int H, int Hkv,
                     int d, float rope_base) {
    if (!out) return fail(nullptr, FS_ERR_ARG, "out is NULL");
    *out = nullptr;
    if (views < 1 || frames < 1 || tok_per_frame < 1 || text_len < 0)
        return fail(nullptr, FS_ERR_ARG, "window sizes must be positive (text_len >= 0)");
    if (H < 1 || Hkv < 1 || H % Hkv) return fail(nullptr, FS_ERR_ARG, "need H, Hkv >= 1 and H %% Hkv == 0");
    const int G = H / Hkv;
    if (fs::kTileRows % G) return fail(nullptr, FS_ERR_ARG, "H/Hkv must divide 128 (got %d)", G);
    if (d != 64 && d != 128) return fail(nullptr, FS_ERR_ARG, "head dim must be 64 or 128 (got %d)", d);
    if (!(rope_base > 0.f) || !std::isfinite(rope_base)) return fail(nullptr, FS_ERR_ARG, "rope_base must be > 0");
    const long long ring = (long long)views * frames * tok_per_frame;
    const long long L = ring + text_len;
    const long long extra = fs::kMaxTail + fs::kMaxVerify;
    if (L + extra > (long long)fs::kMaxKeyTiles * fs::kTileRows)
        return fail(nullptr, FS_ERR_ARG, "window too long: L + %lld must be <= %d", extra,
                    fs::kMaxKeyTiles * fs::kTileRows);

    fs_stream* s = new (std::nothrow) fs_stream();
    if (!s) return fail(nullptr, FS_ERR_OOM, "host allocation failed");
    s->V = views;
    s->T = frames;
    s->n = tok_per_frame;
    s->X = text_len;
    s->H = H;
    s->Hkv = Hkv;
    s->G = G;
    s->d = d;
    s->base = rope_base;
    s->ring_rows = int(ring);
    s->L = int(L);
    s->step_tokens = views * tok_per_frame + text_len;
    s->rows_cap = int(L + extra);
    if (const char* e = std::getenv("FS_REBASE_STEPS")) {
        const long v = std::strtol(e, nullptr, 10);
        if (v >= 1 && v <= 4096) s->rebase_every = int(v);
    }
    // Angle indices reach (L + tail + block - 1) + (R - 1) * n.
    const long long rope_rows = (long long)s->rows_cap + (long long)(s->rebase_every - 1) * tok_per_frame;
    if (rope_rows > (1ll << 24)) {
        delete s;
        return fail(nullptr, FS_ERR_ARG, "RoPE table too large: lower FS_REBASE_STEPS");
    }
    s->rope_rows = int(rope_rows);
    s->slot_frame.assign(frames, -1);
    if (const char* e = std::getenv("FS_WAIT_LIMIT_NS")) s->wait_limit_ns = std::strtoull(e, nullptr, 10);

    auto bail = [&](int code) {
        free_all(s);
        delete s;
        return code;
    };
    cudaError_t e = cudaGetDevice(&s->device);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&s->num_sms, cudaDevAttrMultiProcessorCount, s->device);
    if (e != cudaSuccess) return bail(fail(nullptr, FS_ERR_CUDA, "no CUDA device: %s", cudaGetErrorString(e)));
    int major = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, s->device);
    if (major != 10) return bail(fail(nullptr, FS_ERR_CUDA, "needs an sm_100 GPU (B200); found major %d", major));

    const size_t cache = size_t(Hkv) * s->rows_cap * d * 2;
    s->part_rows_cap = 2 * s->num_sms;
    const size_t part_o = size_t(s->part_rows_cap) * fs::kTileRows * d * sizeof(float);
    const size_t part_ml = size_t(s->part_rows_cap) * fs::kTileRows * sizeof(float2);
    if (cudaMalloc(&s->K_cache, cache) != cudaSuccess || cudaMalloc(&s->V_cache, cache) != cudaSuccess ||
        cudaMalloc(&s->Kh, cache) != cudaSuccess || cudaMalloc(&s->Kl, cache) != cudaSuccess ||
        cudaMalloc(&s->V16, cache) != cudaSuccess || cudaMalloc(&s->dstate, sizeof(fs::RingState)) != cudaSuccess ||
        cudaMalloc(&s->err, sizeof(unsigned)) != cudaSuccess || cudaMalloc(&s->part_o, part_o) != cudaSuccess ||
        cudaMalloc(&s->part_ml, part_ml) != cudaSuccess) {
        cudaGetLastError();
        return bail(fail(nullptr, FS_ERR_OOM, "device allocation of %zu bytes failed", 5 * cache + part_o));
    }
    // Every operand row starts finite (zero): rows past a call's last key are
    // masked by position, and 0 x finite stays 0 in P V.
    if (cudaMemset(s->K_cache, 0, cache) != cudaSuccess || cudaMemset(s->V_cache, 0, cache) != cudaSuccess ||
        cudaMemset(s->Kh, 0, cache) != cudaSuccess || cudaMemset(s->Kl, 0, cache) != cudaSuccess ||
        cudaMemset(s->V16, 0, cache) != cudaSuccess || cudaMemset(s->dstate, 0, sizeof(fs::RingState)) != cudaSuccess ||
        cudaMemset(s->err, 0, sizeof(unsigned)) != cudaSuccess)
        return bail(fail(nullptr, FS_ERR_CUDA, "cudaMemset failed"));
    e = cudaSuccess;
    s->rope = rope_acquire(s->device, d, rope_base, s->rope_rows, &e);
    if (!s->rope) {
        cudaGetLastError();
        return bail(fail(nullptr, e == cudaErrorMemoryAllocation ? FS_ERR_OOM : FS_ERR_CUDA,
                         "RoPE table (%d rows) failed: %s", s->rope_rows, cudaGetErrorString(e)));
    }
    const size_t rope = size_t(s->rope_rows) * (d / 2) * sizeof(float2);
    s->cache_bytes = (long long)(5 * cache + part_o + part_ml + sizeof(unsigned) + sizeof(fs::RingState));
    (void)rope;

    const uint64_t row_bytes = uint64_t(d) * 2;
    const CUtensorMapDataType f16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    int rc = FS_OK;
    // Pair loads: 64 key rows of K hi / lo; all 128 key rows of d/2 V columns.
    if (!rc) rc = make_map(nullptr, &s->tmap_kh2, s->Kh, d, s->rows_cap, Hkv, row_bytes, row_bytes * s->rows_cap,
                           fs::kTileRows / 2, 1, f16);
    if (!rc) rc = make_map(nullptr, &s->tmap_kl2, s->Kl, d, s->rows_cap, Hkv, row_bytes, row_bytes * s->rows_cap,
                           fs::kTileRows / 2, 1, f16);
    if (!rc) rc = make_map(nullptr, &s->tmap_v16h, s->V16, d, s->rows_cap, Hkv, row_bytes, row_bytes * s->rows_cap,
                           fs::kTileRows, 1, f16, uint32_t(d / 2),
                           d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
    if (!rc) rc = make_map(nullptr, &s->tmap_v1, s->V16, d, s->rows_cap, Hkv, row_bytes, row_bytes * s->rows_cap,
                           fs::kTileRows, 1, f16, 64u, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return bail(rc);
    *out = s;
    return FS_OK;
}

int fs_stream_destroy(fs_stream_t s) {
    if (!s) return FS_OK;
    cudaStreamSynchronize(s->stream);
    if (s->copy_in) cudaStreamSynchronize(s->copy_in);
    if (s->copy_out) cudaStreamSynchronize(s->copy_out);
    free_all(s);
    delete s;
    return FS_OK;
}

int fs_stream_set_stream(fs_stream_t s, void* cuda_stream) {
    if (!s) return fail(nullptr, FS_ERR_ARG, "NULL handle");
    s->stream = static_cast<cudaStream_t>(cuda_stream);
    return FS_OK;
}

int fs_stream_reset(fs_stream_t s) {
    if (!s) return fail(nullptr, FS_ERR_ARG, "NULL handle");
    s->state = FS_STATE_EXPECT_PREFILL;
    s->head = 0;
    s->tail = 0;
    s->steps = 0;
    s->slot_frame.assign(s->T, -1);
    return FS_OK;
}

int fs_stream_insert(fs_stream_t s, const void* K_new, const void* V_new) {
    if (!s) return fail(nullptr, FS_ERR_ARG, "NULL handle");
    if (!K_new || !V_new) return fail(s, FS_ERR_ARG, "K_new/V_new is NULL");
    if (!aligned16(K_new) || !aligned16(V_new)) return fail(s, FS_ERR_ARG, "K_new/V_new must be 16-byte aligned");
    const bool prefill = s->state == FS_STATE_EXPECT_PREFILL;
    int rc = do_insert(s, K_new, V_new, prefill ? s->L : s->step_tokens, prefill ? 0 : 1, 0);
    if (rc) return rc;
    after_window_insert(s, prefill);
    return FS_OK;
}

int fs_stream_insert_batch(fs_stream_t* handles, int n, const void* const* K_new, const void* const* V_new) {
    if (!handles || !K_new || !V_new || n < 1) return fail(nullptr, FS_ERR_ARG, "NULL array or n < 1");
    fs_stream_t s0 = handles[0];
    if (!s0) return fail(nullptr, FS_ERR_ARG, "NULL handle");
    const bool prefill = s0->state == FS_STATE_EXPECT_PREFILL;
    for (int i = 0; i < n; ++i) {
        fs_stream_t s = handles[i];
        if (!s) return fail(s0, FS_ERR_ARG, "handle %d is NULL", i);
        if (!K_new[i] || !V_new[i] || !aligned16(K_new[i]) || !aligned16(V_new[i]))
            return fail(s0, FS_ERR_ARG, "K_new/V_new of layer %d NULL or not 16-byte aligned", i);
        if (s->V != s0->V || s->T != s0->T || s->n != s0->n || s->X != s0->X || s->Hkv != s0->Hkv ||
            s->d != s0->d || s->rows_cap != s0->rows_cap || s->rebase_every != s0->rebase_every ||
            s->rope != s0->rope || s->device != s0->device)
            return fail(s0, FS_ERR_ARG, "handle %d differs in shape, RoPE table or device from handle 0", i);
        if (s->stream != s0->stream) return fail(s0, FS_ERR_ARG, "handle %d is on another stream", i);
        if ((s->state == FS_STATE_EXPECT_PREFILL) != prefill)
            return fail(s0, FS_ERR_STATE, "handles mix prefill and window-step states (handle %d)", i);
        for (int j = 0; j < i; ++j)
            if (handles[j] == s) return fail(s0, FS_ERR_ARG, "handle %d appears twice", i);
    }
    const int tokens = prefill ? s0->L : s0->step_tokens;
    for (int b = 0; b < n; b += fs::kMaxInsertBatch) {
        const int cnt = n - b < fs::kMaxInsertBatch ? n - b : fs::kMaxInsertBatch;
        InsertParams p = insert_params(s0, prefill ? 0 : 1, tokens, 0);
        for (int i = 0; i < cnt; ++i) p.layer[i] = layer_of(handles[b + i], K_new[b + i], V_new[b + i]);
        p.layers = cnt;
        FS_CUDA(s0, fs::launch_kv_stream_insert(p, s0->stream));
        s0->launches += 1;
    }
    for (int i = 0; i < n; ++i) after_window_insert(handles[i], prefill);
    return FS_OK;
}

int fs_stream_insert_proj(fs_stream_t s, const void* X, const void* W, int d_model) {
    if (!s) return fail(nullptr, FS_ERR_ARG, "NULL handle");
    if (!X || !W) return fail(s, FS_ERR_ARG, "X/W is NULL");
    if (!aligned16(X) || !aligned16(W)) return fail(s, FS_ERR_ARG, "X/W must be 16-byte aligned");
    if (d_model < 8 || d_model % 8) return fail(s, FS_ERR_ARG, "d_model must be a positive multiple of 8 (got %d)", d_model);
    const bool prefill = s->state == FS_STATE_EXPECT_PREFILL;
    const int N = prefill ? s->L : s->step_tokens;
    const uint64_t row = uint64_t(d_model) * 2;
    const int outs = 2 * s->Hkv * s->d;
    CUtensorMap tx, tw;
    int rc = make_map(s, &tx, X, d_model, N, 1, row, row * N, 128, 1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 64);
    if (!rc) rc = make_map(s, &tw, W, d_model, outs, 1, row, row * outs, 256, 1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 64);
    if (rc) return rc;
    fs::ProjParams p;
    std::memset(&p, 0, sizeof p);
    p.w = shape_of(s);
    p.mode = prefill ? 0 : 1;
    p.N = N;
    p.d_model = d_model;
    p.Hkv = s->Hkv;
    p.d = s->d;
    p.rows_cap = s->rows_cap;
    p.rebase_every = s->rebase_every;
    p.rope = s->rope;
    p.K = s->K_cache;
    p.V = s->V_cache;
    p.Kh = s->Kh;
    p.Kl = s->Kl;
    p.V16 = s->V16;
    p.state = s->dstate;
    p.err = s->err;
    p.wait_limit_ns = s->wait_limit_ns;
    FS_CUDA(s, fs::launch_kv_proj(p, tx, tw, s->stream));
    s->launches += 1;
    if (!prefill && s->k_host + 1 >= s->rebase_every) {
        // A re-base step: the projection wrote the new rows' bf16 K/V; the whole
        // window is re-rotated from the cache at k = 0.
        InsertParams q = insert_params(s, 3, 0, 0);
        q.layer[0] = layer_of(s, nullptr, nullptr);
        q.layers = 1;
        FS_CUDA(s, fs::launch_kv_stream_insert(q, s->stream));
        s->launches += 1;
    }
    after_window_insert(s, prefill);
    return FS_OK;
}

int fs_stream_attend(fs_stream_t s, const void* Q, void* out) {
    if (!s) return fail(nullptr, FS_ERR_ARG, "NULL handle");
    if (!Q || !out) return fail(s, FS_ERR_ARG, "Q/out is NULL");
    if (!aligned16(Q) || !aligned16(out)) return fail(s, FS_ERR_ARG, "Q/out must be 16-byte aligned");
    if (Q == out) return fail(s, FS_ERR_ARG, "out must not alias Q");
    if (s->state == FS_STATE_EXPECT_PREFILL) return fail(s, FS_ERR_STATE, "attend before the first insert");
    const bool pre = s->state == FS_STATE_PREFILLED;
    return do_attend(s, Q, out, pre ? s->L : s->step_tokens, pre ? fs::kQueryPrefill : fs::kQueryStep, s->L);
}

int fs_stream_append(fs_stream_t s, const void* K_acc, const void* V_acc, int n_acc) {
    if (!s) return fail(nullptr, FS_ERR_ARG, "NULL handle");
    if (!K_acc || !V_acc) return fail(s, FS_ERR_ARG, "K_acc/V_acc is NULL");
    if (!aligned16(K_acc) || !aligned16(V_acc)) return fail(s, FS_ERR_ARG, "K_acc/V_acc must be 16-byte aligned");
    if (n_acc < 1) return fail(s, FS_ERR_ARG, "n_acc must be >= 1");
    if (s->tail + n_acc > FS_MAX_TAIL_TOKENS)
        return fail(s, FS_ERR_ARG, "decode tail would hold %d tokens; the limit is %d", s->tail + n_acc,
                    FS_MAX_TAIL_TOKENS);
    if (s->state == FS_STATE_EXPECT_PREFILL) return fail(s, FS_ERR_STATE, "append before the first insert");
    int rc = do_insert(s, K_acc, V_acc, n_acc, 2, s->L + s->tail);
    if (rc) return rc;
    s->tail += n_acc;
    return FS_OK;
}

int fs_stream_attend_ext(fs_stream_t s, const void* Q_x, const void* K_x, const void* V_x, int n_x, void* out) {
    if (!s) return fail(nullptr, FS_ERR_ARG, "NULL handle");
    int rc = check_block_args(s, Q_x, K_x, V_x, n_x, out);
    if (rc) return rc;
    if (n_x * s->G <= fs::kTileRows) return verify_small(s, Q_x, K_x, V_x, n_x, out);
    CUtensorMap tq;
    rc = make_query_map(s, &tq, Q_x, n_x);
    if (rc) return rc;
    const int key_rows = s->L + s->tail + n_x;
    rc = do_insert(s, K_x, V_x, n_x, 2, s->L + s->tail);
    if (rc) return rc;
    AttnParams p = attn_params(s, n_x, fs::kQueryVerify, key_rows, out);
    p.splits = choose_splits(s, p.q_tiles, key_rows);
    return launch_attention(s, p, tq);
}

// Same computation as fs_stream_attend_ext, with the split-KV partials in the
// fixed device array of stream_attn.cu instead of the handle's scratch, and no
// allocation on any path (the handle's buffers were allocated at create). The
// split count is the one fs_stream_attend_ext would use, capped so the
// partials fit the array; calls whose query tiles alone do not fit are
// rejected. Callers: drafting / verification loops that run under a device
// memory budget fixed at start-up and may not allocate per call (see
// static_split_scratch in stream_attn.cu). The first call on a device looks
// up the array's address (cudaGetSymbolAddress with that device current).
int fs_stream_attend_ext_static(fs_stream_t s, const void* Q_x, const void* K_x, const void* V_x, int n_x,
                                void* out) {
    if (!s) return fail(nullptr, FS_ERR_ARG, "NULL handle");
    int rc = check_block_args(s, Q_x, K_x, V_x, n_x, out);
    if (rc) return rc;
    const int key_rows = s->L + s->tail + n_x;
    const int q_tiles = (n_x * s->G + fs::kTileRows - 1) / fs::kTileRows;
    // Partial tiles per split, a deliberate upper bound: query tiles padded to
    // whole pairs (the kernel writes q_tiles * Hkv of them).
    const int tiles_padded = 2 * ((q_tiles + 1) / 2) * s->Hkv;
    const int cap = fs::static_split_scratch_tiles();
    if (tiles_padded > cap)
        return fail(s, FS_ERR_ARG,
                    "attend_ext_static: %d query tiles x %d kv heads need %d partial tiles per key split; "
                    "the static split scratch holds %d",
                    q_tiles, s->Hkv, tiles_padded, cap);
    int splits = choose_splits(s, q_tiles, key_rows);
    if (splits > cap / tiles_padded) splits = cap / tiles_padded;
    float* part_o = nullptr;
    float2* part_ml = nullptr;
    FS_CUDA(s, fs::static_split_scratch(&part_o, &part_ml));
    CUtensorMap tq;
    rc = make_query_map(s, &tq, Q_x, n_x);
    if (rc) return rc;
    rc = do_insert(s, K_x, V_x, n_x, 2, s->L + s->tail);
    if (rc) return rc;
    AttnParams p = attn_params(s, n_x, fs::kQueryVerify, key_rows, out);
    p.splits = splits;
    p.part_o = part_o;
    p.part_ml = part_ml;
    return launch_attention(s, p, tq);
}

// Insert + attend from host buffers. Three streams keep the copy engines and
// the SMs busy at once: the handle's own copy-in stream stages this call's
// K/V/Q (after the previous call's kernels have consumed the staging buffer),
// the caller's stream runs the kernels once those copies have landed (and the
// previous call's output has left the staging buffer), and the handle's
// copy-out stream returns the output. Consecutive calls on different handles
// (layers) therefore overlap one layer's upload, another's kernels and a
// third's download; fs_stream_sync waits for all three streams.
int fs_frame_attend(fs_stream_t s, const void* Q, const void* K, const void* V, int H, int Hkv, int d, void* out) {
    if (!s) return fail(nullptr, FS_ERR_ARG, "NULL handle");
    if (!Q || !K || !V || !out) return fail(s, FS_ERR_ARG, "NULL tensor pointer");
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out))
        return fail(s, FS_ERR_ARG, "pointers must be 16-byte aligned");
    if (out == Q || out == K || out == V) return fail(s, FS_ERR_ARG, "out must not alias an input");
    if (H < 1 || Hkv < 1 || H % Hkv) return fail(s, FS_ERR_ARG, "need H, Hkv >= 1 and H %% Hkv == 0");
    const int G = H / Hkv;
    if (fs::kTileRows % G) return fail(s, FS_ERR_ARG, "H/Hkv must divide 128 (got %d)", G);
    if (d != 64 && d != 128) return fail(s, FS_ERR_ARG, "head dim must be 64 or 128 (got %d)", d);
    fs::FrameParams p;
    std::memset(&p, 0, sizeof p);
    p.views = s->V;
    p.n = s->n;
    p.H = H;
    p.Hkv = Hkv;
    p.G = G;
    p.d = d;
    p.q_tiles = (s->n * G + fs::kTileRows - 1) / fs::kTileRows;
    p.q_scale = float(1.4426950408889634 / std::sqrt(double(d)));
    p.Q = static_cast<const uint16_t*>(Q);
    p.K = static_cast<const uint16_t*>(K);
    p.V = static_cast<const uint16_t*>(V);
    p.out = static_cast<float*>(out);
    p.err = s->err;
    p.wait_limit_ns = s->wait_limit_ns;
    FS_CUDA(s, fs::launch_frame_attn(p, s->stream));
    s->launches += 1;
    return FS_OK;
}

int fs_stream_step_host(fs_stream_t s, const void* K_new_h, const void* V_new_h, const void* Q_h, void* out_h) {
    if (!s) return fail(nullptr, FS_ERR_ARG, "NULL handle");
    if (!K_new_h || !V_new_h || !Q_h || !out_h) return fail(s, FS_ERR_ARG, "NULL host pointer");
    const int nt = s->state == FS_STATE_EXPECT_PREFILL ? s->L : s->step_tokens;
    const size_t kv = size_t(nt) * s->Hkv * s->d * 2;
    const size_t qb = size_t(nt) * s->H * s->d * 2;  // Q, bf16
    const size_t ob = 2 * qb;                           // out, fp32
    const size_t need = 2 * kv + qb + ob + 4 * 256;
    if (!s->copy_in) {
        FS_CUDA(s, cudaStreamCreateWithFlags(&s->copy_in, cudaStreamNonBlocking));
        FS_CUDA(s, cudaStreamCreateWithFlags(&s->copy_out, cudaStreamNonBlocking));
        FS_CUDA(s, cudaEventCreateWithFlags(&s->ev_in, cudaEventDisableTiming));
        FS_CUDA(s, cudaEventCreateWithFlags(&s->ev_done, cudaEventDisableTiming));
        FS_CUDA(s, cudaEventCreateWithFlags(&s->ev_out, cudaEventDisableTiming));
    }
    if (need > s->stage_bytes) {
        // Grown on first use (sized for the largest call so far), outside any capture.
        FS_CUDA(s, cudaStreamSynchronize(s->stream));
        FS_CUDA(s, cudaStreamSynchronize(s->copy_in));
        FS_CUDA(s, cudaStreamSynchronize(s->copy_out));
        cudaFree(s->stage);
        s->stage = nullptr;
        s->stage_bytes = 0;
        if (cudaMalloc(&s->stage, need) != cudaSuccess) {
            cudaGetLastError();
            return fail(s, FS_ERR_OOM, "staging allocation of %zu bytes failed", need);
        }
        s->stage_bytes = need;
    }
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    char* base = static_cast<char*>(s->stage);
    void* dK = base;
    void* dV = base + up(kv);
    void* dQ = base + 2 * up(kv);
    void* dO = base + 2 * up(kv) + up(qb);
    // Inputs: after the previous call's kernels have read the staging buffer.
    FS_CUDA(s, cudaStreamWaitEvent(s->copy_in, s->ev_done, 0));
    FS_CUDA(s, cudaMemcpyAsync(dK, K_new_h, kv, cudaMemcpyHostToDevice, s->copy_in));
    FS_CUDA(s, cudaMemcpyAsync(dV, V_new_h, kv, cudaMemcpyHostToDevice, s->copy_in));
    FS_CUDA(s, cudaMemcpyAsync(dQ, Q_h, qb, cudaMemcpyHostToDevice, s->copy_in));
    FS_CUDA(s, cudaEventRecord(s->ev_in, s->copy_in));
    // Kernels: after the inputs landed and the previous output left.
    FS_CUDA(s, cudaStreamWaitEvent(s->stream, s->ev_in, 0));
    FS_CUDA(s, cudaStreamWaitEvent(s->stream, s->ev_out, 0));
    int rc = fs_stream_insert(s, dK, dV);
    if (rc) return rc;
    rc = fs_stream_attend(s, dQ, dO);
    if (rc) return rc;
    FS_CUDA(s, cudaEventRecord(s->ev_done, s->stream));
    // Output.
    FS_CUDA(s, cudaStreamWaitEvent(s->copy_out, s->ev_done, 0));
    FS_CUDA(s, cudaMemcpyAsync(out_h, dO, ob, cudaMemcpyDeviceToHost, s->copy_out));
    FS_CUDA(s, cudaEventRecord(s->ev_out, s->copy_out));
    return FS_OK;
}

int fs_stream_sync(fs_stream_t s) {
    if (!s) return fail(nullptr, FS_ERR_ARG, "NULL handle");
    FS_CUDA(s, cudaStreamSynchronize(s->stream));
    if (s->copy_in) FS_CUDA(s, cudaStreamSynchronize(s->copy_in));
    if (s->copy_out) FS_CUDA(s, cudaStreamSynchronize(s->copy_out));
    return check_err_word(s);
}

int fs_stream_info(fs_stream_t s, fs_stream_info_t* info) {
    if (!s || !info) return fail(s, FS_ERR_ARG, "NULL argument");
    info->views = s->V;
    info->frames = s->T;
    info->tok_per_frame = s->n;
    info->text_len = s->X;
    info->H = s->H;
    info->Hkv = s->Hkv;
    info->d = s->d;
    info->window_len = s->L;
    info->step_tokens = s->step_tokens;
    info->state = s->state;
    info->insert_tokens = s->state == FS_STATE_EXPECT_PREFILL ? s->L : s->step_tokens;
    info->query_tokens = s->state == FS_STATE_EXPECT_PREFILL ? 0 : (s->state == FS_STATE_PREFILLED ? s->L : s->step_tokens);
    info->head = s->head;
    info->steps = s->steps;
    info->cache_bytes = s->cache_bytes;
    info->launches = s->launches;
    info->tail_tokens = s->tail;
    info->rebase_every = s->rebase_every;
    return FS_OK;
}

int fs_stream_debug_export(fs_stream_t s, void* K_phys, void* V_phys, int32_t* pos_phys, int32_t* frame_id_phys) {
    if (!s) return fail(nullptr, FS_ERR_ARG, "NULL handle");
    if (s->state == FS_STATE_EXPECT_PREFILL) return fail(s, FS_ERR_STATE, "nothing inserted yet");
    FS_CUDA(s, cudaStreamSynchronize(s->stream));
    const int rows = s->L + s->tail;
    const size_t row_bytes = size_t(s->d) * 2;
    for (int h = 0; h < s->Hkv; ++h) {
        const size_t src = size_t(h) * s->rows_cap * row_bytes;
        const size_t dst = size_t(h) * rows * row_bytes;
        if (K_phys)
            FS_CUDA(s, cudaMemcpy(static_cast<char*>(K_phys) + dst, reinterpret_cast<char*>(s->K_cache) + src,
                                  rows * row_bytes, cudaMemcpyDeviceToHost));
        if (V_phys)
            FS_CUDA(s, cudaMemcpy(static_cast<char*>(V_phys) + dst, reinterpret_cast<char*>(s->V_cache) + src,
                                  rows * row_bytes, cudaMemcpyDeviceToHost));
    }
    if (pos_phys) {
        // Positions as the attention kernel derives them (same device function,
        // head from the device-resident ring state).
        int* dpos = nullptr;
        FS_CUDA(s, cudaMalloc(&dpos, size_t(rows) * sizeof(int)));
        cudaError_t e = fs::launch_positions(shape_of(s), s->dstate, rows, dpos, s->stream);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s->stream);
        if (e == cudaSuccess) e = cudaMemcpy(pos_phys, dpos, size_t(rows) * sizeof(int), cudaMemcpyDeviceToHost);
        cudaFree(dpos);
        if (e != cudaSuccess) return fail(s, FS_ERR_CUDA, "position export failed: %s", cudaGetErrorString(e));
    }
    if (frame_id_phys) {
        for (int r = 0; r < rows; ++r) {
            if (r >= s->ring_rows) {
                frame_id_phys[r] = -1;
            } else {
                const int slot = (r % (s->T * s->n)) / s->n;
                frame_id_phys[r] = int32_t(s->slot_frame[slot]);
            }
        }
    }
    return check_err_word(s);
}

int fs_stream_debug_wait_probe(fs_stream_t s, int limit_us) {
    if (!s) return fail(nullptr, FS_ERR_ARG, "NULL handle");
    if (limit_us < 1 || limit_us > 1000000) return fail(s, FS_ERR_ARG, "limit_us must be in [1, 1e6]");
    FS_CUDA(s, fs::launch_wait_probe(s->err, (unsigned long long)limit_us * 1000ull, s->stream));
    return fs_stream_sync(s);
}

const char* fs_stream_last_error(fs_stream_t s) { return s ? s->last_error.c_str() : g_last_error.c_str(); }

const char* fs_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"
