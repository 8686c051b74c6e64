// moe_api.cu -- the C ABI declared in include/moe.h: argument validation,
// workspace layout, TMA tensor maps and the launch sequence of one layer.
//
// One call of moe_ffn_forward enqueues, on the caller's stream:
//   route_kernel   top-k, softmax, histogram, scan, permutation, padded layout
//                  (from 1024 tokens: route_topk_kernel + route_place_kernel)
//   quant_kernel   per-token e4m3 quantisation (FP8) and zeroing of out32
//   stage-1 GEMM   TMA gather of each expert's token rows, GEMM with w1/w3 +
//                  SwiGLU (+ MX quantisation of h)
//   stage-2 GEMM   GEMM with w2 + routing-weighted scatter-add into out32
//   finalize       out32 -> bf16 out
// (rocketrecap.com "FlyDSL kernels in JAX", paragraph 2 and timestamp 5:56.)
#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "bwd.cuh"
#include "kernels.cuh"

namespace moe {

__device__ int g_status_word = 0;

namespace {

std::atomic<int> g_opt_path{0};
std::atomic<int> g_opt_splitk{0};
std::atomic<int> g_opt_timeout_ms{2000};
std::atomic<int> g_opt_test_stall{0};
std::atomic<int> g_opt_test_corrupt{0};
std::atomic<int> g_opt_gather{0};

// ---------------------------------------------------------------- profiling

struct ProfRecord {
    int kernel;
    int launches;  // kernel launches between the two events
    cudaEvent_t start, stop;
};
std::atomic<int> g_prof_on{0};
std::mutex g_prof_mutex;
std::vector<ProfRecord> g_prof_records;
std::vector<cudaEvent_t> g_prof_pool;

cudaEvent_t prof_event() {
    if (!g_prof_pool.empty()) {
        cudaEvent_t e = g_prof_pool.back();
        g_prof_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

// Records events around one kernel launch when profiling is on.
struct ProfScope {
    int kernel;
    cudaStream_t stream;
    int launches;
    cudaEvent_t start = nullptr;
    ProfScope(int k, cudaStream_t s, int n = 1) : kernel(k), stream(s), launches(n) {
        if (!g_prof_on.load()) return;
        std::lock_guard<std::mutex> lock(g_prof_mutex);
        start = prof_event();
        if (start) cudaEventRecord(start, stream);
    }
    ~ProfScope() {
        if (!start) return;
        std::lock_guard<std::mutex> lock(g_prof_mutex);
        cudaEvent_t stop = prof_event();
        if (!stop) return;
        cudaEventRecord(stop, stream);
        g_prof_records.push_back({kernel, launches, start, stop});
    }
};

// ---------------------------------------------------------------- per-context state
// The status word's device address, the SM count and the resident CTA pairs
// are looked up once per CUDA context (not per device ordinal: after a device
// reset, or under another driver-API context on the same device, an address
// taken in the old context is no longer valid).  A context is identified by
// the driver's unique context id (cuCtxGetId), which is never reused.

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_fn(const char* name) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<Fn>(p);
}

}  // namespace

// Key of the context current on this thread: the driver's context id, which
// is never reused (or, where the driver offers no ids, one key per device
// ordinal).  False when no context is current yet.
bool context_key(unsigned long long* key) {
    static CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    int dev = 0;
    if (get_current) {
        CUcontext ctx = nullptr;
        if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
        if (get_id && get_id(ctx, key) == CUDA_SUCCESS) return true;
    }
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    *key = ~0ull - (unsigned long long)dev;
    return true;
}

namespace {

struct CtxInfo {
    unsigned long long ctx_id;
    int* status;
    int num_sms;
    int max_pairs[2][2];  // [stage-1][fp8]
};
constexpr int kMaxContexts = 64;
CtxInfo g_ctx[kMaxContexts];
int g_ctx_count = 0, g_ctx_next = 0;
std::mutex g_ctx_mutex;

// Per-context state of the current context, looked up (and its context made
// current by the runtime, if none was) on first use.
int context_info(CtxInfo* out) {
    std::lock_guard<std::mutex> lock(g_ctx_mutex);
    unsigned long long key = 0;
    if (context_key(&key)) {
        for (int i = 0; i < g_ctx_count; ++i)
            if (g_ctx[i].ctx_id == key) {
                *out = g_ctx[i];
                return MOE_OK;
            }
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    CtxInfo c{};
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
    if (cudaDeviceGetAttribute(&c.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MOE_ERR_CUDA;
    for (int st = 0; st < 2; ++st)
        for (int f = 0; f < 2; ++f) c.max_pairs[st][f] = gemm_max_pairs(st + 1, f != 0);
    c.status = static_cast<int*>(p);
    if (!context_key(&key)) return MOE_ERR_CUDA;  // the lookup above made a context current
    c.ctx_id = key;
    g_ctx[g_ctx_next] = c;
    g_ctx_next = (g_ctx_next + 1) % kMaxContexts;
    if (g_ctx_count < kMaxContexts) ++g_ctx_count;
    *out = c;
    return MOE_OK;
}

// ---------------------------------------------------------------- workspace

constexpr int kRegions = 18;

struct Layout {
    size_t off[kRegions];
    size_t size[kRegions];
    size_t total;
    int A, MT_max, S_max;
};

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool dims_ok(int T, int H, int F, int E, int k, int dtype) {
    return T >= 0 && H > 0 && F > 0 && E >= 1 && E <= kMaxExperts && k >= 1 && k <= E && k <= kMaxTopK &&
           (dtype == MOE_BF16 || dtype == MOE_FP8_E4M3 || dtype == MOE_MXFP4);
}

// e4m3 activations and h (FP8 and MX FP4 weights) or bf16 throughout
bool e4m3_acts(int dtype) { return dtype != MOE_BF16; }

Layout make_layout(int T, int H, int F, int E, int k, int dtype) {
    Layout L{};
    const size_t A = (size_t)T * k;
    const size_t eb = e4m3_acts(dtype) ? 1 : 2;
    L.A = (int)A;
    L.MT_max = (int)((A + kBlockM - 1) / kBlockM) + E;  // sum over experts of ceil(n_e / 128)
    L.S_max = L.MT_max * kBlockM;
    const size_t S = L.S_max;
    size_t sz[kRegions] = {};
    sz[MOE_WS_TOPK_IDS] = 4 * A;
    sz[MOE_WS_TOPK_W] = 4 * A;
    sz[MOE_WS_COUNTS] = 4 * (size_t)E;
    sz[MOE_WS_OFFSETS] = 4 * (size_t)(E + 1);
    sz[MOE_WS_PERM] = 4 * A;
    sz[MOE_WS_INV_PERM] = 4 * A;
    sz[MOE_WS_SLOT_OF] = 4 * A;
    sz[MOE_WS_XS] = e4m3_acts(dtype) ? (size_t)T * H : 0;  // per-token e4m3 rows (BF16 reads x itself)
    sz[MOE_WS_SX] = e4m3_acts(dtype) ? 4 * (size_t)T : 0;
    sz[MOE_WS_H] = S * act_pitch((long)F * eb);
    sz[MOE_WS_H_SF] = e4m3_acts(dtype) ? (size_t)L.MT_max * (F / 128) * 512 : 0;
    sz[MOE_WS_OUT32] = 4 * (size_t)T * H;
    sz[MOE_WS_NUM_MTILES] = 4;
    sz[MOE_WS_SLOT_ASSIGN] = 4 * S;
    sz[MOE_WS_MTILE_EXPERT] = 4 * (size_t)L.MT_max;
    sz[MOE_WS_ROUTE_BLOCKS] = 4 * (size_t)((T + 255) / 256) * E;
    sz[MOE_WS_XG] = S * act_pitch((long)H * eb);
    sz[MOE_WS_SX_SLOT] = e4m3_acts(dtype) ? 4 * S : 0;
    size_t off = 0;
    for (int r = 0; r < kRegions; ++r) {
        L.off[r] = off;
        L.size[r] = sz[r];
        off = align_up(off + sz[r], 1024);
    }
    L.total = off;
    return L;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------- tensor maps

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// 2-D row-major matrix [rows, cols] of elements of `eb` bytes, rows `pitch`
// bytes apart; box = 128 bytes
// of K by box_rows rows, 128-byte swizzle (matches the MMA descriptors).
bool make_map(CUtensorMap* map, const void* base, size_t rows, size_t cols, size_t pitch, int eb, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)pitch};
    const cuuint32_t box[2] = {(cuuint32_t)(128 / eb), (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(map, eb == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                          const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Map of a buffer of 128-byte rows copied as they are (no swizzle), box_rows
// rows per copy: the preshuffled weight blocks (already in the operand's
// shared-memory image) and the tiled scale chunks of h.
bool make_map_rows(CUtensorMap* map, const void* base, size_t rows, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {128, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {128};
    const cuuint32_t box[2] = {128, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int launch_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// ---------------------------------------------------------------- tensor-map cache
// The tensor maps of a call depend only on the buffers' addresses and the
// problem's shape, so they are encoded once per (workspace, weights, shape,
// tile configuration) and reused by later calls with the same arguments.

struct MapKey {
    const void* x;
    const void* ws;
    const void* w13;
    const void* w2;
    int T, H, F, E, k, dtype, cfg1, cfg2;
    bool operator==(const MapKey& o) const {
        return x == o.x && ws == o.ws && w13 == o.w13 && w2 == o.w2 && T == o.T && H == o.H && F == o.F && E == o.E &&
               k == o.k && dtype == o.dtype && cfg1 == o.cfg1 && cfg2 == o.cfg2;
    }
};
struct MapSet {
    CUtensorMap tg1, ta1, ta1s, ta2, ta2s, tb1, tb2, tsf2;
};
constexpr int kMapCache = 16;
struct MapEntry {
    MapKey key;
    MapSet maps;
    bool valid;
};
MapEntry g_maps[kMapCache];
int g_maps_next = 0;
std::mutex g_maps_mutex;

bool find_maps(const MapKey& key, MapSet* out) {
    std::lock_guard<std::mutex> lock(g_maps_mutex);
    for (const MapEntry& m : g_maps)
        if (m.valid && m.key == key) {
            *out = m.maps;
            return true;
        }
    return false;
}

void store_maps(const MapKey& key, const MapSet& maps) {
    std::lock_guard<std::mutex> lock(g_maps_mutex);
    g_maps[g_maps_next] = {key, maps, true};
    g_maps_next = (g_maps_next + 1) % kMapCache;
}

}  // namespace

// ---------------------------------------------------------------- argument checks
// The host-side checks of a layer call, in the order both layer entry points
// apply them (dimensions, null pointers, supported shapes, alignment); the
// workspace size is checked after them.
int check_forward_args(const void* x, const float* logits, const void* w13, const void* s13, const void* w2,
                       const void* s2, int T, int H, int F, int E, int k, int dtype, const void* out, const void* ws) {
    if (!dims_ok(T, H, F, E, k, dtype)) return MOE_ERR_INVALID_ARG;
    const bool fp8 = e4m3_acts(dtype);
    if (!w13 || !w2 || !ws || (fp8 && (!s13 || !s2))) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!x || !logits || !out)) return MOE_ERR_INVALID_ARG;
    if (H % 128 || F % 128) return MOE_ERR_UNSUPPORTED;
    if ((long long)T * k > 262144) return MOE_ERR_UNSUPPORTED;
    const void* ptrs[] = {x, logits, w13, s13, w2, s2, out, ws};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return MOE_ERR_ALIGNMENT;
    return MOE_OK;
}

namespace {

// K splits of the second GEMM: enough work units for every SM when the layer
// is small (decode), 1 otherwise.  Must divide F/128.
int choose_splits(int mt_est, int n_tiles, int k_tiles, int num_sms) {
    const int forced = g_opt_splitk.load();
    if (forced > 0) return forced;
    for (int s = 1; s <= k_tiles / 4; ++s) {
        if (k_tiles % s) continue;
        if ((long)mt_est * n_tiles * s >= 6L * num_sms) return s;
    }
    return 1;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_workspace_size(int T, int H, int F, int E, int k, int dtype) {
    if (!dims_ok(T, H, F, E, k, dtype)) return 0;
    return make_layout(T, H, F, E, k, dtype).total;
}

long long moe_workspace_region(int T, int H, int F, int E, int k, int dtype, int which, size_t* bytes) {
    if (!dims_ok(T, H, F, E, k, dtype) || which < 0 || which >= kRegions) return -1;
    const Layout L = make_layout(T, H, F, E, k, dtype);
    if (bytes) *bytes = L.size[which];
    return (long long)L.off[which];
}

int moe_set_option(int option, int value) {
    switch (option) {
        case MOE_OPT_PATH:
            if (value < 0 || value > 4) return MOE_ERR_INVALID_ARG;
            return g_opt_path.exchange(value);
        case MOE_OPT_SPLITK:
            if (value < 0) return MOE_ERR_INVALID_ARG;
            return g_opt_splitk.exchange(value);
        case MOE_OPT_TIMEOUT_MS:
            if (value < 1) return MOE_ERR_INVALID_ARG;
            return g_opt_timeout_ms.exchange(value);
        case MOE_OPT_TEST_STALL:
            if (value < 0 || value > 1) return MOE_ERR_INVALID_ARG;
            return g_opt_test_stall.exchange(value);
        case MOE_OPT_TEST_CORRUPT:
            if (value < 0 || value > 3) return MOE_ERR_INVALID_ARG;
            return g_opt_test_corrupt.exchange(value);
        case MOE_OPT_GATHER:
            if (value < 0 || value > 2) return MOE_ERR_INVALID_ARG;
            return g_opt_gather.exchange(value);
        default:
            return MOE_ERR_INVALID_ARG;
    }
}

int moe_prepare_weights(const void* w1, const void* w3, const float* s1, const float* s3, const void* w2,
                        void* w13_out, float* s13_out, void* w2_out, int E, int F, int H, int dtype, void* stream) {
    if (!w1 || !w3 || !w2 || !w13_out || !w2_out || E < 1 || E > kMaxExperts || F <= 0 || H <= 0)
        return MOE_ERR_INVALID_ARG;
    if (dtype != MOE_BF16 && dtype != MOE_FP8_E4M3) return MOE_ERR_INVALID_ARG;
    const bool fp8 = dtype == MOE_FP8_E4M3;
    if (fp8 && (!s1 || !s3 || !s13_out)) return MOE_ERR_INVALID_ARG;
    if (F % 128 || H % 128) return MOE_ERR_UNSUPPORTED;
    const void* ptrs[] = {w1, w3, w2, w13_out, w2_out, fp8 ? s13_out : nullptr};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return MOE_ERR_ALIGNMENT;
    const int eb = fp8 ? 1 : 2;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    ProfScope ps(MOE_KERNEL_PREPARE, st, fp8 ? 3 : 2);
    if (launch_preshuffle(static_cast<const uint8_t*>(w1), static_cast<const uint8_t*>(w3),
                          static_cast<uint8_t*>(w13_out), E, F, 2 * F, H * eb, true, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (launch_preshuffle(static_cast<const uint8_t*>(w2), nullptr, static_cast<uint8_t*>(w2_out), E, H, H, F * eb,
                          false, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (fp8 && launch_interleave_scales(s1, s3, s13_out, E, F, st) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}

int moe_prepare_weights_mx(const void* w1, const void* w3, const void* s1, const void* s3, const void* w2,
                           const void* s2, void* w13_out, void* s13_out, void* w2_out, void* s2_out, int E, int F,
                           int H, void* stream) {
    if (!w1 || !w3 || !s1 || !s3 || !w2 || !s2 || !w13_out || !s13_out || !w2_out || !s2_out || E < 1 ||
        E > kMaxExperts || F <= 0 || H <= 0)
        return MOE_ERR_INVALID_ARG;
    if (F % 128 || H % 128) return MOE_ERR_UNSUPPORTED;
    const void* ptrs[] = {w1, w3, s1, s3, w2, s2, w13_out, s13_out, w2_out, s2_out};
    for (const void* p : ptrs)
        if (!aligned16(p)) return MOE_ERR_ALIGNMENT;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    ProfScope ps(MOE_KERNEL_PREPARE, st, 4);
    auto u8 = [](const void* p) { return static_cast<const uint8_t*>(p); };
    if (launch_mx_prepare(u8(w1), u8(w3), u8(s1), u8(s3), static_cast<uint8_t*>(w13_out),
                          static_cast<uint8_t*>(s13_out), E, F, 2 * F, H, true, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (launch_mx_prepare(u8(w2), nullptr, u8(s2), nullptr, static_cast<uint8_t*>(w2_out),
                          static_cast<uint8_t*>(s2_out), E, H, H, F, false, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

int moe_route(const float* logits, int T, int E, int k, int32_t* topk_ids, float* topk_w, int32_t* counts,
              int32_t* offsets, int32_t* perm, int32_t* inv_perm, void* ws, size_t ws_bytes, void* stream) {
    (void)ws;
    (void)ws_bytes;
    if (T < 0 || E < 1 || E > kMaxExperts || k < 1 || k > E || k > kMaxTopK) return MOE_ERR_INVALID_ARG;
    if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!logits || !topk_ids || !topk_w || !perm || !inv_perm)) return MOE_ERR_INVALID_ARG;
    if ((long long)T * k > 262144) return MOE_ERR_UNSUPPORTED;
    RouteOutputs o{topk_ids, topk_w, counts, offsets, perm, inv_perm, nullptr, nullptr, nullptr, nullptr};
    return launch_status(launch_route(logits, T, E, k, o, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

// The d_ff-sharded layer's arguments (see moe_ffn_forward_dff).
struct Dff {
    int n_ranks, rank;
    float* const* peer_out32;
    unsigned int* const* peer_counter;
};

// The layer call: the whole layer (dff == nullptr), or one rank's part of the
// d_ff-sharded layer (its GEMMs on its d_ff slice, the scatter-add into the
// owners' combine rows, and the signal to every rank; no rounding).
int forward_impl(const void* x, const float* logits, const void* w13, const void* s13, const void* w2,
                 const void* s2, int T, int H, int F, int E, int k, int dtype, void* out, void* ws, size_t ws_bytes,
                 void* stream, const Dff* dff) {
    const int rc_args = check_forward_args(x, logits, w13, s13, w2, s2, T, H, F, E, k, dtype, dff ? ws : out, ws);
    if (rc_args != MOE_OK) return rc_args;
    const bool fp8 = e4m3_acts(dtype);          // e4m3 activations and h
    const bool mxw = dtype == MOE_MXFP4;        // MX FP4 weights with block scales
    const Layout L = make_layout(T, H, F, E, k, dtype);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    const int opt_path = g_opt_path.load();  // read once per call
    if (opt_path == 4 && L.A > 32) return MOE_ERR_UNSUPPORTED;  // forced tiny-batch tiles
    PeerCounters counters{};
    if (dff)
        for (int g = 0; g < dff->n_ranks; ++g) counters.c[g] = dff->peer_counter[g];
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) return dff ? launch_status(launch_dff_signal(counters, dff->n_ranks, st)) : MOE_OK;

    CtxInfo ctx{};
    if (context_info(&ctx) != MOE_OK) return MOE_ERR_CUDA;
    int* status = ctx.status;
    const int num_sms = ctx.num_sms;
    auto max_pairs = [&](int stage, bool f8) { return ctx.max_pairs[stage - 1][f8 ? 1 : 0]; };
    uint8_t* w = static_cast<uint8_t*>(ws);
    auto reg = [&](int r) { return w + L.off[r]; };
    const int eb = fp8 ? 1 : 2;

    // Tile configuration (see launch_gemm), by the average rows per expert:
    //   <= 64 (decode-sized): the first GEMM on one-CTA 128 x 256 tiles, the
    //     second on 128 x 128 tiles with K split so that every SM streams
    //     weights (its long K would leave most SMs idle otherwise);
    //   up to 512: 128 x 256 tiles for both;
    //   from 512 on: CTA pairs (below that, an expert's last, lone 128-row
    //     tile makes a pair compute too many rows twice).
    // One-CTA 128 x 256 tiles where the pair kernel cannot be resident;
    // 128-wide tiles when a dimension is not a multiple of 256.
    // (The tiny-batch tiles, 32 activation rows per stage with deeper
    // pipelines, are only used when forced: measured against the small-batch
    // configuration at 16 tokens they were not faster.)
    const bool small_batch = L.A <= 64 * E;
    int cfg1, cfg2;
    if (opt_path == 0) {
        cfg1 = (L.A < 512 * E) ? 2 : 0;
        cfg2 = small_batch ? 1 : cfg1;
    } else {
        cfg1 = cfg2 = opt_path - 1;
    }
    // MX FP4 weights: 128 x 128 one-CTA tiles (room in TMEM for both operands'
    // scales); the tiny-batch form (32 activation rows per stage, deeper
    // pipelines) only when forced: at 16 tokens it measured 284 us a layer
    // against 274 us for the 128-row form
    if (mxw) cfg1 = cfg2 = (opt_path == 4) ? 3 : 1;
    if ((2 * F) % gemm_block_n(1, fp8, cfg1, mxw)) cfg1 = 1;
    if (H % gemm_block_n(2, fp8, cfg2, mxw)) cfg2 = 1;
    if (cfg1 == 0 && max_pairs(1, fp8) < 1) cfg1 = 2;
    if (cfg2 == 0 && max_pairs(2, fp8) < 1) cfg2 = 2;
    const int bn1 = gemm_block_n(1, fp8, cfg1, mxw);
    const int bn2 = gemm_block_n(2, fp8, cfg2, mxw);
    if ((2 * F) % bn1 || H % bn2) return MOE_ERR_UNSUPPORTED;

    // stage 1 gathers token rows: from the per-token e4m3 rows (FP8) or from
    // x itself (BF16), one-row boxes of 128 bytes
    const void* a1_base = fp8 ? (const void*)reg(MOE_WS_XS) : x;
    const MapKey mkey{a1_base, ws, w13, w2, T, H, F, E, k, dtype, cfg1, cfg2};
    MapSet ms;
    if (!find_maps(mkey, &ms)) {
        if (!make_map(&ms.tg1, a1_base, T, H, (size_t)H * eb, eb, 1) ||
            !make_map(&ms.ta1, reg(MOE_WS_XG), L.S_max, H, act_pitch((long)H * eb), eb, kBlockM) ||
            !make_map(&ms.ta1s, reg(MOE_WS_XG), L.S_max, H, act_pitch((long)H * eb), eb, 32) ||
            !make_map(&ms.ta2, reg(MOE_WS_H), L.S_max, F, act_pitch((long)F * eb), eb, kBlockM) ||
            !make_map(&ms.ta2s, reg(MOE_WS_H), L.S_max, F, act_pitch((long)F * eb), eb, 32))
            return MOE_ERR_CUDA;
        if (cfg1 == 0 && !make_map_rows(&ms.tb1, w13, (size_t)E * (2 * F) * (H * eb / 128), kWBlockRows))
            return MOE_ERR_CUDA;
        if (cfg2 == 0 && !make_map_rows(&ms.tb2, w2, (size_t)E * H * (F * eb / 128), kWBlockRows))
            return MOE_ERR_CUDA;
        if (cfg2 == 0 && fp8 && !make_map_rows(&ms.tsf2, reg(MOE_WS_H_SF), (size_t)L.MT_max * (F / 128) * 4, 4))
            return MOE_ERR_CUDA;
        store_maps(mkey, ms);
    }
    // The first GEMM's activation rows: gathered by TMA inside the GEMM from
    // the per-token rows, or tile copies of the rows a gather pass wrote in the
    // padded layout.  A tile of many rows needs 32 four-row gathers per K
    // step, which keeps the copy engine from feeding the tensor cores, so the
    // gather pass is the default (MOE_OPT_GATHER selects either).
    const int opt_gather = g_opt_gather.load();
    const bool tma_gather = (opt_gather == 1);
    const GemmMaps maps1{&ms.ta1, &ms.ta1s, cfg1 == 0 ? &ms.tb1 : nullptr, tma_gather ? &ms.tg1 : nullptr};
    const GemmMaps maps2{&ms.ta2, &ms.ta2s, cfg2 == 0 ? &ms.tb2 : nullptr,
                         (cfg2 == 0 && fp8) ? &ms.tsf2 : nullptr};
    // grid: one CTA per SM at most; pairs: whole clusters that can be resident
    auto grid_for = [&](int stage, int c, long units_per_mtile) {
        if (c == 0) {
            const long clusters = std::min<long>((long)max_pairs(stage, fp8), (long)L.MT_max * units_per_mtile);
            return (int)(2 * std::max<long>(clusters, 1));
        }
        return (int)std::min<long>((long)L.MT_max * units_per_mtile, num_sms);
    };

    // 1. routing and the expert-padded layout
    RouteOutputs o{reinterpret_cast<int32_t*>(reg(MOE_WS_TOPK_IDS)), reinterpret_cast<float*>(reg(MOE_WS_TOPK_W)),
                   reinterpret_cast<int32_t*>(reg(MOE_WS_COUNTS)), reinterpret_cast<int32_t*>(reg(MOE_WS_OFFSETS)),
                   reinterpret_cast<int32_t*>(reg(MOE_WS_PERM)), reinterpret_cast<int32_t*>(reg(MOE_WS_INV_PERM)),
                   reinterpret_cast<int32_t*>(reg(MOE_WS_SLOT_OF)), reinterpret_cast<int32_t*>(reg(MOE_WS_SLOT_ASSIGN)),
                   reinterpret_cast<int32_t*>(reg(MOE_WS_MTILE_EXPERT)),
                   reinterpret_cast<int32_t*>(reg(MOE_WS_NUM_MTILES)),
                   reinterpret_cast<int32_t*>(reg(MOE_WS_ROUTE_BLOCKS))};
    {
        ProfScope ps(MOE_KERNEL_ROUTE, st, route_launches(T, o));
        if (launch_route(logits, T, E, k, o, st) != cudaSuccess) return MOE_ERR_CUDA;
    }
    // failure-detection test hook: overwrite one entry of a routing table with
    // an index far out of range (bytes 0x7F), as a corrupted table would hold
    const int corrupt = g_opt_test_corrupt.load();
    if (corrupt) {
        void* target = corrupt == 1 ? (void*)o.slot_assign : corrupt == 2 ? (void*)o.mtile_expert : (void*)o.num_mtiles;
        if (cudaMemsetAsync(target, 0x7F, sizeof(int32_t), st) != cudaSuccess) return MOE_ERR_CUDA;
    }

    // 2. per-token quantisation (FP8) -- with the gather into the padded
    // layout, or alone for the first GEMM's TMA gather -- and zeroing of the
    // combine buffer
    const int* num_mt = o.num_mtiles;
    float* out32 = reinterpret_cast<float*>(reg(MOE_WS_OUT32));
    float* sx = fp8 ? reinterpret_cast<float*>(reg(MOE_WS_SX)) : nullptr;
    {
        ProfScope ps(MOE_KERNEL_QUANT, st);
        const cudaError_t e =
            tma_gather ? launch_quant(fp8, static_cast<const __nv_bfloat16*>(x), T, H, fp8 ? reg(MOE_WS_XS) : nullptr,
                                      sx, dff ? nullptr : out32, st)
                       : launch_gather(fp8, static_cast<const __nv_bfloat16*>(x), T, H, k, o.slot_of, L.S_max,
                                       reg(MOE_WS_XG), sx, fp8 ? reinterpret_cast<float*>(reg(MOE_WS_SX_SLOT)) : nullptr,
                                       dff ? nullptr : out32, status, st);
        if (e != cudaSuccess) return MOE_ERR_CUDA;
    }

    const unsigned long long timeout_ns = (unsigned long long)g_opt_timeout_ms.load() * 1000000ull;

    // 3. stage 1: GEMM with w1/w3 on the gathered token rows, SwiGLU epilogue
    GemmArgs g1{};
    g1.num_mtiles = num_mt;
    g1.mtile_expert = o.mtile_expert;
    g1.slot_assign = o.slot_assign;
    g1.row_scale = sx;
    g1.row_scale_slot = fp8 ? reinterpret_cast<const float*>(reg(MOE_WS_SX_SLOT)) : nullptr;
    g1.col_scale = (fp8 && !mxw) ? static_cast<const float*>(s13) : nullptr;
    g1.b_sf = mxw ? static_cast<const uint8_t*>(s13) : nullptr;
    g1.b_blocks = static_cast<const uint8_t*>(w13);
    g1.b_evict_first = small_batch ? 1 : 0;  // one m-tile per expert: each weight block is read once
    g1.out = reg(MOE_WS_H);
    g1.out_sf = fp8 ? reg(MOE_WS_H_SF) : nullptr;
    g1.rows_b = 2 * F;
    g1.n_tiles = 2 * F / bn1;
    g1.k_tiles = H * eb / 128;
    g1.splits = 1;
    g1.out_pitch = act_pitch((long)F * eb);
    g1.f_tiles = F / 128;
    g1.topk = k;
    g1.T = T;
    g1.timeout_ns = timeout_ns;
    g1.status = status;
    g1.test_stall = g_opt_test_stall.load();
    g1.counts = o.counts;
    g1.num_experts = E;
    g1.mt_max = L.MT_max;
    g1.a_gather = tma_gather ? 1 : 0;
    g1.group_m = (cfg1 != 1) ? 1 : 0;
    {
        ProfScope ps(MOE_KERNEL_STAGE1, st);
        if (launch_gemm(1, fp8, cfg1, maps1, g1, grid_for(1, cfg1, g1.n_tiles), st, mxw) != cudaSuccess)
            return MOE_ERR_CUDA;
    }

    // 4. stage 2: GEMM with w2, weighted scatter-add epilogue
    GemmArgs g2 = g1;
    g2.row_scale = nullptr;
    g2.test_stall = 0;
    g2.group_m = (cfg2 == 0 || cfg2 == 2) ? 1 : 0;
    g2.col_scale = (fp8 && !mxw) ? static_cast<const float*>(s2) : nullptr;
    g2.b_sf = mxw ? static_cast<const uint8_t*>(s2) : nullptr;
    g2.topk_w = o.topk_w;
    g2.a_sf = fp8 ? reg(MOE_WS_H_SF) : nullptr;
    g2.b_blocks = static_cast<const uint8_t*>(w2);
    g2.b_evict_first = small_batch ? 1 : 0;
    g2.out = out32;
    g2.out_sf = nullptr;
    g2.rows_b = H;
    g2.n_tiles = H / bn2;
    g2.k_tiles = F * eb / 128;
    const int mt_est = std::min(L.MT_max, (L.A + kBlockM - 1) / kBlockM + std::min(E, L.A));
    g2.splits = (cfg2 == 0) ? choose_splits((mt_est + 1) / 2, g2.n_tiles, g2.k_tiles, std::max(1, num_sms / 2))
                            : choose_splits(mt_est, g2.n_tiles, g2.k_tiles, num_sms);
    if (g2.splits < 1 || g2.k_tiles % g2.splits) return MOE_ERR_UNSUPPORTED;
    g2.out_pitch = (long)H * 4;
    if (dff) {  // add into the owners' combine rows (peer memory)
        g2.n_ranks = dff->n_ranks;
        g2.rank = dff->rank;
        g2.rows_per_rank = (T + dff->n_ranks - 1) / dff->n_ranks;
        for (int g = 0; g < dff->n_ranks; ++g) g2.peer_out[g] = dff->peer_out32[g];
        g2.out = dff->peer_out32[dff->rank];
    }
    {
        ProfScope ps(MOE_KERNEL_STAGE2, st);
        if (launch_gemm(2, fp8, cfg2, maps2, g2, grid_for(2, cfg2, (long)g2.n_tiles * g2.splits), st, mxw) !=
            cudaSuccess)
            return MOE_ERR_CUDA;
    }
    if (dff) return launch_status(launch_dff_signal(counters, dff->n_ranks, st));

    // 5. fp32 -> bf16
    ProfScope ps(MOE_KERNEL_FINALIZE, st);
    return launch_status(launch_finalize(out32, static_cast<__nv_bfloat16*>(out), (size_t)T * H, num_sms, st));
}

}  // namespace

extern "C" {

int moe_ffn_forward(const void* x, const float* logits, const void* w13, const void* s13, const void* w2,
                    const void* s2, int T, int H, int F, int E, int k, int dtype, void* out, void* ws,
                    size_t ws_bytes, void* stream) {
    return forward_impl(x, logits, w13, s13, w2, s2, T, H, F, E, k, dtype, out, ws, ws_bytes, stream, nullptr);
}

int moe_ffn_forward_dff(const void* x, const float* logits, const void* w13, const void* s13, const void* w2,
                        const void* s2, int T, int H, int F_shard, int E, int k, int dtype, int n_ranks, int rank,
                        float* const* peer_out32, unsigned int* const* peer_counter, void* ws, size_t ws_bytes,
                        void* stream) {
    if (n_ranks < 1 || n_ranks > kMaxRanks || rank < 0 || rank >= n_ranks || !peer_out32 || !peer_counter)
        return MOE_ERR_INVALID_ARG;
    for (int g = 0; g < n_ranks; ++g) {
        if (!peer_out32[g] || !peer_counter[g]) return MOE_ERR_INVALID_ARG;
        if (!aligned16(peer_out32[g]) || (reinterpret_cast<uintptr_t>(peer_counter[g]) & 3u))
            return MOE_ERR_ALIGNMENT;
    }
    const Dff dff{n_ranks, rank, peer_out32, peer_counter};
    return forward_impl(x, logits, w13, s13, w2, s2, T, H, F_shard, E, k, dtype, nullptr, ws, ws_bytes, stream,
                        &dff);
}

int moe_dff_finalize(float* out32_rows, void* out, int rows, int H, const unsigned int* counter, unsigned int target,
                     void* stream) {
    if (rows < 0 || H <= 0 || H % 128 || (rows > 0 && (!out32_rows || !out)) || !counter) return MOE_ERR_INVALID_ARG;
    if ((out32_rows && !aligned16(out32_rows)) || (out && !aligned16(out)) ||
        (reinterpret_cast<uintptr_t>(counter) & 3u))
        return MOE_ERR_ALIGNMENT;
    CtxInfo ctx{};
    if (context_info(&ctx) != MOE_OK) return MOE_ERR_CUDA;
    const unsigned long long timeout_ns = (unsigned long long)g_opt_timeout_ms.load() * 1000000ull;
    return launch_status(launch_dff_finalize(out32_rows, static_cast<__nv_bfloat16*>(out), (size_t)rows * H, counter,
                                             target, timeout_ns, ctx.status, ctx.num_sms,
                                             static_cast<cudaStream_t>(stream)));
}

int moe_profile_enable(int on) { return g_prof_on.exchange(on ? 1 : 0); }

int moe_profile_read(double* ms_total, int* launches, int reset) {
    std::lock_guard<std::mutex> lock(g_prof_mutex);
    if (ms_total)
        for (int i = 0; i < MOE_KERNEL_COUNT; ++i) ms_total[i] = 0.0;
    if (launches)
        for (int i = 0; i < MOE_KERNEL_COUNT; ++i) launches[i] = 0;
    int rc = MOE_OK;
    for (const ProfRecord& r : g_prof_records) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess) {
            rc = MOE_ERR_CUDA;
            continue;
        }
        if (ms_total) ms_total[r.kernel] += ms;
        if (launches) launches[r.kernel] += r.launches;
    }
    if (reset) {
        for (const ProfRecord& r : g_prof_records) {
            g_prof_pool.push_back(r.start);
            g_prof_pool.push_back(r.stop);
        }
        g_prof_records.clear();
    }
    return rc;
}

int moe_get_status(void* stream) {
    CtxInfo ctx{};
    if (context_info(&ctx) != MOE_OK) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, ctx.status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpy(ctx.status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return MOE_ERR_CUDA;
    return v;
}

}  // extern "C"

// ---------------------------------------------------------------- backward pass
// Workspace: the forward layout of the BF16 layer (routing tables, gathered x,
// h, the fp32 row buffer -- here dx32) followed by the backward's own regions.

namespace {

enum BwdRegion { kBwGU = 0, kBwDYG, kBwDOG, kBwDGU, kBwDW, kBwRegions };

struct BwdLayout {
    Layout fwd;
    size_t off[kBwRegions];
    size_t total;
};

BwdLayout make_bwd_layout(int T, int H, int F, int E, int k) {
    BwdLayout B{};
    B.fwd = make_layout(T, H, F, E, k, MOE_BF16);
    const size_t S = B.fwd.S_max;
    size_t sz[kBwRegions];
    sz[kBwGU] = S * act_pitch(8L * F);   // fp32 g|u rows [S, 2F]
    sz[kBwDYG] = S * act_pitch(2L * H);  // dy per slot [S, H]
    sz[kBwDOG] = S * act_pitch(2L * H);  // w_a dy per slot [S, H]
    sz[kBwDGU] = S * act_pitch(4L * F);  // dg|du [S, 2F]
    sz[kBwDW] = 4 * (size_t)B.fwd.A;     // routing-weight gradients
    size_t off = B.fwd.total;
    for (int r = 0; r < kBwRegions; ++r) {
        B.off[r] = off;
        off = align_up(off + sz[r], 1024);
    }
    B.total = off;
    return B;
}

bool bwd_dims_ok(int T, int H, int F, int E, int k) {
    return dims_ok(T, H, F, E, k, MOE_BF16) && H % 128 == 0 && F % 128 == 0;
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

enum TrainPart { kTrainForward = 0, kTrainBackwardSaved = 1, kTrainBackward = 2 };

// The training forward and the two forms of the backward share one workspace
// layout.  kTrainForward: routing, x gathered into the slot layout, g/u/h
// (kept for the backward), the second GEMM with the weighted combine, the bf16
// output.  kTrainBackwardSaved: the backward from what the forward kept.
// kTrainBackward: the backward with its own routing and g/u/h recompute.
int train_impl(int part, const void* x, const float* logits, const void* w1, const void* w3, const void* w2,
               const void* dy, int T, int H, int F, int E, int k, void* out, void* dx, void* dw1, void* dw3,
               void* dw2, float* dlogits, void* ws, size_t ws_bytes, void* stream) {
    const bool fwd = part == kTrainForward;
    const bool bwd = !fwd;
    const bool recompute = part == kTrainBackward;
    if (!bwd_dims_ok(T, H, F, E, k)) return MOE_ERR_INVALID_ARG;
    if (!w1 || !w3 || !w2 || !ws || (bwd && (!dw1 || !dw3 || !dw2))) return MOE_ERR_INVALID_ARG;
    if (T > 0 && ((part != kTrainBackwardSaved && (!x || !logits)) || (fwd && !out) || (bwd && (!dy || !dx || !dlogits))))
        return MOE_ERR_INVALID_ARG;
    for (const void* ptr : {w1, w3, w2, (const void*)ws})
        if (!aligned16(ptr)) return MOE_ERR_ALIGNMENT;
    if (bwd)
        for (const void* ptr : {(const void*)dw1, (const void*)dw3, (const void*)dw2})
            if (!aligned16(ptr)) return MOE_ERR_ALIGNMENT;
    if (T > 0) {
        if (part != kTrainBackwardSaved && (!aligned16(x) || !aligned4(logits))) return MOE_ERR_ALIGNMENT;
        if (fwd && !aligned16(out)) return MOE_ERR_ALIGNMENT;
        if (bwd && (!aligned16(dy) || !aligned16(dx) || !aligned4(dlogits))) return MOE_ERR_ALIGNMENT;
    }
    const BwdLayout B = make_bwd_layout(T, H, F, E, k);
    const Layout& L = B.fwd;
    if (ws_bytes < B.total) return MOE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) {  // no tokens: nothing to compute; every weight gradient is zero
        if (fwd) return MOE_OK;
        const size_t n = (size_t)E * F * H * 2;
        if (cudaMemsetAsync(dw1, 0, n, st) != cudaSuccess || cudaMemsetAsync(dw3, 0, n, st) != cudaSuccess ||
            cudaMemsetAsync(dw2, 0, n, st) != cudaSuccess)
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    CtxInfo ctx{};
    if (context_info(&ctx) != MOE_OK) return MOE_ERR_CUDA;
    int* status = ctx.status;
    const int num_sms = ctx.num_sms;
    uint8_t* w = static_cast<uint8_t*>(ws);
    auto reg = [&](int r) { return w + L.off[r]; };
    auto breg = [&](int r) { return w + B.off[r]; };
    const int S = L.S_max;
    const unsigned long long timeout_ns = (unsigned long long)g_opt_timeout_ms.load() * 1000000ull;
    const long p2H = act_pitch(2L * H), p4F = act_pitch(4L * F), p2F = act_pitch(2L * F), p8F = act_pitch(8L * F);

    RouteOutputs o{reinterpret_cast<int32_t*>(reg(MOE_WS_TOPK_IDS)), reinterpret_cast<float*>(reg(MOE_WS_TOPK_W)),
                   reinterpret_cast<int32_t*>(reg(MOE_WS_COUNTS)), reinterpret_cast<int32_t*>(reg(MOE_WS_OFFSETS)),
                   reinterpret_cast<int32_t*>(reg(MOE_WS_PERM)), reinterpret_cast<int32_t*>(reg(MOE_WS_INV_PERM)),
                   reinterpret_cast<int32_t*>(reg(MOE_WS_SLOT_OF)), reinterpret_cast<int32_t*>(reg(MOE_WS_SLOT_ASSIGN)),
                   reinterpret_cast<int32_t*>(reg(MOE_WS_MTILE_EXPERT)),
                   reinterpret_cast<int32_t*>(reg(MOE_WS_NUM_MTILES)),
                   reinterpret_cast<int32_t*>(reg(MOE_WS_ROUTE_BLOCKS))};
    float* rows32 = reinterpret_cast<float*>(reg(MOE_WS_OUT32));  // the forward's combine, or dx32
    float* dwa = reinterpret_cast<float*>(breg(kBwDW));

    // 1. routing (the backward from saved activations reuses the forward's),
    // and the slot gather: x (forward, recompute) and dy, w_a dy (backward)
    {
        ProfScope ps(fwd ? MOE_KERNEL_ROUTE : MOE_KERNEL_BWD_AUX, st, part == kTrainBackwardSaved ? 0 : route_launches(T, o));
        if (part != kTrainBackwardSaved && launch_route(logits, T, E, k, o, st) != cudaSuccess) return MOE_ERR_CUDA;
    }
    // failure-detection test hook (as in the forward): one routing-table entry
    // overwritten with an index far out of range after the routing
    const int corrupt = g_opt_test_corrupt.load();
    if (corrupt && part != kTrainBackwardSaved) {
        void* target = corrupt == 1 ? (void*)o.slot_assign : corrupt == 2 ? (void*)o.mtile_expert : (void*)o.num_mtiles;
        if (cudaMemsetAsync(target, 0x7F, sizeof(int32_t), st) != cudaSuccess) return MOE_ERR_CUDA;
    }
    {
        ProfScope ps(fwd ? MOE_KERNEL_QUANT : MOE_KERNEL_BWD_AUX, st);
        SlotGatherArgs g{};
        g.x = part == kTrainBackwardSaved ? nullptr : static_cast<const __nv_bfloat16*>(x);
        g.dy = bwd ? static_cast<const __nv_bfloat16*>(dy) : nullptr;
        g.num_mtiles = o.num_mtiles;
        g.mt_max = L.MT_max;
        g.slot_assign = o.slot_assign;
        g.topk_w = o.topk_w;
        g.num_assign = L.A;
        g.topk = k;
        g.H = H;
        g.pitch = p2H / 2;
        g.xg = reinterpret_cast<__nv_bfloat16*>(reg(MOE_WS_XG));
        g.dyg = reinterpret_cast<__nv_bfloat16*>(breg(kBwDYG));
        g.dog = reinterpret_cast<__nv_bfloat16*>(breg(kBwDOG));
        g.status = status;
        if (launch_slot_gather(g, S, st) != cudaSuccess) return MOE_ERR_CUDA;
        if (cudaMemsetAsync(rows32, 0, (size_t)T * H * 4, st) != cudaSuccess) return MOE_ERR_CUDA;
        if (bwd && cudaMemsetAsync(dwa, 0, (size_t)L.A * 4, st) != cudaSuccess) return MOE_ERR_CUDA;
    }

    // tensor maps: 64-element x 128-row boxes for K-major operands, 64 x 64
    // for MN-major ones (all bf16, 128-byte swizzle)
    CUtensorMap mXg, mW1, mW3, mH, mW2k, mDyg, mW2mn, mDgu, mW1mn, mW3mn, mDogmn, mHmn, mDgumn, mXgmn;
    if (!make_map(&mXg, reg(MOE_WS_XG), S, H, p2H, 2, 128) ||
        !make_map(&mW1, w1, (size_t)E * F, H, (size_t)H * 2, 2, 128) ||
        !make_map(&mW3, w3, (size_t)E * F, H, (size_t)H * 2, 2, 128))
        return MOE_ERR_CUDA;
    if (fwd && (!make_map(&mH, reg(MOE_WS_H), S, F, p2F, 2, 128) ||
                !make_map(&mW2k, w2, (size_t)E * H, F, (size_t)F * 2, 2, 128)))
        return MOE_ERR_CUDA;
    if (bwd && (!make_map(&mDyg, breg(kBwDYG), S, H, p2H, 2, 128) ||
                !make_map(&mW2mn, w2, (size_t)E * H, F, (size_t)F * 2, 2, 64) ||
                !make_map(&mDgu, breg(kBwDGU), S, 2L * F, p4F, 2, 128) ||
                !make_map(&mW1mn, w1, (size_t)E * F, H, (size_t)H * 2, 2, 64) ||
                !make_map(&mW3mn, w3, (size_t)E * F, H, (size_t)H * 2, 2, 64) ||
                !make_map(&mDogmn, breg(kBwDOG), S, H, p2H, 2, 64) ||
                !make_map(&mHmn, reg(MOE_WS_H), S, F, p2F, 2, 64) ||
                !make_map(&mDgumn, breg(kBwDGU), S, 2L * F, p4F, 2, 64) ||
                !make_map(&mXgmn, reg(MOE_WS_XG), S, H, p2H, 2, 64)))
        return MOE_ERR_CUDA;

    BwdArgs base{};
    base.num_mtiles = o.num_mtiles;
    base.mtile_expert = o.mtile_expert;
    base.slot_assign = o.slot_assign;
    base.counts = o.counts;
    base.topk_w = o.topk_w;
    base.num_experts = E;
    base.mt_max = L.MT_max;
    base.topk = k;
    base.T = T;
    base.F = F;
    base.timeout_ns = timeout_ns;
    base.status = status;
    // one CTA per SM at most; pairs: whole clusters that can be resident.
    // Pairs wherever the tile is 256 wide (DW: an even number of 128-row
    // output tiles); the pair kernels' residency is looked up once per context.
    const int opt_path = g_opt_path.load();  // 2, 3 or 4: one-SM tiles only
    auto pairs_for = [&](int mode) {
        if (opt_path >= 2) return 0;
        static std::mutex mu;
        static unsigned long long key[5] = {0, 0, 0, 0, 0};
        static int val[5] = {0, 0, 0, 0, 0};
        std::lock_guard<std::mutex> lock(mu);
        if (key[mode] != ctx.ctx_id) {
            val[mode] = bwd_max_pairs(mode);
            key[mode] = ctx.ctx_id;
        }
        return val[mode];
    };
    auto grid_for = [&](int mode, bool pair, long units) {
        if (pair) return (int)(2 * std::max<long>(1, std::min<long>(units, pairs_for(mode))));
        return (int)std::max<long>(1, std::min<long>(units, num_sms));
    };
    const long mt_pairs = (L.MT_max + 1) / 2 + E;  // upper bound of the m-tile pairs over all experts

    // 2. g, u (fp32, kept for the backward) and h = bf16(silu(g) u)
    if (fwd || recompute) {
        BwdArgs a = base;
        a.n_tiles = F / 128;
        a.k_tiles = H / 64;
        a.b_rows = F;
        a.out = breg(kBwGU);
        a.out_pitch = p8F;
        a.out2 = reg(MOE_WS_H);
        a.out2_pitch = p2F;
        const bool pair = pairs_for(kBwdGU) > 0;
        ProfScope ps(fwd ? MOE_KERNEL_STAGE1 : MOE_KERNEL_BWD_GU, st);
        if (launch_bwd_gemm(kBwdGU, 256, pair, mXg, mW1, mW3, a,
                            grid_for(kBwdGU, pair, (pair ? mt_pairs : L.MT_max) * a.n_tiles), st) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    if (fwd) {
        // 3. the forward's second GEMM: w_a (h . W2_e^T) added into the token's fp32 row, then bf16
        const int bn = (H % 256 == 0) ? 256 : 128;
        BwdArgs a = base;
        a.n_tiles = H / bn;
        a.k_tiles = F / 64;
        a.b_rows = H;
        a.out = rows32;
        a.out_pitch = (long)H * 4;
        const bool pair = bn == 256 && pairs_for(kFwdW2) > 0;
        {
            ProfScope ps(MOE_KERNEL_STAGE2, st);
            if (launch_bwd_gemm(kFwdW2, bn, pair, mH, mW2k, mW2k, a,
                                grid_for(kFwdW2, pair, (pair ? mt_pairs : L.MT_max) * a.n_tiles), st) != cudaSuccess)
                return MOE_ERR_CUDA;
        }
        ProfScope ps(MOE_KERNEL_FINALIZE, st);
        return launch_status(launch_finalize(rows32, static_cast<__nv_bfloat16*>(out), (size_t)T * H, num_sms, st));
    }
    // 3. dh = w_a W2^T dy -> dg, du and the routing-weight gradients
    {
        const int bn = (F % 256 == 0) ? 256 : 128;
        BwdArgs a = base;
        a.n_tiles = F / bn;
        a.k_tiles = H / 64;
        a.b_rows = H;
        a.out = breg(kBwDGU);
        a.out_pitch = p4F;
        a.gu = breg(kBwGU);
        a.gu_pitch = p8F;
        a.hbuf = reg(MOE_WS_H);
        a.h_pitch = p2F;
        a.dw = dwa;
        const bool pair = bn == 256 && pairs_for(kBwdDH) > 0;
        ProfScope ps(MOE_KERNEL_BWD_DH, st);
        if (launch_bwd_gemm(kBwdDH, bn, pair, mDyg, mW2mn, mW2mn, a,
                            grid_for(kBwdDH, pair, (pair ? mt_pairs : L.MT_max) * a.n_tiles), st) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    // 4. dx: the k experts' contributions meet in fp32, then one rounding
    {
        const int bn = (H % 256 == 0) ? 256 : 128;
        BwdArgs a = base;
        a.n_tiles = H / bn;
        a.k_tiles = 2 * F / 64;
        a.out = rows32;
        a.out_pitch = (long)H * 4;
        const bool pair = bn == 256 && pairs_for(kBwdDX) > 0;
        ProfScope ps(MOE_KERNEL_BWD_DX, st);
        if (launch_bwd_gemm(kBwdDX, bn, pair, mDgu, mW1mn, mW3mn, a,
                            grid_for(kBwdDX, pair, (pair ? mt_pairs : L.MT_max) * a.n_tiles), st) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    {
        ProfScope ps(MOE_KERNEL_BWD_AUX, st);
        if (launch_finalize(rows32, static_cast<__nv_bfloat16*>(dx), (size_t)T * H, num_sms, st) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    // 5. dW2_e = (w dy)^T h and [dW1_e; dW3_e] = [dg; du]^T x over each expert's slots
    {
        const int bn = (F % 256 == 0) ? 256 : 128;
        BwdArgs a = base;
        a.m_tiles = H / 128;
        a.n_tiles = F / bn;
        a.out = dw2;
        a.out2 = dw2;
        a.out_pitch = (long)F * 2;
        a.split = H;
        a.expert_stride = (long)H * F * 2;
        a.n_fast = H > F ? 1 : 0;
        const bool pair = bn == 256 && a.m_tiles % 2 == 0 && pairs_for(kBwdDW) > 0;
        const long units = (long)E * (pair ? a.m_tiles / 2 : a.m_tiles) * a.n_tiles;
        ProfScope ps(MOE_KERNEL_BWD_DW2, st);
        if (launch_bwd_gemm(kBwdDW, bn, pair, mDogmn, mHmn, mHmn, a, grid_for(kBwdDW, pair, units), st) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    {
        const int bn = (H % 256 == 0) ? 256 : 128;
        BwdArgs a = base;
        a.m_tiles = 2 * F / 128;
        a.n_tiles = H / bn;
        a.out = dw1;
        a.out2 = dw3;
        a.out_pitch = (long)H * 2;
        a.split = F;
        a.expert_stride = (long)F * H * 2;
        a.n_fast = 2 * F > H ? 1 : 0;  // dg|du (2F columns) is read once, x's H columns from L2
        const bool pair = bn == 256 && a.m_tiles % 2 == 0 && pairs_for(kBwdDW) > 0;
        const long units = (long)E * (pair ? a.m_tiles / 2 : a.m_tiles) * a.n_tiles;
        ProfScope ps(MOE_KERNEL_BWD_DW13, st);
        if (launch_bwd_gemm(kBwdDW, bn, pair, mDgumn, mXgmn, mXgmn, a, grid_for(kBwdDW, pair, units), st) !=
            cudaSuccess)
            return MOE_ERR_CUDA;
    }
    // 6. router
    {
        ProfScope ps(MOE_KERNEL_BWD_AUX, st);
        if (launch_dlogits(o.topk_ids, o.topk_w, dwa, T, E, k, dlogits, st) != cudaSuccess) return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

}  // namespace

extern "C" {

size_t moe_backward_workspace_size(int T, int H, int F, int E, int k) {
    if (!bwd_dims_ok(T, H, F, E, k)) return 0;
    return make_bwd_layout(T, H, F, E, k).total;
}

int moe_ffn_forward_train(const void* x, const float* logits, const void* w1, const void* w3, const void* w2, int T,
                          int H, int F, int E, int k, void* out, void* ws, size_t ws_bytes, void* stream) {
    return train_impl(kTrainForward, x, logits, w1, w3, w2, nullptr, T, H, F, E, k, out, nullptr, nullptr, nullptr,
                      nullptr, nullptr, ws, ws_bytes, stream);
}

int moe_ffn_backward_saved(const void* w1, const void* w3, const void* w2, const void* dy, int T, int H, int F, int E,
                           int k, void* dx, void* dw1, void* dw3, void* dw2, float* dlogits, void* ws, size_t ws_bytes,
                           void* stream) {
    return train_impl(kTrainBackwardSaved, nullptr, nullptr, w1, w3, w2, dy, T, H, F, E, k, nullptr, dx, dw1, dw3,
                      dw2, dlogits, ws, ws_bytes, stream);
}

int moe_ffn_backward(const void* x, const float* logits, const void* w1, const void* w3, const void* w2,
                     const void* dy, int T, int H, int F, int E, int k, void* dx, void* dw1, void* dw3, void* dw2,
                     float* dlogits, void* ws, size_t ws_bytes, void* stream) {
    return train_impl(kTrainBackward, x, logits, w1, w3, w2, dy, T, H, F, E, k, nullptr, dx, dw1, dw3, dw2, dlogits,
                      ws, ws_bytes, stream);
}

}  // extern "C"
