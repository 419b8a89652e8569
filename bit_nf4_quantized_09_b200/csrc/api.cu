// C ABI of libqlora_nf4.so: argument checks, workspace layout, TMA tensor
// maps and the launch sequence of each call. All compute happens in the
// kernels of quantize.cu, gemm_fused.cu and gemm_skinny.cu.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/qlora_nf4.h"
#include "kernels.h"

using namespace qlora;

namespace {

// ------------------------------------------------------------ options ----
std::atomic<int64_t> g_small_m_max{16};
std::atomic<int64_t> g_fail_launches{0};
std::atomic<int64_t> g_timeout_us{1000000};
std::atomic<int64_t> g_stall_producer{0};
std::atomic<int64_t> g_launch_count{0};
std::atomic<int64_t> g_skinny_max_splits{0};
thread_local std::string g_last_error;

// One-shot event requests of qlora_profile_next_launch, per kernel id.
std::mutex g_prof_mu;
cudaEvent_t g_prof_events[3][2] = {};

void take_profile_events(int kernel, cudaEvent_t* start, cudaEvent_t* stop) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    *start = g_prof_events[kernel][0];
    *stop = g_prof_events[kernel][1];
    g_prof_events[kernel][0] = g_prof_events[kernel][1] = nullptr;
}

qlora_status cuda_fail(cudaError_t e, const char* where) {
    g_last_error = std::string(where) + ": " + cudaGetErrorString(e);
    // a launch refused for its configuration also sets the thread's last
    // error; read it here so that later launches checked through
    // cudaGetLastError do not report it again
    (void)cudaGetLastError();
    return QLORA_ERR_CUDA;
}

#define QLORA_TRY(expr, where)                          \
    do {                                                \
        cudaError_t e_ = (expr);                        \
        if (e_ != cudaSuccess) return cuda_fail(e_, where); \
    } while (0)

// A launch of `nkernels` kernels of this library.
#define QLORA_LAUNCH(expr, nkernels, where)             \
    do {                                                \
        cudaError_t e_ = (expr);                        \
        if (e_ != cudaSuccess) return cuda_fail(e_, where); \
        g_launch_count += (nkernels);                   \
    } while (0)


// Host-side fault injection: consumes one "launch" and reports a failure
// before anything reaches the GPU.
bool injected_failure() {
    int64_t n = g_fail_launches.load();
    while (n > 0) {
        if (g_fail_launches.compare_exchange_weak(n, n - 1)) {
            g_last_error = "injected launch failure";
            return true;
        }
    }
    return false;
}

// ------------------------------------------------------------ NF4 tables --
// Independent host computation of the levels (normal quantiles by Newton's
// method on Phi) and of the decision thresholds: for each neighbour pair the
// exact midpoint rounded toward -infinity to fp32, so that "v > threshold"
// means "v is strictly nearer the upper level" and an exact tie stays below.
double std_normal_quantile(double p) {
    // Phi is concave on x >= 0, so Newton's method from x = 0 climbs
    // monotonically to the root for p > 1/2.
    double x = 0.0;
    for (int i = 0; i < 200; ++i) {
        const double f = 0.5 * std::erfc(-x / std::sqrt(2.0)) - p;
        const double d = std::exp(-0.5 * x * x) / std::sqrt(2.0 * M_PI);
        const double nx = x - f / d;
        if (nx == x) break;
        x = nx;
    }
    return x;
}

Nf4Tables build_tables() {
    Nf4Tables t{};
    const double top = 0.9677083;
    double v[16];
    int n = 0;
    for (int k = 0; k < 8; ++k) v[n++] = std_normal_quantile(top - k * ((top - 0.5) / 8.0));   // 8 positive
    for (int k = 0; k < 7; ++k) v[n++] = -std_normal_quantile(top - k * ((top - 0.5) / 7.0));  // 7 negative
    v[n++] = 0.0;                                                                           // exact zero
    std::sort(v, v + 16);
    for (int k = 0; k < 16; ++k) t.level[k] = static_cast<float>(v[k] / v[15]);
    for (int k = 0; k < 15; ++k) {
        const double mid = (static_cast<double>(t.level[k]) + static_cast<double>(t.level[k + 1])) * 0.5;
        float f = static_cast<float>(mid);
        if (static_cast<double>(f) > mid) f = std::nextafter(f, -INFINITY);
        t.thresh[k] = f;
    }
    return t;
}

const Nf4Tables& tables() {
    static const Nf4Tables t = build_tables();
    return t;
}

// ------------------------------------------------------------- devices ----
struct DeviceState {
    bool ready = false;
    qlora_status status = QLORA_OK;
    int sms = 0;
};
std::mutex g_dev_mu;
DeviceState g_dev[64];

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Checks the current device once (sm_100, 148-SM class) and opts the big
// kernels in to their shared-memory sizes.
qlora_status device_ready(int* sms_out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) return QLORA_ERR_UNSUPPORTED_DEVICE;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceState& d = g_dev[dev];
    if (!d.ready) {
        d.ready = true;
        int major = 0, minor = 0;
        if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) {
            d.status = cuda_fail(e, "cudaDeviceGetAttribute");
        } else if (major != 10 || minor != 0) {
            g_last_error = "device is not sm_100 (compute capability " + std::to_string(major) + "." +
                           std::to_string(minor) + ")";
            d.status = QLORA_ERR_UNSUPPORTED_DEVICE;
        } else if ((e = fused_init_device()) != cudaSuccess || (e = skinny_init_device()) != cudaSuccess ||
                   (e = gemv_mma_init_device()) != cudaSuccess || (e = merge_tc_init_device()) != cudaSuccess) {
            d.status = cuda_fail(e, "cudaFuncSetAttribute");
        } else if (!g_encode) {
            void* fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q);
            if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
                d.status = cuda_fail(e == cudaSuccess ? cudaErrorSymbolNotFound : e, "cuTensorMapEncodeTiled");
            else
                g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        }
    }
    if (sms_out) *sms_out = d.sms;
    return d.status;
}

// Recently encoded tensor maps, keyed by everything that goes into one, so a
// caller that reuses its buffers pays for cuTensorMapEncodeTiled once.
struct MapKey {
    const void* base;
    uint64_t d0, d1, row_bytes;
    uint32_t b0, b1;
    int dt, sw;
    bool operator==(const MapKey& o) const {
        return base == o.base && d0 == o.d0 && d1 == o.d1 && row_bytes == o.row_bytes && b0 == o.b0 && b1 == o.b1 &&
               dt == o.dt && sw == o.sw;
    }
};
constexpr int kMapCacheSize = 64;
std::mutex g_map_mu;
MapKey g_map_keys[kMapCacheSize];
CUtensorMap g_map_vals[kMapCacheSize];
bool g_map_used[kMapCacheSize] = {};
int g_map_next = 0;

// 2-D tiled tensor map over a row-major [d1, d0] array (d0 contiguous).
qlora_status make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1,
                      uint64_t row_bytes, uint32_t b0, uint32_t b1, CUtensorMapSwizzle sw, const char* what) {
    const MapKey key{base, d0, d1, row_bytes, b0, b1, static_cast<int>(dt), static_cast<int>(sw)};
    {
        std::lock_guard<std::mutex> lk(g_map_mu);
        for (int i = 0; i < kMapCacheSize; ++i)
            if (g_map_used[i] && g_map_keys[i] == key) {
                *m = g_map_vals[i];
                return QLORA_OK;
            }
    }
    const cuuint64_t dims[2] = {d0, d1};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {b0, b1};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        g_last_error = std::string("cuTensorMapEncodeTiled(") + what + ") failed: " + std::to_string(r);
        return QLORA_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lk(g_map_mu);
    g_map_keys[g_map_next] = key;
    g_map_vals[g_map_next] = *m;
    g_map_used[g_map_next] = true;
    g_map_next = (g_map_next + 1) % kMapCacheSize;
    return QLORA_OK;
}

#define QLORA_MAP(...)                            \
    do {                                          \
        qlora_status s_ = make_map(__VA_ARGS__);  \
        if (s_ != QLORA_OK) return s_;            \
    } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t up256(size_t x) { return (x + 255) & ~size_t(255); }
inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

bool rank_ok(int r) { return r == 8 || r == 16 || r == 32 || r == 64; }

// Reduction splits of a skinny matmul: the CTAs of a row tile form a cluster
// of S = 1, 2, 4 or 8 that reduces in distributed shared memory; S doubles
// while the launch stays within about two CTAs per SM of a 148-SM B200 and
// every split keeps a reduction step. Four 24 KB stages (two CTAs per SM).
constexpr int64_t kTargetCtas = 296;
constexpr int kPlanSms = 148;  // the SM count the split plans are tuned for (any count runs them)
constexpr int kSkinnyStagesUsed = 4;
constexpr int kSkinnyChunksUsed = 1;
int skinny_splits(int64_t tiles, int64_t red);

// Whole output tiles (at least as many as SMs) and at least two row tiles:
// the fused matmuls may run in CTA pairs that share each dequantised weight
// tile (the workspace then holds partial tiles for a stream-K tail).
bool pairs_possible(int64_t M, int64_t tiles_n) {
    const int64_t tiles_m = cdiv(M, kFusedBM);
    return tiles_m >= 2 && tiles_m * tiles_n >= kPlanSms;
}


// ------------------------------------------------------- the low-rank side --
// The adapter side of a forward or backward call. One adapter (P = 1);
// several adapters over one frozen base, each token row using the one its id
// names (ids set; rank R = P r, adapter k in columns [k r, (k + 1) r) of the
// rank-r inputs); or the projections of a group, which share the input and
// sit side by side in the output (group set; projection i in columns
// [i r, (i + 1) r)).
struct Lora {
    int r = 0;
    int P = 1;
    bool group = false;
    const int* ids = nullptr;
    int R() const { return r * P; }
    // 64-column chunks of the concatenated rank-r inputs
    int chunks() const { return static_cast<int>((R() + 63) / 64); }
    // problems of the backward down-projection (a group: one per projection)
    int down_bwd() const { return group ? P : chunks(); }
    // problems of dB (a group: one per projection)
    int grad_b() const { return group ? P : chunks(); }
};

constexpr int kMaxMultiRank = 256;  // P r of several adapters: four 64-column chunks

// A weight, or the weights of a group read as one weight of sum(N_i) rows,
// whose codes lie back to back in one buffer.
struct Weights {
    const qlora_nf4_weight* w = nullptr;
    int P = 1;
    int64_t N = 0, K = 0;
    int64_t off[kMaxGroups + 1] = {};  // first row of each weight; off[P] = N
    int64_t rows(int i) const { return off[i + 1] - off[i]; }
};

// ------------------------------------------------------- workspace layout --
// Head of every fwd/bwd workspace: the device status word, then the tickets
// of the small-batch kernel and the stream-K flags of the fused matmuls;
// cleared by one memset at the start of each call (the kernels also leave
// their tickets at zero).
struct Layout {
    size_t header = 0;                                   // bytes cleared per call
    size_t status = 0, ctrY = 0, flags = 0;
    size_t skpart = 0;                                    // fused matmul: partial tiles of stream-K contributors
    size_t cT = 0, cflat = 0, sT = 0, partY = 0;  // forward
    size_t sU = 0;                                // backward
    size_t total = 0;
    int64_t ldc = 0;
    GemvMmaPlan reg_gemv{1, 1, 2, 1};
};

// UMMA N of a rank-r problem of `w` columns (at most 64).
int rank_pad(int w) { return w <= 16 ? 16 : (w <= 32 ? 32 : 64); }

// Column tiles of the fused forward: 256-column tiles per weight of a group.
int64_t fwd_tiles_n(const Weights& W, bool group) {
    if (!group) return cdiv(W.N, 256);
    int64_t t = 0;
    for (int i = 0; i < W.P; ++i) t += cdiv(W.rows(i), 256);
    return t;
}

Layout layout_for(int op, int64_t M, const Weights& W, const Lora& lo) {
    Layout L;
    const int64_t N = W.N, K = W.K;
    const int R = lo.R();
    L.ldc = (N + 3) / 4 * 4;  // constants row pitch: a multiple of 16 bytes
    const int64_t ntiles = cdiv(N, 128);
    L.status = 0;
    L.ctrY = 256;
    L.flags = L.ctrY + 4 * static_cast<size_t>(ntiles);
    L.header = up256(L.flags + 4 * static_cast<size_t>(kPlanSms));
    size_t off = L.header;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += up256(bytes);
        return at;
    };
    L.cT = take(static_cast<size_t>(K / kBlock) * L.ldc * 4);
    // the fused matmul's partial tiles, one per CTA, when it splits tiles
    const bool fwd = op == QLORA_OP_FWD;
    const int64_t tiles_n = fwd ? fwd_tiles_n(W, lo.group) : cdiv(K, 256);
    const int64_t part_ctas = pairs_possible(M, tiles_n) ? kPlanSms : fused_partial_ctas(M, tiles_n, fwd ? K : N, kPlanSms);
    L.skpart = take(static_cast<size_t>(part_ctas) * kFusedBM * kFusedBN * 4);
    L.sT = take(static_cast<size_t>(M) * R * 2);
    if (fwd) {
        if (M <= kGemvMmaMaxM) {
            // the small-batch kernel may run (its token limit is a runtime option)
            L.reg_gemv = gemv_mma_plan(M, N, K, kPlanSms);
            L.partY = take(static_cast<size_t>(L.reg_gemv.max_parts) * M * N * 4);
            // a group's block constants decoded in block order for the
            // register-fed kernel (its weights keep their own mean and s2)
            if (lo.group) L.cflat = take(static_cast<size_t>(N * K / kBlock) * 4);
        }
    } else {
        L.sU = take(static_cast<size_t>(M) * R * 2);
    }
    L.total = off;
    return L;
}

// A profiling event record; inside stream capture it becomes an external
// event-record node, so it also times every replay of the captured graph.
cudaError_t record_profile_event(cudaEvent_t ev, cudaStream_t st) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    const cudaError_t e = cudaStreamIsCapturing(st, &cs);
    if (e != cudaSuccess) return e;
    return cs == cudaStreamCaptureStatusActive ? cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal)
                                               : cudaEventRecord(ev, st);
}

// A weight stored with double quantisation needs qabsmax, s2 and mean; one
// stored without it (absmax set) needs only its fp32 constants.
qlora_status check_weight(const qlora_nf4_weight* w) {
    if (!w || !w->codes) return QLORA_ERR_INVALID_ARG;
    if (!w->absmax && (!w->qabsmax || !w->s2 || !w->mean)) return QLORA_ERR_INVALID_ARG;
    if (w->N <= 0 || w->K <= 0 || w->K % kBlock != 0 || w->N % 8 != 0) return QLORA_ERR_BAD_SHAPE;
    if (!aligned16(w->codes)) return QLORA_ERR_MISALIGNED;
    if (w->absmax) return aligned16(w->absmax) ? QLORA_OK : QLORA_ERR_MISALIGNED;
    if (!aligned16(w->qabsmax) || !aligned16(w->s2) || (reinterpret_cast<uintptr_t>(w->mean) & 3u))
        return QLORA_ERR_MISALIGNED;
    return QLORA_OK;
}

// The weights of a call: one, or the P weights of a group, which must share
// K and the storage form and keep their codes back to back in one buffer.
qlora_status check_weights(const qlora_nf4_weight* w, int P, Weights* out) {
    if (!w || P < 1 || P > kMaxGroups) return QLORA_ERR_INVALID_ARG;
    out->w = w;
    out->P = P;
    out->K = w[0].K;
    out->off[0] = 0;
    for (int i = 0; i < P; ++i) {
        const qlora_status s = check_weight(w + i);
        if (s != QLORA_OK) return s;
        if (w[i].K != out->K) return QLORA_ERR_BAD_SHAPE;
        if ((w[i].absmax == nullptr) != (w[0].absmax == nullptr)) {
            g_last_error = "the weights of a group must all use the same storage (with or without double quantisation)";
            return QLORA_ERR_INVALID_ARG;
        }
        if (i > 0 && w[i].codes != w[i - 1].codes + w[i - 1].N * w[i - 1].K / 2) {
            g_last_error = "the codes of the weights of a group must lie back to back in one buffer";
            return QLORA_ERR_INVALID_ARG;
        }
        out->off[i + 1] = out->off[i] + w[i].N;
    }
    out->N = out->off[P];
    return QLORA_OK;
}

BlockConstants constants_of(const qlora_nf4_weight* w) {
    if (w->absmax) return BlockConstants{nullptr, nullptr, nullptr, w->absmax};
    return BlockConstants{w->qabsmax, w->s2, w->mean, nullptr};
}

uint64_t timeout_ns() { return static_cast<uint64_t>(std::max<int64_t>(1, g_timeout_us.load())) * 1000ull; }

CUtensorMapSwizzle swizzle_for_rank(int NR) {
    return NR == 16 ? CU_TENSOR_MAP_SWIZZLE_32B : (NR == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
}

// Map of `cols` columns of a row-major bf16 matrix of `rows` rows and row
// pitch `ld` elements, starting at `base`, read as MN-major [64 rows, NR
// columns] tiles (B, sU, sT and their chunks); columns past `cols` read as
// zeros.
qlora_status make_rank_map(CUtensorMap* m, const uint16_t* base, int64_t rows, int cols, int64_t ld, int NR,
                           const char* what) {
    return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, cols, rows, static_cast<uint64_t>(ld) * 2, NR, 64,
                    swizzle_for_rank(NR), what);
}

int skinny_splits(int64_t tiles, int64_t red) {
    const int64_t KT = std::max<int64_t>(1, cdiv(red, 64));
    int64_t cap = g_skinny_max_splits.load();
    if (cap <= 0 || cap > 8) cap = 8;
    int64_t s = 1;
    while (2 * s <= cap && std::max<int64_t>(tiles, 1) * 2 * s <= kTargetCtas && 2 * s * kSkinnyChunksUsed <= KT)
        s *= 2;
    return static_cast<int>(s);
}

SkinnyProblem skinny_problem(int64_t rows, int64_t red, int a_mn, int b_mn, int mode, int ncols, int64_t out_ld) {
    SkinnyProblem p{};
    p.rows = rows;
    p.red = red;
    p.a_mn_major = a_mn;
    p.b_mn_major = b_mn;
    p.mode = mode;
    p.ncols = ncols;
    p.out_ld = out_ld;
    p.scale = 1.0f;
    return p;
}

// sT = bf16(s X A^T) [M, R] in 64-column chunks (one skinny problem each);
// with row ids, the columns of every adapter but the row's own are zero.
qlora_status down_fwd(const uint16_t* X, int64_t M, int64_t K, const uint16_t* A, const Lora& lo, float scale,
                      uint16_t* sT, int* status, cudaStream_t st) {
    const int R = lo.R(), nch = lo.chunks(), NR = rank_pad(std::min(R, 64));
    SkinnyMaps maps;
    SkinnyArgs a{};
    a.NR = NR;
    a.splits = skinny_splits(cdiv(M, 128) * nch, K);
    a.stages = kSkinnyStagesUsed;
    a.chunks = kSkinnyChunksUsed;
    CUtensorMap tx;
    QLORA_MAP(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, K, M, K * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B, "X");
    for (int c = 0; c < nch; ++c) {
        const int w = std::min(64, R - 64 * c);
        maps.a[c] = tx;
        QLORA_MAP(&maps.b[c], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A + static_cast<int64_t>(64 * c) * K, K, w, K * 2, 64,
                  NR, CU_TENSOR_MAP_SWIZZLE_128B, "A");
        SkinnyProblem& p = a.p[c];
        p = skinny_problem(M, K, 0, 0, kSkinnyOutBf16, w, R);
        p.scale = scale;
        p.out_bf16 = sT + 64 * c;
        p.row_ids = lo.ids;
        p.ids_col0 = 64 * c;
        p.ids_r = lo.r;
    }
    a.status = status;
    a.timeout_ns = timeout_ns();
    if (injected_failure()) return QLORA_ERR_CUDA;
    QLORA_LAUNCH(launch_skinny(maps, a, nch, st), 1, "skinny(sT)");
    return QLORA_OK;
}

// sU = bf16(s dY B) [M, R]: 64-column chunks of B [N, R] (row ids mask as
// above), or for a group one problem per projection, sU_i = s dY_i B_i with
// dY_i the projection's columns of dY and B_i its rows of B [N, r].
qlora_status down_bwd(const uint16_t* dY, int64_t M, const Weights& W, const uint16_t* B, const Lora& lo, float scale,
                      uint16_t* sU, int* status, cudaStream_t st) {
    const int R = lo.R(), np = lo.down_bwd();
    const int NR = lo.group ? rank_pad(lo.r) : rank_pad(std::min(R, 64));
    const int64_t N = W.N;
    int64_t red_max = 0;
    for (int c = 0; c < np; ++c) red_max = std::max(red_max, lo.group ? W.rows(c) : N);
    SkinnyMaps maps;
    SkinnyArgs a{};
    a.NR = NR;
    a.splits = skinny_splits(cdiv(M, 128) * np, red_max);
    a.stages = kSkinnyStagesUsed;
    a.chunks = kSkinnyChunksUsed;
    for (int c = 0; c < np; ++c) {
        const int64_t n0 = lo.group ? W.off[c] : 0, red = lo.group ? W.rows(c) : N;
        const int w = lo.group ? lo.r : std::min(64, R - 64 * c);
        QLORA_MAP(&maps.a[c], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dY + n0, red, M, N * 2, 64, 128,
                  CU_TENSOR_MAP_SWIZZLE_128B, "dY");
        qlora_status s = lo.group ? make_rank_map(&maps.b[c], B + n0 * lo.r, red, lo.r, lo.r, NR, "B")
                                  : make_rank_map(&maps.b[c], B + 64 * c, N, w, R, NR, "B");
        if (s != QLORA_OK) return s;
        SkinnyProblem& p = a.p[c];
        p = skinny_problem(M, red, 0, 1, kSkinnyOutBf16, w, R);
        p.scale = scale;
        p.out_bf16 = sU + (lo.group ? c * lo.r : 64 * c);
        p.row_ids = lo.ids;
        p.ids_col0 = 64 * c;
        p.ids_r = lo.r;
    }
    a.status = status;
    a.timeout_ns = timeout_ns();
    if (injected_failure()) return QLORA_ERR_CUDA;
    QLORA_LAUNCH(launch_skinny(maps, a, np, st), 1, "skinny(sU)");
    return QLORA_OK;
}

std::atomic<int64_t> g_fused_pairs{1};
std::atomic<int64_t> g_fused_tail{0};

// The fused launches of a call. CTA pairs take whole waves of tiles; when
// their last wave would be short (at most kTailPercent of the SMs busy) its
// tiles go instead to the one-CTA kernel, split stream-K over every SM and
// launched as the pair launch's programmatic dependent. Without pairs, one
// one-CTA launch over all tiles.
constexpr int64_t kTailPercent = 85;
struct FusedPlan {
    int pair_ctas = 0;                      // CTAs of the pair launch (0: none)
    int64_t tail_first = 0, tail_tiles = 0;  // tiles of the one-CTA launch (pair order; 0 tiles: all)
    int tail_ctas = 0;                      // CTAs of the one-CTA launch (0: none)
};
FusedPlan fused_plan(int64_t M, int64_t tiles_n, int64_t red, int sms) {
    FusedPlan p;
    const int cap = std::min(sms, kPlanSms);
    const int64_t tiles_m = cdiv(M, kFusedBM);
    if (g_fused_pairs.load() == 0 || tiles_m < 2 || tiles_m * tiles_n < cap) {
        p.tail_ctas = fused_ctas(M, tiles_n, red, cap);
        return p;
    }
    const int64_t all = 2 * tiles_n * cdiv(tiles_m, 2);
    const int64_t wave = cap & ~1;
    const int64_t full = all / wave * wave, rest = all - full;
    if (g_fused_tail.load() == 0 || full == 0 || rest == 0 || rest * 100 > wave * kTailPercent ||
        !pairs_possible(M, tiles_n)) {
        p.pair_ctas = static_cast<int>(all);
        return p;
    }
    p.pair_ctas = static_cast<int>(full);
    p.tail_first = full;
    p.tail_tiles = rest;
    p.tail_ctas = fused_ctas_for(rest, red, cap);
    return p;
}

// The projections of a group as column groups of one fused forward; a
// single weight is one group.
void set_groups(FusedArgs* fa, const Weights& W, const Lora& lo) {
    if (!lo.group) {
        fa->ngroups = 1;
        fa->group_end[0] = W.N;
        fa->group_rank_x[0] = 0;
        return;
    }
    fa->ngroups = W.P;
    for (int i = 0; i < W.P; ++i) {
        fa->group_end[i] = W.off[i + 1];
        fa->group_rank_x[i] = i * lo.r;
    }
}

// ------------------------------------------- forward and backward bodies --
// Checks shared by every forward and backward call form.
qlora_status check_lora(const Lora& lo, int64_t M) {
    if (!rank_ok(lo.r)) return QLORA_ERR_UNSUPPORTED_RANK;
    if (lo.P < 1) return QLORA_ERR_INVALID_ARG;
    if (lo.group && lo.P > kMaxGroups) return QLORA_ERR_INVALID_ARG;
    if (lo.R() > kMaxMultiRank) return QLORA_ERR_UNSUPPORTED_RANK;
    if (lo.P > 1 && !lo.group && M > 0 && (!lo.ids || (reinterpret_cast<uintptr_t>(lo.ids) & 3u)))
        return lo.ids ? QLORA_ERR_MISALIGNED : QLORA_ERR_INVALID_ARG;
    return QLORA_OK;
}

// cT (the transposed decoded constants the fused matmuls read): each weight
// of a group at its own column offset.
qlora_status decode_constants_t(const Weights& W, const Layout& L, float* cT, cudaStream_t st) {
    for (int i = 0; i < W.P; ++i) {
        const int64_t cols = i == W.P - 1 ? L.ldc - W.off[i] : W.rows(i);
        QLORA_LAUNCH(launch_decode_constants_t(constants_of(W.w + i), W.rows(i), W.K, L.ldc, cols, cT + W.off[i], st), 1,
                     "decode constants");
    }
    return QLORA_OK;
}

qlora_status fwd_impl(const uint16_t* X, int64_t M, const Weights& W, const uint16_t* A, const uint16_t* B,
                      const Lora& lo, float alpha, uint16_t* Y, uint16_t* sT_save, void* ws, size_t ws_bytes,
                      void* stream) {
    qlora_status s = check_lora(lo, M);
    if (s != QLORA_OK) return s;
    if (M < 0) return QLORA_ERR_BAD_SHAPE;
    if (!std::isfinite(alpha)) return QLORA_ERR_INVALID_ARG;
    if (M == 0) return QLORA_OK;
    if (!X || !A || !B || !Y || !ws) return QLORA_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(Y) || !aligned16(ws) ||
        (sT_save && !aligned16(sT_save)))
        return QLORA_ERR_MISALIGNED;
    const int64_t N = W.N, K = W.K;
    const int r = lo.r, R = lo.R();
    const Layout L = layout_for(QLORA_OP_FWD, M, W, lo);
    if (ws_bytes < L.total) return QLORA_ERR_WORKSPACE_TOO_SMALL;
    if (injected_failure()) return QLORA_ERR_CUDA;
    int sms = 0;
    if ((s = device_ready(&sms)) != QLORA_OK) return s;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* base = static_cast<uint8_t*>(ws);
    int* status = reinterpret_cast<int*>(base + L.status);
    float* cT = reinterpret_cast<float*>(base + L.cT);
    uint16_t* sT = sT_save ? sT_save : reinterpret_cast<uint16_t*>(base + L.sT);
    const float scale = alpha / static_cast<float>(r);

    QLORA_TRY(cudaMemsetAsync(base, 0, L.header, st), "clear status and tickets");
    if (injected_failure()) return QLORA_ERR_CUDA;
    if (M <= std::min<int64_t>(g_small_m_max.load(), kGemvMmaMaxM)) {
        // few tokens: rank-r down-projection, then the weight-streaming
        // small-batch kernel, launched as its programmatic dependent so the
        // weight stream starts while sT is still being computed
        const float* cflat = nullptr;
        if (lo.group) {
            // each weight's block constants, decoded into one array in block order
            cflat = reinterpret_cast<const float*>(base + L.cflat);
            for (int i = 0; i < W.P; ++i)
                QLORA_LAUNCH(launch_decode_constants(constants_of(W.w + i), W.rows(i) * K / kBlock,
                                                     const_cast<float*>(cflat) + W.off[i] * K / kBlock, sms, st),
                             1, "decode constants");
        }
        if ((s = down_fwd(X, M, K, A, lo, scale, sT, status, st)) != QLORA_OK) return s;
        CUtensorMap t_codes, t_x;
        QLORA_MAP(&t_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, W.w[0].codes, K / 2, N, K / 2, 128, 256,
                  CU_TENSOR_MAP_SWIZZLE_128B, "codes");
        QLORA_MAP(&t_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, K, M, K * 2, 64, static_cast<uint32_t>(M),
                  CU_TENSOR_MAP_SWIZZLE_128B, "X");
        GemvMmaArgs ga{};
        ga.qabsmax = W.w[0].qabsmax;
        ga.s2 = W.w[0].s2;
        ga.mean = W.w[0].mean;
        ga.absmax = lo.group ? cflat : W.w[0].absmax;
        ga.M = M;
        ga.N = N;
        ga.K = K;
        ga.rank_cols = lo.group ? r : R;
        ga.sT_ld = R;
        ga.B_ld = lo.group ? r : R;
        ga.ngroups = lo.group ? W.P : 1;
        for (int i = 0; i < ga.ngroups; ++i) {
            ga.group_end[i] = lo.group ? W.off[i + 1] : N;
            ga.group_rank_x[i] = lo.group ? i * r : 0;
        }
        ga.ctas = L.reg_gemv.ctas;
        ga.units = L.reg_gemv.units;
        ga.stages = L.reg_gemv.stages;
        ga.const_vec = (K / kBlock) % 4 == 0 &&
                       (ga.absmax ? reinterpret_cast<uintptr_t>(ga.absmax) % 16 == 0
                                  : reinterpret_cast<uintptr_t>(ga.qabsmax) % 4 == 0);
        ga.part = reinterpret_cast<float*>(base + L.partY);
        ga.counter = reinterpret_cast<int*>(base + L.ctrY);
        ga.sT = sT;
        ga.B = B;
        ga.Y = Y;
        ga.status = status;
        ga.timeout_ns = timeout_ns();
        if (injected_failure()) return QLORA_ERR_CUDA;
        cudaEvent_t ev0, ev1;
        take_profile_events(QLORA_KERNEL_FUSED_FWD, &ev0, &ev1);
        if (ev0) QLORA_TRY(record_profile_event(ev0, st), "profile event");
        // an event record between the two launches would break the
        // programmatic edge, so a profiled call launches in plain order
        QLORA_LAUNCH(launch_gemv_mma(t_codes, t_x, ga, tables(), ev0 == nullptr, st), 1, "register gemv");
        if (ev1) QLORA_TRY(record_profile_event(ev1, st), "profile event");
        return QLORA_OK;
    }
    if ((s = decode_constants_t(W, L, cT, st)) != QLORA_OK) return s;
    if ((s = down_fwd(X, M, K, A, lo, scale, sT, status, st)) != QLORA_OK) return s;

    CUtensorMap t_act, t_codes, t_c, t_lact, t_lw;
    QLORA_MAP(&t_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, K, M, K * 2, 64, 256, CU_TENSOR_MAP_SWIZZLE_128B, "X");
    QLORA_MAP(&t_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, W.w[0].codes, K / 2, N, K / 2, 32, 256,
              CU_TENSOR_MAP_SWIZZLE_32B, "codes");
    QLORA_MAP(&t_c, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, cT, L.ldc, K / kBlock, L.ldc * 4, 256, 1, CU_TENSOR_MAP_SWIZZLE_NONE,
              "constants");
    QLORA_MAP(&t_lact, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, sT, R, M, R * 2, 64, 256, CU_TENSOR_MAP_SWIZZLE_128B, "sT");
    // B [N, R] (one adapter or several side by side), or the stacked B_i [N, r] of a group
    const int bcols = lo.group ? r : R;
    QLORA_MAP(&t_lw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, bcols, N, bcols * 2, 64, 256, CU_TENSOR_MAP_SWIZZLE_128B, "B");
    FusedArgs fa{};
    fa.M = M;
    fa.out_cols = N;
    fa.red = K;
    fa.rank_cols = lo.group ? r : R;
    fa.rank_steps = lo.group ? 1 : lo.chunks();
    set_groups(&fa, W, lo);
    fa.ctas = fused_ctas(M, fused_tiles_n(fa), K, std::min(sms, kPlanSms));
    fa.out = Y;
    fa.part = reinterpret_cast<float*>(base + L.skpart);
    fa.flags = reinterpret_cast<int*>(base + L.flags);
    fa.status = status;
    fa.timeout_ns = timeout_ns();
    fa.stall_producer = static_cast<int>(g_stall_producer.exchange(0));
    if (injected_failure()) return QLORA_ERR_CUDA;
    // whole tiles in CTA pairs that share each dequantised weight tile, the
    // tiles of a short last wave stream-K
    const FusedPlan plan = fused_plan(M, fused_tiles_n(fa), K, sms);
    CUtensorMap h_codes, h_c;
    if (plan.pair_ctas) {
        QLORA_MAP(&h_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, W.w[0].codes, K / 2, N, K / 2, 32, 128,
                  CU_TENSOR_MAP_SWIZZLE_32B, "codes");
        QLORA_MAP(&h_c, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, cT, L.ldc, K / kBlock, L.ldc * 4, 128, 1,
                  CU_TENSOR_MAP_SWIZZLE_NONE, "constants");
    }
    cudaEvent_t ev0, ev1;
    take_profile_events(QLORA_KERNEL_FUSED_FWD, &ev0, &ev1);
    if (ev0) QLORA_TRY(record_profile_event(ev0, st), "profile event");
    // programmatic dependent of the sT launch: the main loop overlaps it
    // (a profiled call keeps plain stream order)
    if (plan.pair_ctas) {
        FusedArgs pa = fa;
        pa.ctas = plan.pair_ctas;
        QLORA_LAUNCH(launch_fused_pair_fwd(t_act, h_codes, h_c, t_lact, t_lw, pa, tables(), ev0 == nullptr, st), 1,
                     "fused forward (pairs)");
    }
    if (plan.tail_ctas) {
        FusedArgs ta = fa;
        ta.ctas = plan.tail_ctas;
        ta.tile_first = plan.tail_first;
        ta.tiles = plan.tail_tiles;
        ta.pair_order = plan.pair_ctas ? 1 : 0;
        ta.stall_producer = plan.pair_ctas ? 0 : fa.stall_producer;
        QLORA_LAUNCH(launch_fused_fwd(t_act, t_codes, t_c, t_lact, t_lw, ta, tables(),
                                      plan.pair_ctas ? true : ev0 == nullptr, st),
                     1, "fused forward");
    }
    if (ev1) QLORA_TRY(record_profile_event(ev1, st), "profile event");
    return QLORA_OK;
}

qlora_status bwd_impl(const uint16_t* dY, const uint16_t* X, int64_t M, const Weights& W, const uint16_t* A,
                      const uint16_t* B, const Lora& lo, float alpha, const uint16_t* sT_in, uint16_t* dX, float* dA,
                      float* dB, void* ws, size_t ws_bytes, void* stream) {
    qlora_status s = check_lora(lo, M);
    if (s != QLORA_OK) return s;
    if (M < 0) return QLORA_ERR_BAD_SHAPE;
    if (!std::isfinite(alpha)) return QLORA_ERR_INVALID_ARG;
    if (!dA || !dB || !A || !B || !ws) return QLORA_ERR_INVALID_ARG;
    if (M > 0 && (!dY || !X || !dX)) return QLORA_ERR_INVALID_ARG;
    if ((M > 0 && (!aligned16(dY) || !aligned16(X) || !aligned16(dX))) || !aligned16(A) || !aligned16(B) ||
        !aligned16(dA) || !aligned16(dB) || !aligned16(ws) || (sT_in && !aligned16(sT_in)))
        return QLORA_ERR_MISALIGNED;
    const int64_t N = W.N, K = W.K;
    const int r = lo.r, R = lo.R();
    const Layout L = layout_for(QLORA_OP_BWD, M, W, lo);
    if (ws_bytes < L.total) return QLORA_ERR_WORKSPACE_TOO_SMALL;
    if (injected_failure()) return QLORA_ERR_CUDA;
    int sms = 0;
    if ((s = device_ready(&sms)) != QLORA_OK) return s;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t dB_cols = lo.group ? r : R;
    if (M == 0) {  // an empty batch: the adapter gradients are exactly zero
        QLORA_TRY(cudaMemsetAsync(dA, 0, static_cast<size_t>(R) * K * 4, st), "zero dA");
        QLORA_TRY(cudaMemsetAsync(dB, 0, static_cast<size_t>(N) * dB_cols * 4, st), "zero dB");
        return QLORA_OK;
    }
    uint8_t* base = static_cast<uint8_t*>(ws);
    int* status = reinterpret_cast<int*>(base + L.status);
    float* cT = reinterpret_cast<float*>(base + L.cT);
    uint16_t* sU = reinterpret_cast<uint16_t*>(base + L.sU);
    const uint16_t* sT = sT_in ? sT_in : reinterpret_cast<uint16_t*>(base + L.sT);
    const float scale = alpha / static_cast<float>(r);
    const int NRc = rank_pad(std::min(R, 64));
    const int nch = lo.chunks(), ndb = lo.grad_b();

    QLORA_TRY(cudaMemsetAsync(base, 0, L.header, st), "clear status and tickets");
    if (injected_failure()) return QLORA_ERR_CUDA;
    if ((s = decode_constants_t(W, L, cT, st)) != QLORA_OK) return s;
    // sU = s dY B, with B read in place (MN-major)
    if ((s = down_bwd(dY, M, W, B, lo, scale, sU, status, st)) != QLORA_OK) return s;
    // sT from the forward, or recomputed
    if (!sT_in) {
        if ((s = down_fwd(X, M, K, A, lo, scale, reinterpret_cast<uint16_t*>(base + L.sT), status, st)) != QLORA_OK)
            return s;
    }

    // dX = dY deq(W) + sU A
    CUtensorMap t_act, t_codes, t_c, t_lact, t_lw;
    QLORA_MAP(&t_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dY, N, M, N * 2, 64, 256, CU_TENSOR_MAP_SWIZZLE_128B, "dY");
    QLORA_MAP(&t_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, W.w[0].codes, K / 2, N, K / 2, 128, 64,
              CU_TENSOR_MAP_SWIZZLE_128B, "codes");
    QLORA_MAP(&t_c, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, cT, L.ldc, K / kBlock, L.ldc * 4, 64, 4, CU_TENSOR_MAP_SWIZZLE_NONE,
              "constants");
    QLORA_MAP(&t_lact, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, sU, R, M, R * 2, 64, 256, CU_TENSOR_MAP_SWIZZLE_128B, "sU");
    QLORA_MAP(&t_lw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, K, R, K * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B, "A");
    FusedArgs fa{};
    fa.M = M;
    fa.out_cols = K;
    fa.red = N;
    fa.rank_cols = R;
    fa.rank_steps = nch;
    fa.ngroups = 1;
    fa.group_end[0] = K;
    fa.group_rank_x[0] = 0;
    fa.ctas = fused_ctas(M, fused_tiles_n(fa), N, std::min(sms, kPlanSms));
    fa.out = dX;
    fa.part = reinterpret_cast<float*>(base + L.skpart);
    fa.flags = reinterpret_cast<int*>(base + L.flags);
    fa.status = status;
    fa.timeout_ns = timeout_ns();
    fa.stall_producer = 0;
    if (injected_failure()) return QLORA_ERR_CUDA;
    const FusedPlan plan = fused_plan(M, fused_tiles_n(fa), N, sms);
    CUtensorMap h_codes, h_c;
    if (plan.pair_ctas) {
        QLORA_MAP(&h_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, W.w[0].codes, K / 2, N, K / 2, 64, 64,
                  CU_TENSOR_MAP_SWIZZLE_64B, "codes");
        QLORA_MAP(&h_c, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, cT, L.ldc, K / kBlock, L.ldc * 4, 64, 2,
                  CU_TENSOR_MAP_SWIZZLE_NONE, "constants");
    }
    cudaEvent_t ev0, ev1;
    take_profile_events(QLORA_KERNEL_FUSED_DX, &ev0, &ev1);
    if (ev0) QLORA_TRY(record_profile_event(ev0, st), "profile event");
    // plain stream order after the rank-r launches (a stream-K tail is the
    // pair launch's programmatic dependent); the adapter gradients, dX's
    // programmatic dependent, read sU and sT from their first step
    if (plan.pair_ctas) {
        FusedArgs pa = fa;
        pa.ctas = plan.pair_ctas;
        QLORA_LAUNCH(launch_fused_pair_dx(t_act, h_codes, h_c, t_lact, t_lw, pa, tables(), false, st), 1,
                     "fused dX (pairs)");
    }
    if (plan.tail_ctas) {
        FusedArgs ta = fa;
        ta.ctas = plan.tail_ctas;
        ta.tile_first = plan.tail_first;
        ta.tiles = plan.tail_tiles;
        ta.pair_order = plan.pair_ctas ? 1 : 0;
        QLORA_LAUNCH(launch_fused_dx(t_act, t_codes, t_c, t_lact, t_lw, ta, tables(), plan.pair_ctas != 0, st), 1,
                     "fused dX");
    }
    if (ev1) QLORA_TRY(record_profile_event(ev1, st), "profile event");

    // dA = sU^T X (as dA^T[K, R] = X^T sU, in 64-column chunks) and dB = dY^T sT
    // (chunks of sT, or per projection of a group dB_i = dY_i^T sT_i), split
    // over tokens
    SkinnyMaps maps;
    SkinnyArgs ga{};
    ga.NR = NRc;
    int64_t grad_tiles = nch * cdiv(K, 128);
    for (int c = 0; c < ndb; ++c) grad_tiles += cdiv(lo.group ? W.rows(c) : N, 128);
    ga.splits = skinny_splits(grad_tiles, M);
    ga.stages = kSkinnyStagesUsed;
    ga.chunks = kSkinnyChunksUsed;
    CUtensorMap t_xt;
    QLORA_MAP(&t_xt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, K, M, K * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B, "X^T");
    int np = 0;
    for (int c = 0; c < nch; ++c, ++np) {
        const int w = std::min(64, R - 64 * c);
        maps.a[np] = t_xt;
        if ((s = make_rank_map(&maps.b[np], sU + 64 * c, M, w, R, NRc, "sU")) != QLORA_OK) return s;
        ga.p[np] = skinny_problem(K, M, 1, 1, kSkinnyOutF32Transposed, w, K);
        ga.p[np].out_f32 = dA + static_cast<int64_t>(64 * c) * K;
    }
    for (int c = 0; c < ndb; ++c, ++np) {
        const int64_t n0 = lo.group ? W.off[c] : 0, rows = lo.group ? W.rows(c) : N;
        const int w = lo.group ? r : std::min(64, R - 64 * c);
        QLORA_MAP(&maps.a[np], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dY + n0, rows, M, N * 2, 64, 64,
                  CU_TENSOR_MAP_SWIZZLE_128B, "dY^T");
        if ((s = make_rank_map(&maps.b[np], sT + (lo.group ? c * r : 64 * c), M, w, R, NRc, "sT")) != QLORA_OK)
            return s;
        ga.p[np] = skinny_problem(rows, M, 1, 1, kSkinnyOutF32, w, dB_cols);
        ga.p[np].out_f32 = dB + (lo.group ? n0 * r : 64 * c);
    }
    ga.status = status;
    ga.timeout_ns = timeout_ns();
    if (injected_failure()) return QLORA_ERR_CUDA;
    // dA and dB need only sU and sT: launched as dX's programmatic
    // dependent they start once every dX tile has started, on the SMs dX's
    // last wave leaves idle (a profiled call keeps plain stream order)
    QLORA_LAUNCH(launch_skinny(maps, ga, np, st, ev1 == nullptr), 1, "skinny(grads)");
    return QLORA_OK;
}

Weights single_weight(const qlora_nf4_weight* w) {
    Weights W;
    W.w = w;
    W.P = 1;
    W.N = w->N;
    W.K = w->K;
    W.off[0] = 0;
    W.off[1] = w->N;
    return W;
}

}  // namespace

// The device word that records bounded waits that ran out in calls without a
// workspace (defined with the no-allocation quantiser's scratch below).
qlora_status call_status_word(int** out);

// =================================================================== ABI ==

extern "C" {

int64_t qlora_nf4_bytes(int64_t N, int64_t K, size_t* codes, size_t* qabsmax, size_t* s2, size_t* mean) {
    if (N <= 0 || K <= 0 || K % kBlock != 0) return -1;
    const int64_t nb = N * K / kBlock, ng = cdiv(nb, kGroup);
    const size_t c = static_cast<size_t>(N * K / 2), q = static_cast<size_t>(nb), s = static_cast<size_t>(ng) * 4, m = 4;
    if (codes) *codes = c;
    if (qabsmax) *qabsmax = q;
    if (s2) *s2 = s;
    if (mean) *mean = m;
    return static_cast<int64_t>(c + q + s + m);
}

size_t qlora_workspace_bytes(int op, int64_t M, int64_t N, int64_t K, int r) {
    if (N <= 0 || K <= 0 || K % kBlock != 0) return 0;
    if (op == QLORA_OP_QUANTIZE) {
        const int64_t nb = N * K / kBlock;
        return up256(static_cast<size_t>(nb) * 4) + dq_mean_scratch_bytes(nb);
    }
    if (op != QLORA_OP_FWD && op != QLORA_OP_BWD) return 0;
    if (M < 0 || !rank_ok(r)) return 0;
    qlora_nf4_weight w{};
    w.N = N;
    w.K = K;
    Lora lo;
    lo.r = r;
    return layout_for(op, M, single_weight(&w), lo).total;
}

const char* qlora_status_string(qlora_status s) {
    switch (s) {
        case QLORA_OK: return "QLORA_OK";
        case QLORA_ERR_INVALID_ARG: return "QLORA_ERR_INVALID_ARG";
        case QLORA_ERR_BAD_SHAPE: return "QLORA_ERR_BAD_SHAPE";
        case QLORA_ERR_MISALIGNED: return "QLORA_ERR_MISALIGNED";
        case QLORA_ERR_UNSUPPORTED_RANK: return "QLORA_ERR_UNSUPPORTED_RANK";
        case QLORA_ERR_WORKSPACE_TOO_SMALL: return "QLORA_ERR_WORKSPACE_TOO_SMALL";
        case QLORA_ERR_CUDA: return "QLORA_ERR_CUDA";
        case QLORA_ERR_DEVICE_TIMEOUT: return "QLORA_ERR_DEVICE_TIMEOUT";
        case QLORA_ERR_UNSUPPORTED_DEVICE: return "QLORA_ERR_UNSUPPORTED_DEVICE";
        case QLORA_ERR_EXCEEDS_STATIC_SCRATCH: return "QLORA_ERR_EXCEEDS_STATIC_SCRATCH";
        default: return "QLORA_ERR_UNKNOWN";
    }
}

const char* qlora_last_error(void) { return g_last_error.c_str(); }

qlora_status qlora_set_option(int option, int64_t value) {
    switch (option) {
        case QLORA_OPT_SMALL_M_MAX: g_small_m_max = value; return QLORA_OK;
        case QLORA_OPT_FAIL_LAUNCHES: g_fail_launches = std::max<int64_t>(0, value); return QLORA_OK;
        case QLORA_OPT_WAIT_TIMEOUT_US:
            if (value <= 0) return QLORA_ERR_INVALID_ARG;
            g_timeout_us = value;
            return QLORA_OK;
        case QLORA_OPT_STALL_PRODUCER: g_stall_producer = value ? 1 : 0; return QLORA_OK;
        case QLORA_OPT_LAUNCH_COUNT: g_launch_count = value; return QLORA_OK;
        case QLORA_OPT_SKINNY_MAX_SPLITS:
            if (value < 0) return QLORA_ERR_INVALID_ARG;
            g_skinny_max_splits = value;
            return QLORA_OK;
        case QLORA_OPT_FUSED_PAIRS: g_fused_pairs = value ? 1 : 0; return QLORA_OK;
        case QLORA_OPT_FUSED_TAIL: g_fused_tail = value ? 1 : 0; return QLORA_OK;
        default: return QLORA_ERR_INVALID_ARG;
    }
}

int64_t qlora_get_option(int option) {
    switch (option) {
        case QLORA_OPT_SMALL_M_MAX: return g_small_m_max.load();
        case QLORA_OPT_FAIL_LAUNCHES: return g_fail_launches.load();
        case QLORA_OPT_WAIT_TIMEOUT_US: return g_timeout_us.load();
        case QLORA_OPT_STALL_PRODUCER: return g_stall_producer.load();
        case QLORA_OPT_LAUNCH_COUNT: return g_launch_count.load();
        case QLORA_OPT_SKINNY_MAX_SPLITS: return g_skinny_max_splits.load();
        case QLORA_OPT_FUSED_PAIRS: return g_fused_pairs.load();
        case QLORA_OPT_FUSED_TAIL: return g_fused_tail.load();
        default: return -1;
    }
}

qlora_status qlora_nf4_tables(float* levels_host, float* thresholds_host) {
    if (!levels_host || !thresholds_host) return QLORA_ERR_INVALID_ARG;
    const Nf4Tables& t = tables();
    std::memcpy(levels_host, t.level, sizeof(t.level));
    std::memcpy(thresholds_host, t.thresh, sizeof(t.thresh));
    return QLORA_OK;
}

namespace {
qlora_status quantize_any(const void* W, bool bf16, int64_t N, int64_t K, uint8_t* codes, uint8_t* qabsmax, float* s2,
                          float* mean, void* ws, size_t ws_bytes, void* stream);
}  // namespace

qlora_status qlora_quantize_nf4(const float* W, int64_t N, int64_t K, uint8_t* codes, uint8_t* qabsmax, float* s2,
                                float* mean, void* ws, size_t ws_bytes, void* stream) {
    return quantize_any(W, false, N, K, codes, qabsmax, s2, mean, ws, ws_bytes, stream);
}

qlora_status qlora_quantize_nf4_bf16(const uint16_t* W, int64_t N, int64_t K, uint8_t* codes, uint8_t* qabsmax,
                                     float* s2, float* mean, void* ws, size_t ws_bytes, void* stream) {
    return quantize_any(W, true, N, K, codes, qabsmax, s2, mean, ws, ws_bytes, stream);
}

namespace {
// Quantise: the encoder (which also zeroes the mean kernel's ticket), the
// mean and the E4M3 group pass.
qlora_status quantize_dq(const void* W, bool bf16, int64_t N, int64_t K, uint8_t* codes, uint8_t* qabsmax, float* s2,
                         float* mean, float* absmax, void* mean_scratch, int sms, cudaStream_t st) {
    const int64_t nb = N * K / kBlock;
    QLORA_LAUNCH(launch_nf4_encode(W, bf16, N, K, codes, absmax, dq_mean_ticket(mean_scratch, nb), tables(), sms, st),
                 1, "nf4_encode");
    if (injected_failure()) return QLORA_ERR_CUDA;
    QLORA_LAUNCH(launch_dq_mean(absmax, nb, mean_scratch, mean, st), 1, "double quantisation mean");
    if (injected_failure()) return QLORA_ERR_CUDA;
    QLORA_LAUNCH(launch_dq_groups(absmax, nb, mean, qabsmax, s2, st), 1, "double quantisation groups");
    return QLORA_OK;
}

qlora_status quantize_any(const void* W, bool bf16, int64_t N, int64_t K, uint8_t* codes, uint8_t* qabsmax, float* s2,
                          float* mean, void* ws, size_t ws_bytes, void* stream) {
    if (!W || !codes || !qabsmax || !s2 || !mean || !ws) return QLORA_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0 || K % kBlock != 0) return QLORA_ERR_BAD_SHAPE;
    if (!aligned16(W) || !aligned16(codes) || !aligned16(qabsmax) || !aligned16(s2) || !aligned16(ws) ||
        (reinterpret_cast<uintptr_t>(mean) & 3u))
        return QLORA_ERR_MISALIGNED;
    if (ws_bytes < qlora_workspace_bytes(QLORA_OP_QUANTIZE, 0, N, K, 0)) return QLORA_ERR_WORKSPACE_TOO_SMALL;
    if (injected_failure()) return QLORA_ERR_CUDA;
    int sms = 0;
    qlora_status s = device_ready(&sms);
    if (s != QLORA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t nb = N * K / kBlock;
    float* absmax = static_cast<float*>(ws);
    void* tree = static_cast<uint8_t*>(ws) + up256(static_cast<size_t>(nb) * 4);
    return quantize_dq(W, bf16, N, K, codes, qabsmax, s2, mean, absmax, tree, sms, st);
}
}  // namespace

namespace {
qlora_status quantize_nodq(const void* W, bool bf16, int64_t N, int64_t K, uint8_t* codes, float* absmax,
                           void* stream) {
    if (!W || !codes || !absmax) return QLORA_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0 || K % kBlock != 0) return QLORA_ERR_BAD_SHAPE;
    if (!aligned16(W) || !aligned16(codes) || !aligned16(absmax)) return QLORA_ERR_MISALIGNED;
    if (injected_failure()) return QLORA_ERR_CUDA;
    int sms = 0;
    qlora_status s = device_ready(&sms);
    if (s != QLORA_OK) return s;
    QLORA_LAUNCH(launch_nf4_encode(W, bf16, N, K, codes, absmax, nullptr, tables(), sms,
                                   static_cast<cudaStream_t>(stream)),
                 1, "nf4_encode");
    return QLORA_OK;
}
}  // namespace

qlora_status qlora_quantize_nf4_nodq(const float* W, int64_t N, int64_t K, uint8_t* codes, float* absmax,
                                     void* stream) {
    return quantize_nodq(W, false, N, K, codes, absmax, stream);
}

qlora_status qlora_quantize_nf4_bf16_nodq(const uint16_t* W, int64_t N, int64_t K, uint8_t* codes, float* absmax,
                                          void* stream) {
    return quantize_nodq(W, true, N, K, codes, absmax, stream);
}

qlora_status qlora_merge_lora(const qlora_nf4_weight* w, const uint16_t* A, const uint16_t* B, int r, float alpha,
                              uint16_t* W_out, void* stream) {
    qlora_status s = check_weight(w);
    if (s != QLORA_OK) return s;
    if (!rank_ok(r)) return QLORA_ERR_UNSUPPORTED_RANK;
    if (!A || !B || !W_out || !std::isfinite(alpha)) return QLORA_ERR_INVALID_ARG;
    if (!aligned16(A) || !aligned16(B) || !aligned16(W_out)) return QLORA_ERR_MISALIGNED;
    if (injected_failure()) return QLORA_ERR_CUDA;
    int sms = 0;
    if ((s = device_ready(&sms)) != QLORA_OK) return s;
    int* status = nullptr;
    if ((s = call_status_word(&status)) != QLORA_OK) return s;
    MergeArgs a{};
    a.codes = w->codes;
    a.c = constants_of(w);
    a.A = A;
    a.B = B;
    a.scale = alpha / static_cast<float>(r);
    a.N = w->N;
    a.K = w->K;
    a.W_out = W_out;
    a.status = status;
    a.timeout_ns = timeout_ns();
    const int64_t N = w->N, K = w->K;
    CUtensorMap mb, ma, mc;
    QLORA_MAP(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, r, N, static_cast<uint64_t>(r) * 2, 64, 128,
              CU_TENSOR_MAP_SWIZZLE_128B, "B");
    QLORA_MAP(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, K, r, K * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B, "A");
    QLORA_MAP(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->codes, K / 2, N, K / 2, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B,
              "codes");
    CUtensorMap mo;
    QLORA_MAP(&mo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W_out, K, N, K * 2, 64, 32, CU_TENSOR_MAP_SWIZZLE_128B, "W_out");
    QLORA_LAUNCH(launch_merge_tc(mb, ma, mc, mo, a, r, tables(), sms, static_cast<cudaStream_t>(stream)), 1,
                 "merge_lora");
    return QLORA_OK;
}

qlora_status qlora_dequantize_nf4(const qlora_nf4_weight* w, uint16_t* W_out, void* stream) {
    if (!W_out) return QLORA_ERR_INVALID_ARG;
    qlora_status s = check_weight(w);
    if (s != QLORA_OK) return s;
    if (!aligned16(W_out)) return QLORA_ERR_MISALIGNED;
    if (injected_failure()) return QLORA_ERR_CUDA;
    int sms = 0;
    if ((s = device_ready(&sms)) != QLORA_OK) return s;
    CUtensorMap t_out;
    QLORA_MAP(&t_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W_out, kBlock, w->N * w->K / kBlock, kBlock * 2, 64, 128,
              CU_TENSOR_MAP_SWIZZLE_128B, "W_out");
    QLORA_LAUNCH(launch_nf4_dequant(t_out, w->codes, constants_of(w), w->N, w->K, tables(), sms,
                                    static_cast<cudaStream_t>(stream)),
                 1, "nf4_dequant");
    return QLORA_OK;
}

qlora_status qlora_linear_fwd(const uint16_t* X, int64_t M, const qlora_nf4_weight* w, const uint16_t* A,
                              const uint16_t* B, int r, float alpha, uint16_t* Y, uint16_t* sT_save, void* ws,
                              size_t ws_bytes, void* stream) {
    qlora_status s = check_weight(w);
    if (s != QLORA_OK) return s;
    Lora lo;
    lo.r = r;
    return fwd_impl(X, M, single_weight(w), A, B, lo, alpha, Y, sT_save, ws, ws_bytes, stream);
}

qlora_status qlora_linear_bwd(const uint16_t* dY, const uint16_t* X, int64_t M, const qlora_nf4_weight* w,
                              const uint16_t* A, const uint16_t* B, int r, float alpha, const uint16_t* sT_in,
                              uint16_t* dX, float* dA, float* dB, void* ws, size_t ws_bytes, void* stream) {
    qlora_status s = check_weight(w);
    if (s != QLORA_OK) return s;
    Lora lo;
    lo.r = r;
    return bwd_impl(dY, X, M, single_weight(w), A, B, lo, alpha, sT_in, dX, dA, dB, ws, ws_bytes, stream);
}

size_t qlora_workspace_bytes_multi(int op, int64_t M, int64_t N, int64_t K, int r, int P) {
    if (N <= 0 || K <= 0 || K % kBlock != 0) return 0;
    if ((op != QLORA_OP_FWD && op != QLORA_OP_BWD) || M < 0 || !rank_ok(r) || P < 1 || P * r > kMaxMultiRank)
        return 0;
    qlora_nf4_weight w{};
    w.N = N;
    w.K = K;
    Lora lo;
    lo.r = r;
    lo.P = P;
    return layout_for(op, M, single_weight(&w), lo).total;
}

qlora_status qlora_linear_fwd_multi(const uint16_t* X, int64_t M, const qlora_nf4_weight* w, const uint16_t* A,
                                    const uint16_t* B, int r, int P, const int32_t* ids, float alpha, uint16_t* Y,
                                    uint16_t* sT_save, void* ws, size_t ws_bytes, void* stream) {
    qlora_status s = check_weight(w);
    if (s != QLORA_OK) return s;
    Lora lo;
    lo.r = r;
    lo.P = P;
    lo.ids = ids;
    return fwd_impl(X, M, single_weight(w), A, B, lo, alpha, Y, sT_save, ws, ws_bytes, stream);
}

qlora_status qlora_linear_bwd_multi(const uint16_t* dY, const uint16_t* X, int64_t M, const qlora_nf4_weight* w,
                                    const uint16_t* A, const uint16_t* B, int r, int P, const int32_t* ids,
                                    float alpha, const uint16_t* sT, uint16_t* dX, float* dA, float* dB, void* ws,
                                    size_t ws_bytes, void* stream) {
    qlora_status s = check_weight(w);
    if (s != QLORA_OK) return s;
    Lora lo;
    lo.r = r;
    lo.P = P;
    lo.ids = ids;
    return bwd_impl(dY, X, M, single_weight(w), A, B, lo, alpha, sT, dX, dA, dB, ws, ws_bytes, stream);
}

size_t qlora_workspace_bytes_group(int op, int64_t M, const int64_t* N, int P, int64_t K, int r) {
    if (!N || P < 1 || P > kMaxGroups || K <= 0 || K % kBlock != 0) return 0;
    if ((op != QLORA_OP_FWD && op != QLORA_OP_BWD) || M < 0 || !rank_ok(r)) return 0;
    qlora_nf4_weight w[kMaxGroups] = {};
    Weights W;
    W.w = w;
    W.P = P;
    W.K = K;
    for (int i = 0; i < P; ++i) {
        if (N[i] <= 0) return 0;
        w[i].N = N[i];
        w[i].K = K;
        W.off[i + 1] = W.off[i] + N[i];
    }
    W.N = W.off[P];
    Lora lo;
    lo.r = r;
    lo.P = P;
    lo.group = true;
    return layout_for(op, M, W, lo).total;
}

qlora_status qlora_linear_fwd_group(const uint16_t* X, int64_t M, const qlora_nf4_weight* w, int P,
                                    const uint16_t* A, const uint16_t* B, int r, float alpha, uint16_t* Y,
                                    uint16_t* sT_save, void* ws, size_t ws_bytes, void* stream) {
    Weights W;
    qlora_status s = check_weights(w, P, &W);
    if (s != QLORA_OK) return s;
    Lora lo;
    lo.r = r;
    lo.P = P;
    lo.group = true;
    return fwd_impl(X, M, W, A, B, lo, alpha, Y, sT_save, ws, ws_bytes, stream);
}

qlora_status qlora_linear_bwd_group(const uint16_t* dY, const uint16_t* X, int64_t M, const qlora_nf4_weight* w,
                                    int P, const uint16_t* A, const uint16_t* B, int r, float alpha,
                                    const uint16_t* sT, uint16_t* dX, float* dA, float* dB, void* ws,
                                    size_t ws_bytes, void* stream) {
    Weights W;
    qlora_status s = check_weights(w, P, &W);
    if (s != QLORA_OK) return s;
    Lora lo;
    lo.r = r;
    lo.P = P;
    lo.group = true;
    return bwd_impl(dY, X, M, W, A, B, lo, alpha, sT, dX, dA, dB, ws, ws_bytes, stream);
}

qlora_status qlora_device_status(const void* ws, int* status_host, void* stream) {
    if (!status_host) return QLORA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int v = 0;
    if (ws) {
        QLORA_TRY(cudaMemcpyAsync(&v, ws, sizeof(int), cudaMemcpyDeviceToHost, st), "read status");
        QLORA_TRY(cudaStreamSynchronize(st), "sync");
    } else {
        // calls without a workspace: the library's own word, cleared once read
        int* w = nullptr;
        const qlora_status s = call_status_word(&w);
        if (s != QLORA_OK) return s;
        QLORA_TRY(cudaMemcpyAsync(&v, w, sizeof(int), cudaMemcpyDeviceToHost, st), "read status");
        QLORA_TRY(cudaMemsetAsync(w, 0, sizeof(int), st), "clear status");
        QLORA_TRY(cudaStreamSynchronize(st), "sync");
    }
    *status_host = (v & kStatusTimeout) ? QLORA_ERR_DEVICE_TIMEOUT : (v ? QLORA_ERR_CUDA : QLORA_OK);
    return QLORA_OK;
}

qlora_status qlora_profile_next_launch(int kernel, void* ev_start, void* ev_stop) {
    if (kernel != QLORA_KERNEL_FUSED_FWD && kernel != QLORA_KERNEL_FUSED_DX) return QLORA_ERR_INVALID_ARG;
    if ((ev_start == nullptr) != (ev_stop == nullptr)) return QLORA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_events[kernel][0] = static_cast<cudaEvent_t>(ev_start);
    g_prof_events[kernel][1] = static_cast<cudaEvent_t>(ev_stop);
    return QLORA_OK;
}

qlora_status qlora_e4m3_encode(const float* x, uint8_t* q, int64_t n, void* stream) {
    if (!x || !q) return QLORA_ERR_INVALID_ARG;
    if (n < 0) return QLORA_ERR_BAD_SHAPE;
    if (n == 0) return QLORA_OK;
    if (injected_failure()) return QLORA_ERR_CUDA;
    qlora_status s = device_ready(nullptr);
    if (s != QLORA_OK) return s;
    QLORA_LAUNCH(launch_e4m3_encode(x, q, n, static_cast<cudaStream_t>(stream)), 1, "e4m3_encode");
    return QLORA_OK;
}

}  // extern "C"

// ======================================================== no allocation ==
// The status word of calls without a workspace (the adapter merge): one
// file-scope device int, read and cleared by qlora_device_status(NULL, ...).
namespace {
static __device__ int g_call_status;
}  // namespace

qlora_status call_status_word(int** out) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_call_status);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status word)");
    *out = static_cast<int*>(p);
    return QLORA_OK;
}

// Quantiser scratch for callers that cannot allocate: one file-scope device
// array, 4 MiB of fp32 block absmax followed by the mean's run sums and
// ticket for 2^20 blocks (768 B). Host code never touches `g_noalloc_scratch`
// directly (on the host its name is only a stand-in); the current context's
// address comes from cudaGetSymbolAddress on every call, so a context
// recreated after cudaDeviceReset gets its own module's address.
namespace {

constexpr int64_t kNoAllocMaxBlocks = int64_t(1) << 20;  // 64M weights
constexpr size_t kNoAllocAbsmaxBytes = static_cast<size_t>(kNoAllocMaxBlocks) * 4;
// sized at compile time for the largest nb; the mean's scratch does not
// shrink as nb grows, so it covers every nb <= kNoAllocMaxBlocks
constexpr size_t kNoAllocTreeBytes = dq_mean_scratch_bytes(kNoAllocMaxBlocks);
constexpr size_t kNoAllocBytes = kNoAllocAbsmaxBytes + kNoAllocTreeBytes;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

qlora_status noalloc_scratch(void** out) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
    if (!p) return cuda_fail(cudaErrorInvalidSymbol, "cudaGetSymbolAddress(static scratch)");
    *out = p;
    return QLORA_OK;
}

}  // namespace

extern "C" qlora_status qlora_quantize_nf4_noalloc(const float* W, int64_t N, int64_t K, uint8_t* codes,
                                                   uint8_t* qabsmax, float* s2, float* mean, void* stream) {
    if (!W || !codes || !qabsmax || !s2 || !mean) return QLORA_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0 || K % kBlock != 0) return QLORA_ERR_BAD_SHAPE;
    if (!aligned16(W) || !aligned16(codes) || !aligned16(qabsmax) || !aligned16(s2) ||
        (reinterpret_cast<uintptr_t>(mean) & 3u))
        return QLORA_ERR_MISALIGNED;
    if (N > kNoAllocMaxBlocks * kBlock / K) {
        g_last_error = "qlora_quantize_nf4_noalloc: N*K = " + std::to_string(N) + "*" + std::to_string(K) +
                       " exceeds the static scratch limit of " + std::to_string(kNoAllocMaxBlocks * kBlock) +
                       " weights; use qlora_quantize_nf4 with a workspace";
        return QLORA_ERR_EXCEEDS_STATIC_SCRATCH;
    }
    if (injected_failure()) return QLORA_ERR_CUDA;
    int sms = 0;
    qlora_status s = device_ready(&sms);
    if (s != QLORA_OK) return s;
    void* scratch = nullptr;
    if ((s = noalloc_scratch(&scratch)) != QLORA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float* absmax = static_cast<float*>(scratch);
    void* tree = static_cast<unsigned char*>(scratch) + kNoAllocAbsmaxBytes;
    return quantize_dq(W, false, N, K, codes, qabsmax, s2, mean, absmax, tree, sms, st);
}
