// Dequant-fused NF4 matmuls on the sm_100 tensor core (tcgen05 + TMEM + TMA).
//
//   forward:  out[M, N] = X[M, K] . deq(W)[N, K]^T + sT[M, r] . B[N, r]^T
//   dX:       out[M, K] = dY[M, N] . deq(W)[N, K]   + sU[M, r] . A[r, K]
//
// "ta-paperlens QLoRA explainer", section 勾配は実際どこへ行くのか: W is stored
// in NF4 and every matmul restores the 4-bit blocks it needs to BF16 on the
// spot; the input gradient passes through deq(W)^T. "waylandz ch.26" 26.2.4:
// the LoRA path adds (alpha/r) B (A x); here (alpha/r) A x arrives precomputed
// in bf16 (sT, sU) and the rank-r product runs as one extra reduction step.
//
// One CTA computes a 256 x 256 output tile (two M=128 UMMAs sharing each
// dequantised weight tile, 512 TMEM columns of fp32 accumulators).
//   warp 8      TMA producer: activation tile, packed codes, decoded constants
//   warps 0-7   dequantisers: one 64-weight block per thread per step, written
//               as bf16 straight into the 128-byte-swizzled UMMA operand layout
//               (K-major for the forward, MN-major for dX); then epilogue
//   warp 9      TMEM owner; lane 0 issues the UMMAs and commits
// Pipelined over 3 shared-memory stages with mbarriers; every wait is bounded.
#include "common.cuh"
#include "kernels.h"

namespace qlora {

namespace {

constexpr uint32_t kActBytes = kFusedBM * kFusedBK * 2;   // 32 KB bf16
constexpr uint32_t kWBytes = kFusedBN * kFusedBK * 2;     // 32 KB bf16
constexpr uint32_t kCodeBytes = kFusedBN * kFusedBK / 2;  // 8 KB packed nibbles
constexpr uint32_t kCBytes = 1024;                        // 256 decoded constants
constexpr uint32_t kOffW = kActBytes;
constexpr uint32_t kOffCodes = kOffW + kWBytes;
constexpr uint32_t kOffC = kOffCodes + kCodeBytes;
constexpr uint32_t kStageBytes = kOffC + kCBytes;  // 73 KB, a multiple of 1024
constexpr uint32_t kBarOffset = kFusedStages * kStageBytes;
constexpr uint32_t kSmemBytes = kBarOffset + 256 + 1024;  // + barriers, + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr int kDequantWarps = 8;

// Dequantise one 64-weight block: 32 code bytes (two 16-byte chunks at c0, c1)
// into eight 16-byte bf16 chunks at dst + chunk_off(j).
template <typename ChunkOff>
__device__ __forceinline__ void dequant_block(const Nf4Tables& tab, float cprime, uint32_t c0, uint32_t c1,
                                              ChunkOff chunk_off) {
    const Nf4BlockLut lut = make_block_lut(tab.level, cprime);
    const uint4 a = lds128(c0), b = lds128(c1);
    const uint32_t words[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        uint32_t o[4];
        lut_decode8(lut, words[j], o);
        sts128(chunk_off(j), o);
    }
}

// Stream-K schedule. The work is the list of (output tile, 64-deep reduction
// step) units, tile-major; CTA c (one per SM) takes the contiguous range
// [c W / P, (c + 1) W / P). Cut at tile boundaries, a range is a list of
// segments. The CTA that holds a tile's last step owns the tile: it also runs
// the rank-r steps and writes the tile. A segment that ends before the tile's
// last step is a contributor: it writes its fp32 partial tile and raises a
// flag. Every CTA walks its segments from last to first, so its contribution
// (the head of the next tile, at the end of its range) comes first and its
// ownership (the tail of a tile, at the start of its range) last: an owner
// finds the partials of the lower-indexed CTAs ready, adds them in CTA order
// (deterministic) and writes the bf16 tile. An owner waits only for CTAs with
// lower indices, which the hardware has dispatched before it.
struct Sched {
    int64_t W;    // tiles * KT
    int P;        // CTAs
    int KT;       // reduction steps per tile
    __device__ int64_t begin(int c) const { return static_cast<int64_t>(c) * W / P; }
    __device__ int cta_of(int64_t u) const { return static_cast<int>(((u + 1) * P - 1) / W); }
};

// Walks the segments of one CTA's range, last to first. Without splitting
// (kSplit false: one CTA per tile) the range is exactly tile c, all of its
// steps.
template <bool kSplit>
struct SegIter {
    const Sched& sc;
    int64_t lo, hi;  // units not yet walked: [lo, hi)
    int64_t tile;
    int k_lo, k_hi;
    __device__ SegIter(const Sched& s, int c)
        : sc(s), lo(kSplit ? s.begin(c) : static_cast<int64_t>(c) * s.KT),
          hi(kSplit ? s.begin(c + 1) : static_cast<int64_t>(c + 1) * s.KT), tile(0), k_lo(0), k_hi(0) {}
    __device__ bool next() {
        if (hi <= lo) return false;
        if (!kSplit) {
            tile = lo / sc.KT;
            k_lo = 0;
            k_hi = sc.KT;
            hi = lo;
            return true;
        }
        tile = (hi - 1) / sc.KT;
        const int64_t t0 = tile * sc.KT;
        const int64_t start = max(lo, t0);
        k_lo = static_cast<int>(start - t0);
        k_hi = static_cast<int>(hi - t0);
        hi = start;
        return true;
    }
    __device__ bool owner() const { return k_hi == sc.KT; }
};

// The output columns of column tile j: [n0, n_lim), and the act-side column
// of its rank input. Tiles are 256 columns, counted group by group.
struct TileCols {
    int64_t n0, n_lim;
    int rank_x;
};
__device__ __forceinline__ TileCols tile_cols(const FusedArgs& a, int64_t j) {
    int64_t start = 0;
    for (int g = 0; g < a.ngroups; ++g) {
        const int64_t cnt = (a.group_end[g] - start + kFusedBN - 1) / kFusedBN;
        if (j < cnt || g == a.ngroups - 1) return TileCols{start + j * kFusedBN, a.group_end[g], a.group_rank_x[g]};
        j -= cnt;
        start = a.group_end[g];
    }
    return TileCols{0, 0, 0};
}

// Row and column tile of tile t of a launch (see FusedArgs::pair_order).
struct TileRC {
    int64_t m, n;
};
__device__ __forceinline__ TileRC tile_rc(const FusedArgs& a, int tiles_n, int64_t t) {
    const int64_t g = a.tile_first + t;
    if (!a.pair_order) return TileRC{g / tiles_n, g % tiles_n};
    const int64_t p = g >> 1, pairs_m = (a.M + 2 * kFusedBM - 1) / (2 * kFusedBM);
    return TileRC{2 * (p % pairs_m) + (g & 1), p / pairs_m};
}

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release(int* p, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

template <bool kTransW, bool kSplit>
__global__ void __launch_bounds__(kFusedThreads, 1)
    fused_nf4_gemm(const __grid_constant__ CUtensorMap tm_act, const __grid_constant__ CUtensorMap tm_codes,
                   const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_lact,
                   const __grid_constant__ CUtensorMap tm_lw, const FusedArgs args, const Nf4Tables tab) {
    // a launch that depends on this one programmatically (the adapter
    // gradients beside dX) is admitted once every tile of this launch has
    // started, i.e. onto the SMs its last wave leaves idle
    asm volatile("griddepcontrol.launch_dependents;");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOffset);
    uint64_t* deq = full + kFusedStages;
    uint64_t* empty = deq + kFusedStages;
    uint64_t* acc = empty + kFusedStages;
    uint64_t* tmem_free = acc + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tmem_free + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* parts_ok = abort_flag + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KT = static_cast<int>((args.red + kFusedBK - 1) / kFusedBK);
    int tiles_n = 0;
    {
        int64_t start = 0;
        for (int g = 0; g < args.ngroups; ++g) {
            tiles_n += static_cast<int>((args.group_end[g] - start + kFusedBN - 1) / kFusedBN);
            start = args.group_end[g];
        }
    }
    const int tiles_m = static_cast<int>((args.M + kFusedBM - 1) / kFusedBM);
    const int64_t tiles = args.tiles > 0 ? args.tiles : static_cast<int64_t>(tiles_m) * tiles_n;
    const Sched sc{tiles * KT, static_cast<int>(gridDim.x), KT};
    const int cta = blockIdx.x;
    const int rank_steps = args.rank_cols > 0 ? args.rank_steps : 0;
    const uint64_t tmo = args.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kFusedStages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(deq + s, kDequantWarps);  // one arrive per dequant warp, every step
            mbar_init(empty + s, 1);
        }
        mbar_init(acc, 1);
        mbar_init(tmem_free, kDequantWarps);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (warp == 8 && lane == 0) {
        tma_prefetch_desc(&tm_act);
        tma_prefetch_desc(&tm_codes);
        tma_prefetch_desc(&tm_c);
        tma_prefetch_desc(&tm_lact);
        tma_prefetch_desc(&tm_lw);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 8) {
        // ------------------------------------------------------ producer --
        if (lane == 0) {
            int last_use[kFusedStages];
            for (int s = 0; s < kFusedStages; ++s) last_use[s] = -1;
            int g = 0;    // ring position over all steps of all segments
            int seg = -1;  // segment index
            SegIter<kSplit> it(sc, cta);
            while (!args.stall_producer && !*abort_flag && it.next()) {
                ++seg;
                const TileRC rc = tile_rc(args, tiles_n, it.tile);
                const int64_t m0 = rc.m * kFusedBM;
                const TileCols tc = tile_cols(args, rc.n);
                const int64_t n0 = tc.n0;
                const int nk = it.k_hi - it.k_lo;
                const int steps = nk + (it.owner() ? rank_steps : 0);
                for (int i = 0; i < steps; ++i, ++g) {
                    const int s = g % kFusedStages;
                    const uint32_t u = static_cast<uint32_t>(g / kFusedStages);
                    if (g >= kFusedStages && !mbar_wait(empty + s, (u - 1) & 1u, tmo, args.status)) {
                        *abort_flag = 1;
                        break;
                    }
                    if (*abort_flag) break;
                    uint8_t* st = smem + s * kStageBytes;
                    if (i < nk) {
                        const int kt = it.k_lo + i;
                        mbar_arrive_expect_tx(full + s, kActBytes + kCodeBytes + kCBytes);
                        tma_load_2d(st, &tm_act, full + s, kt * kFusedBK, static_cast<int>(m0));
                        if (!kTransW) {
                            // codes rows n0.., bytes of k-block kt; constants of k-block kt, rows n0..
                            tma_load_2d(st + kOffCodes, &tm_codes, full + s, kt * (kFusedBK / 2), static_cast<int>(n0));
                            tma_load_2d(st + kOffC, &tm_c, full + s, static_cast<int>(n0), kt);
                        } else {
                            // codes rows kt*64.. (reduction), bytes of columns n0..n0+255
                            tma_load_2d(st + kOffCodes, &tm_codes, full + s, static_cast<int>(n0 / 2), kt * kFusedBK);
                            tma_load_2d(st + kOffC, &tm_c, full + s, kt * kFusedBK, static_cast<int>(n0 / kBlock));
                        }
                    } else {
                        const int c = i - nk;  // rank step: columns 64c .. 64c + 63 of the rank term
                        if (c == 0) {
                            // the rank-r input (sT or sU) comes from the preceding
                            // launch, of which this one may be a programmatic dependent
                            asm volatile("griddepcontrol.wait;" ::: "memory");
                            // the rank steps land in weight-tile regions, one of which
                            // the previous segment's epilogue uses as scratch: wait for it
                            if (seg > 0 &&
                                !mbar_wait(tmem_free, static_cast<uint32_t>(seg - 1) & 1u, tmo, args.status)) {
                                *abort_flag = 1;
                                break;
                            }
                        }
                        mbar_arrive_expect_tx(full + s, kActBytes + kWBytes);
                        tma_load_2d(st, &tm_lact, full + s, tc.rank_x + 64 * c, static_cast<int>(m0));
                        if (!kTransW) {
                            tma_load_2d(st + kOffW, &tm_lw, full + s, 64 * c, static_cast<int>(n0));
                        } else {
                            for (int a = 0; a < 4; ++a)
                                tma_load_2d(st + kOffW + a * 8192, &tm_lw, full + s, static_cast<int>(n0) + 64 * a,
                                            64 * c);
                        }
                    }
                    last_use[s] = static_cast<int>(u);
                }
            }
            // make sure no copy is still landing in shared memory at exit
            for (int s = 0; s < kFusedStages; ++s)
                if (last_use[s] >= 0) mbar_wait(full + s, static_cast<uint32_t>(last_use[s]) & 1u, tmo, nullptr);
        }
        __syncwarp();
    } else if (warp == 9) {
        // ----------------------------------------------------------- MMA --
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, kFusedBN, false, kTransW);
            bool ok = true;
            int g = 0, seg = 0;
            SegIter<kSplit> it(sc, cta);
            while (ok && it.next()) {
                // the accumulator must have been read out by the previous epilogue
                if (seg > 0 && !mbar_wait(tmem_free, static_cast<uint32_t>(seg - 1) & 1u, tmo, args.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int nk = it.k_hi - it.k_lo;
                const int steps = nk + (it.owner() ? rank_steps : 0);
                for (int i = 0; i < steps; ++i, ++g) {
                    const int s = g % kFusedStages;
                    const uint32_t u = static_cast<uint32_t>(g / kFusedStages);
                    if (!mbar_wait(full + s, u & 1u, tmo, args.status) || !mbar_wait(deq + s, u & 1u, tmo, args.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t act = smem_u32(smem + s * kStageBytes);
                    const uint32_t wt = act + kOffW;
                    const int ksub = (i < nk) ? (kFusedBK / 16) : (min(64, args.rank_cols - 64 * (i - nk)) + 15) / 16;
                    for (int kk = 0; kk < ksub; ++kk) {
                        const uint64_t bdesc = kTransW ? sw128_desc(wt + kk * 2048, 8192, 1024)
                                                       : sw128_desc(wt + kk * 32, 16, 1024);
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint64_t adesc = sw128_desc(act + h * 16384 + kk * 32, 16, 1024);
                            umma_f16(tmem + h * 256, adesc, bdesc, idesc, (i > 0 || kk > 0) ? 1u : 0u);
                        }
                    }
                    umma_commit(empty + s);
                }
                umma_commit(acc);  // arrives once every UMMA of the segment has completed
                ++seg;
            }
            if (!ok) {
                *abort_flag = 1;
                __threadfence_block();
                umma_commit(acc);  // releases an epilogue waiting on this segment
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------- dequantise, then epilogue --
        const int t = threadIdx.x;  // 0..255
        const int q = warp & 3, h = warp >> 2;
        const int row_l = h * 128 + q * 32 + lane;  // tile row of this thread in the epilogue
        bool ok = true;
        int g = 0, seg = 0;
        SegIter<kSplit> it(sc, cta);
        while (it.next()) {
            const TileRC rc = tile_rc(args, tiles_n, it.tile);
            const int64_t m0 = rc.m * kFusedBM;
            const TileCols tc = tile_cols(args, rc.n);
            const int64_t n0 = tc.n0;
            const int nk = it.k_hi - it.k_lo;
            const int steps = nk + (it.owner() ? rank_steps : 0);
            for (int i = 0; ok && i < steps; ++i, ++g) {
                const int s = g % kFusedStages;
                const uint32_t u = static_cast<uint32_t>(g / kFusedStages);
                // every lane waits; the outcome is made warp-uniform before any branch
                ok = __all_sync(0xFFFFFFFFu, mbar_wait(full + s, u & 1u, tmo, args.status));
                if (!ok) break;
                if (i < nk) {
                    uint8_t* st = smem + s * kStageBytes;
                    const uint32_t codes = smem_u32(st + kOffCodes);
                    const uint32_t wt = smem_u32(st + kOffW);
                    const float* cs = reinterpret_cast<const float*>(st + kOffC);
                    if (!kTransW) {
                        // row t of the weight tile; codes rows are 32 B, 32-byte swizzled
                        const uint32_t crow = codes + t * 32;
                        const uint32_t sw = (t >> 2) & 1;
                        const uint32_t wrow = wt + t * 128;
                        dequant_block(tab, cs[t], crow + ((0 ^ sw) << 4), crow + ((1 ^ sw) << 4),
                                      [&](int j) { return wrow + ((static_cast<uint32_t>(j) ^ (t & 7)) << 4); });
                    } else {
                        // weight row nl (reduction index), k-block a of the 4 in the tile
                        const int nl = t & 63, a = t >> 6;
                        const uint32_t crow = codes + nl * 128;
                        const uint32_t sw = nl & 7;
                        const uint32_t dst = wt + a * 8192 + (nl >> 3) * 1024 + (nl & 7) * 128;
                        dequant_block(tab, cs[a * 64 + nl], crow + (((2 * a) ^ sw) << 4),
                                      crow + (((2 * a + 1) ^ sw) << 4),
                                      [&](int j) { return dst + ((static_cast<uint32_t>(j) ^ sw) << 4); });
                    }
                    fence_proxy_async_smem();  // this thread's tile stores -> visible to the tensor core
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(deq + s);
            }
            if (!ok) *abort_flag = 1;

            // ------------------------------------------ segment epilogue --
            const bool acc_ok = __all_sync(0xFFFFFFFFu, mbar_wait(acc, static_cast<uint32_t>(seg) & 1u, tmo, args.status));
            tc_fence_after();
            const bool good = __all_sync(0xFFFFFFFFu, acc_ok && !*abort_flag);
            const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16) + h * 256;
            // A partial tile is private scratch laid out for the epilogue
            // threads: float4 i of 32-column chunk c of thread t lives at
            // ((c * 8 + i) * 256 + t), so each warp instruction moves 512
            // contiguous bytes.
            const int64_t tile_floats = static_cast<int64_t>(kFusedBM) * kFusedBN;
            if (kSplit && !it.owner()) {
                // contributor: the fp32 partial tile, then the flag
                float4* my_part = reinterpret_cast<float4*>(args.part + static_cast<int64_t>(cta) * tile_floats) + t;
                const bool live = m0 + row_l < args.M;  // rows past M are never read back
                for (int c = 0; c < kFusedBN / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(trow + 32 * c, r);
                    tmem_ld_wait();
                    if (good && live) {
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            my_part[(c * 8 + i) * 256] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                                                     __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(tmem_free);
                __threadfence();
                epi_bar();
                if (t == 0 && good) st_release(args.flags + cta, 1);
            } else {
                // owner: wait for the contributors of the tile's earlier steps
                const int first = (kSplit && it.k_lo > 0) ? sc.cta_of(it.tile * KT) : cta;
                const int last = cta - 1;
                if (first <= last) {  // only a split tile waits and fences
                if (t == 0) {
                    int okp = good ? 1 : 0;
                    const uint64_t t0 = global_timer_ns();
                    for (int cc = first; cc <= last && okp; ++cc) {
                        while (ld_acquire(args.flags + cc) == 0) {
                            if (global_timer_ns() - t0 > tmo) {
                                atomicOr(args.status, kStatusTimeout);
                                okp = 0;
                                break;
                            }
                        }
                    }
                    *parts_ok = okp;
                }
                epi_bar();
                __threadfence();
                }
                const bool write = good && (first > last || *parts_ok);
                const int64_t row = m0 + row_l;
                // 2 KB scratch of this warp in stage 0's weight region, idle now
                const uint32_t scratch = smem_u32(smem + kOffW) + warp * 2048;
                for (int c = 0; c < kFusedBN / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(trow + 32 * c, r);
                    tmem_ld_wait();
                    if (write && row < args.M) {
                        float v[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
                        for (int cc = first; cc <= last; ++cc) {
                            const float4* src =
                                reinterpret_cast<const float4*>(args.part + static_cast<int64_t>(cc) * tile_floats) + t;
                            float4 pv[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i) pv[i] = __ldcg(src + (c * 8 + i) * 256);
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                v[4 * i] += pv[i].x;
                                v[4 * i + 1] += pv[i].y;
                                v[4 * i + 2] += pv[i].z;
                                v[4 * i + 3] += pv[i].w;
                            }
                        }
                        // this row's 32 columns as bf16 into the warp's scratch:
                        // 64-byte rows, 16-byte pieces XOR-swizzled by the row
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const uint32_t w4[4] = {pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                                                    pack_bf16x2(v[8 * j + 4], v[8 * j + 5]),
                                                    pack_bf16x2(v[8 * j + 6], v[8 * j + 7])};
                            sts128(scratch + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4), w4);
                        }
                    }
                    __syncwarp();
                    if (write) {
                        // whole 64-byte row segments: 8 rows of the warp per store
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int rr = 8 * i + (lane >> 2), pc = lane & 3;
                            const int64_t orow = m0 + row_l - lane + rr;
                            const int64_t ocol = n0 + 32 * c + 8 * pc;
                            const uint4 d = lds128(scratch + rr * 64 + ((pc ^ ((rr >> 1) & 3)) << 4));
                            if (orow < args.M && ocol < tc.n_lim)
                                *reinterpret_cast<uint4*>(args.out + orow * args.out_cols + ocol) = d;
                        }
                    }
                    __syncwarp();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(tmem_free);
            }
            ++seg;
            if (!ok) break;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    // launched as a programmatic dependent, the grid completes only after its
    // primary (and so after everything that one waited for); otherwise a no-op
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---------------------------------------------------------------------------
// CTA pairs (whole tiles). Two CTAs of a cluster take the same 256-column
// weight tile and two neighbouring 256-row activation tiles. Each
// dequantises only its half of the weight tile (128 of its N rows; for dX 128
// of its output columns, 16 KB either way) into its own shared memory, and one
// thread then copies that half into the partner's weight stage with a bulk
// shared-to-shared copy that completes on the partner's barrier as
// transaction bytes; every weight tile is decoded once per pair instead of
// once per CTA. Each CTA runs the same cta_group::1 UMMAs on its own full
// copy.
//
// Three rings: activation tiles (3 stages, loaded by one producer lane),
// this CTA's half of the packed codes and constants (6 stages, another lane,
// so codes arrive far ahead of their use) and decoded weight tiles (3
// stages). The dequantiser warps form two groups that take the steps in
// turn. A weight stage is rewritten only when both CTAs' UMMAs have consumed
// it (multicast commit), because the partner copies into it; the rank-r
// weight tile of a rank step is loaded into the weight stage by the group
// that owns the step.
// ---------------------------------------------------------------------------
constexpr int kPA = 3, kPW = 3, kPC = 6;                 // ring depths: activations, weights, codes
constexpr uint32_t kPCodeBytes = 4096;                    // this CTA's half of a step's codes
constexpr uint32_t kPCStage = kPCodeBytes + 1024;         // + its half of the constants (512 B used)
constexpr uint32_t kPOffW = kPA * kActBytes;              // 96 KB
constexpr uint32_t kPOffCodes = kPOffW + kPW * kWBytes;   // 192 KB
constexpr uint32_t kPBarOffset = kPOffCodes + kPC * kPCStage;
constexpr uint32_t kPSmemBytes = kPBarOffset + 512 + 1024;

template <bool kTransW>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kFusedThreads, 1)
    fused_nf4_gemm_pair(const __grid_constant__ CUtensorMap tm_act, const __grid_constant__ CUtensorMap tm_codes,
                        const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_lact,
                        const __grid_constant__ CUtensorMap tm_lw, const FusedArgs args, const Nf4Tables tab) {
    asm volatile("griddepcontrol.launch_dependents;");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* a_full = reinterpret_cast<uint64_t*>(smem + kPBarOffset);
    uint64_t* a_empty = a_full + kPA;
    uint64_t* w_full = a_empty + kPA;
    uint64_t* w_empty = w_full + kPW;
    uint64_t* c_full = w_empty + kPW;
    uint64_t* c_empty = c_full + kPC;
    uint64_t* acc = c_empty + kPC;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank(), peer = rank ^ 1u;
    const int KT = static_cast<int>((args.red + kFusedBK - 1) / kFusedBK);
    int tiles_n = 0;
    {
        int64_t start = 0;
        for (int g = 0; g < args.ngroups; ++g) {
            tiles_n += static_cast<int>((args.group_end[g] - start + kFusedBN - 1) / kFusedBN);
            start = args.group_end[g];
        }
    }
    // the pair's column tile and this CTA's row tile, column-major: the row
    // pairs of one column tile are neighbours, run in the same wave and share
    // its packed codes through L2 (the second row tile of the last row pair
    // may lie past M: its rows are zero-filled and never written)
    const int pair = blockIdx.x >> 1;
    const int pairs_m = static_cast<int>((args.M + 2 * kFusedBM - 1) / (2 * kFusedBM));
    const int64_t m0 = (static_cast<int64_t>(pair % pairs_m) * 2 + rank) * kFusedBM;
    const TileCols tc = tile_cols(args, pair / pairs_m);
    const int64_t n0 = tc.n0;
    const int rank_steps = args.rank_cols > 0 ? args.rank_steps : 0;
    const int steps = KT + rank_steps;
    const uint64_t tmo = args.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPA; ++s) {
            mbar_init(a_full + s, 1);
            mbar_init(a_empty + s, 1);   // this CTA's UMMAs
        }
        for (int s = 0; s < kPW; ++s) {
            mbar_init(w_full + s, 4);    // the owning group's 4 warps (+ the partner's half as bytes)
            mbar_init(w_empty + s, 2);   // both CTAs' UMMAs
        }
        for (int s = 0; s < kPC; ++s) {
            mbar_init(c_full + s, 1);
            mbar_init(c_empty + s, 4);   // the consuming group's 4 warps
        }
        mbar_init(acc, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (warp == 8 && lane == 0) {
        tma_prefetch_desc(&tm_act);
        tma_prefetch_desc(&tm_codes);
        tma_prefetch_desc(&tm_c);
        tma_prefetch_desc(&tm_lact);
        tma_prefetch_desc(&tm_lw);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_sync();  // the partner's barriers are initialised before any remote copy
    const uint32_t tmem = *tmem_slot;

    if (warp == 8) {
        // --------------------------------------------------- producers --
        if (lane == 0 && !args.stall_producer) {
            // activation tiles (X or dY; sT or sU in the rank steps), 3 ahead
            int last = -1;
            for (int i = 0; i < steps; ++i) {
                const int s = i % kPA;
                const uint32_t u = static_cast<uint32_t>(i / kPA);
                if (i >= kPA && !mbar_wait(a_empty + s, (u - 1) & 1u, tmo, args.status)) {
                    *abort_flag = 1;
                    break;
                }
                if (*abort_flag) break;
                uint8_t* st = smem + s * kActBytes;
                mbar_arrive_expect_tx(a_full + s, kActBytes);
                if (i < KT) {
                    tma_load_2d(st, &tm_act, a_full + s, i * kFusedBK, static_cast<int>(m0));
                } else {
                    const int c = i - KT;
                    if (c == 0) asm volatile("griddepcontrol.wait;" ::: "memory");  // sT / sU of the preceding launch
                    tma_load_2d(st, &tm_lact, a_full + s, tc.rank_x + 64 * c, static_cast<int>(m0));
                }
                last = i;
            }
            for (int i = max(0, last - kPA + 1); i <= last; ++i)
                mbar_wait(a_full + i % kPA, static_cast<uint32_t>(i / kPA) & 1u, tmo, nullptr);
        } else if (lane == 1 && !args.stall_producer) {
            // this CTA's half of the codes and constants, 6 ahead
            int last = -1;
            for (int i = 0; i < KT; ++i) {
                const int s = i % kPC;
                const uint32_t u = static_cast<uint32_t>(i / kPC);
                if (i >= kPC && !mbar_wait(c_empty + s, (u - 1) & 1u, tmo, args.status)) {
                    *abort_flag = 1;
                    break;
                }
                if (*abort_flag) break;
                uint8_t* st = smem + kPOffCodes + s * kPCStage;
                mbar_arrive_expect_tx(c_full + s, kPCodeBytes + 512);
                if (!kTransW) {
                    tma_load_2d(st, &tm_codes, c_full + s, i * (kFusedBK / 2),
                                static_cast<int>(n0) + 128 * static_cast<int>(rank));
                    tma_load_2d(st + kPCodeBytes, &tm_c, c_full + s, static_cast<int>(n0) + 128 * static_cast<int>(rank),
                                i);
                } else {
                    tma_load_2d(st, &tm_codes, c_full + s, static_cast<int>(n0 / 2) + 64 * static_cast<int>(rank),
                                i * kFusedBK);
                    tma_load_2d(st + kPCodeBytes, &tm_c, c_full + s, i * kFusedBK,
                                static_cast<int>(n0 / kBlock) + 2 * static_cast<int>(rank));
                }
                last = i;
            }
            for (int i = max(0, last - kPC + 1); i <= last; ++i)
                mbar_wait(c_full + i % kPC, static_cast<uint32_t>(i / kPC) & 1u, tmo, nullptr);
        }
        __syncwarp();
    } else if (warp == 9) {
        // ----------------------------------------------------------- MMA --
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, kFusedBN, false, kTransW);
            bool ok = true;
            tc_fence_after();
            for (int i = 0; i < steps; ++i) {
                const int sa = i % kPA, sw = i % kPW;
                if (!mbar_wait(a_full + sa, static_cast<uint32_t>(i / kPA) & 1u, tmo, args.status) ||
                    !mbar_wait_cluster(w_full + sw, static_cast<uint32_t>(i / kPW) & 1u, tmo, args.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t act = smem_u32(smem + sa * kActBytes);
                const uint32_t wt = smem_u32(smem + kPOffW + sw * kWBytes);
                const int ksub = (i < KT) ? (kFusedBK / 16) : (min(64, args.rank_cols - 64 * (i - KT)) + 15) / 16;
                for (int kk = 0; kk < ksub; ++kk) {
                    const uint64_t bdesc = kTransW ? sw128_desc(wt + kk * 2048, 8192, 1024)
                                                   : sw128_desc(wt + kk * 32, 16, 1024);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint64_t adesc = sw128_desc(act + h * 16384 + kk * 32, 16, 1024);
                        umma_f16(tmem + h * 256, adesc, bdesc, idesc, (i > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                umma_commit(a_empty + sa);
                umma_commit_multicast(w_empty + sw, 0x3);  // the weight stage is free in both CTAs' view
            }
            umma_commit(acc);  // arrives once every UMMA has completed (also after an abort)
            if (!ok) {
                *abort_flag = 1;
                __threadfence_block();
            }
        }
        __syncwarp();
    } else {
        // ------------------------------- dequantise half tiles, then epilogue --
        // group G (warps 4G .. 4G + 3) takes the steps i with i % 2 == G;
        // thread tl decodes N row 128 rank + tl (forward) or output-column
        // block 2 rank + tl / 64, reduction row tl % 64 (dX)
        const int G = warp >> 2, tl = (warp & 3) * 32 + lane;
        const bool leader = (warp & 3) == 0 && lane == 0;
        const uint32_t w_full_remote = mapa_shared(smem_u32(w_full), peer);
        constexpr uint32_t kHalf = kWBytes / 2;  // this CTA's half of the weight tile
        bool ok = true;
        for (int i = G; ok && i < steps; i += 2) {
            const int sw = i % kPW;
            // both CTAs' UMMAs are done with the weight stage's previous use
            if (i >= kPW)
                ok = __all_sync(0xFFFFFFFFu, mbar_wait_cluster(w_empty + sw, static_cast<uint32_t>(i / kPW - 1) & 1u,
                                                               tmo, args.status));
            if (!ok) break;
            uint8_t* wst = smem + kPOffW + sw * kWBytes;
            const uint32_t wt = smem_u32(wst);
            if (i < KT) {
                const int sc = i % kPC;
                ok = __all_sync(0xFFFFFFFFu, mbar_wait(c_full + sc, static_cast<uint32_t>(i / kPC) & 1u, tmo,
                                                       args.status));
                if (!ok) break;
                uint8_t* cst = smem + kPOffCodes + sc * kPCStage;
                const uint32_t codes = smem_u32(cst);
                const float* cs = reinterpret_cast<const float*>(cst + kPCodeBytes);
                uint32_t c0, c1, dst;
                float cprime;
                int swz;
                if (!kTransW) {
                    // codes rows are 32 B, 32-byte swizzled; W row n = 128 rank + tl
                    const uint32_t crow = codes + tl * 32;
                    const uint32_t sw32 = (tl >> 2) & 1;
                    c0 = crow + ((0 ^ sw32) << 4);
                    c1 = crow + ((1 ^ sw32) << 4);
                    const int n = 128 * static_cast<int>(rank) + tl;
                    dst = static_cast<uint32_t>(n) * 128u;
                    swz = n & 7;
                    cprime = cs[tl];
                } else {
                    // codes rows are 64 B (this CTA's 128 output columns), 64-byte swizzled
                    const int nl = tl & 63, al = tl >> 6, a = 2 * static_cast<int>(rank) + al;
                    const uint32_t crow = codes + nl * 64;
                    const uint32_t sw64 = (nl >> 1) & 3;
                    c0 = crow + (((2 * al) ^ sw64) << 4);
                    c1 = crow + (((2 * al + 1) ^ sw64) << 4);
                    dst = static_cast<uint32_t>(a * 8192 + (nl >> 3) * 1024 + (nl & 7) * 128);
                    swz = nl & 7;
                    cprime = cs[al * 64 + nl];
                }
                const Nf4BlockLut lutb = make_block_lut(tab.level, cprime);
                const uint4 ca = lds128(c0), cb = lds128(c1);
                __syncwarp();
                if (lane == 0) mbar_arrive(c_empty + sc);  // the codes stage has been read
                const uint32_t words[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint32_t o[4];
                    lut_decode8(lutb, words[j], o);
                    sts128(wt + dst + ((static_cast<uint32_t>(j) ^ static_cast<uint32_t>(swz)) << 4), o);
                }
                fence_proxy_async_smem();  // -> visible to the tensor core and the bulk copy
                // the group's half is complete: one thread sends it to the partner
                asm volatile("bar.sync %0, 128;" ::"r"(2 + G) : "memory");
                if (leader) {
                    mbar_arrive_expect_tx(w_full + sw, kHalf);  // the partner's half, coming the same way
                    bulk_copy_to_cluster(mapa_shared(wt + kHalf * rank, peer), wt + kHalf * rank, kHalf,
                                         w_full_remote + static_cast<uint32_t>(sw) * 8u);
                } else if (lane == 0) {
                    mbar_arrive(w_full + sw);
                }
            } else {
                // rank step: the rank-r weight tile straight into the weight stage
                if (leader) {
                    const int c = i - KT;
                    mbar_arrive_expect_tx(w_full + sw, kWBytes);
                    if (!kTransW) {
                        tma_load_2d(wst, &tm_lw, w_full + sw, 64 * c, static_cast<int>(n0));
                    } else {
                        for (int a = 0; a < 4; ++a)
                            tma_load_2d(wst + a * 8192, &tm_lw, w_full + sw, static_cast<int>(n0) + 64 * a, 64 * c);
                    }
                } else if (lane == 0) {
                    mbar_arrive(w_full + sw);
                }
            }
        }
        if (!ok) *abort_flag = 1;

        // ------------------------------------------------------ epilogue --
        const int q = warp & 3, h = warp >> 2;
        const int row_l = h * 128 + q * 32 + lane;
        const bool acc_ok = __all_sync(0xFFFFFFFFu, mbar_wait(acc, 0u, tmo, args.status));
        tc_fence_after();
        const bool write = __all_sync(0xFFFFFFFFu, acc_ok && !*abort_flag);
        const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16) + h * 256;
        const int64_t row = m0 + row_l;
        // 2 KB scratch of this warp in the first activation stage, idle now
        // (every UMMA has completed and every activation copy has landed)
        const uint32_t scratch = smem_u32(smem) + warp * 2048;
        for (int c = 0; c < kFusedBN / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(trow + 32 * c, r);
            tmem_ld_wait();
            if (write && row < args.M) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t w4[4] = {pack_bf16x2(__uint_as_float(r[8 * j]), __uint_as_float(r[8 * j + 1])),
                                            pack_bf16x2(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3])),
                                            pack_bf16x2(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5])),
                                            pack_bf16x2(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7]))};
                    sts128(scratch + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4), w4);
                }
            }
            __syncwarp();
            if (write) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int rr = 8 * i + (lane >> 2), pc = lane & 3;
                    const int64_t orow = m0 + row_l - lane + rr;
                    const int64_t ocol = n0 + 32 * c + 8 * pc;
                    const uint4 d = lds128(scratch + rr * 64 + ((pc ^ ((rr >> 1) & 3)) << 4));
                    if (orow < args.M && ocol < tc.n_lim)
                        *reinterpret_cast<uint4*>(args.out + orow * args.out_cols + ocol) = d;
                }
            }
            __syncwarp();
        }
        tc_fence_before();
    }

    tc_fence_before();
    __syncthreads();
    // the partner may still copy into this CTA's shared memory until it has
    // passed its own main loop
    cluster_sync();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");  // as in fused_nf4_gemm
}

template <bool kTransW>
cudaError_t launch_fused(const CUtensorMap& act, const CUtensorMap& codes, const CUtensorMap& cT,
                         const CUtensorMap& lact, const CUtensorMap& lw, const FusedArgs& a, const Nf4Tables& tab,
                         bool pdl, cudaStream_t st) {
    // the highest scheduling priority: work overlapping this launch only
    // takes SMs its tiles leave idle
    int least = 0, greatest = 0;
    cudaError_t e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(a.ctas));
    cfg.blockDim = dim3(kFusedThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    const int64_t tiles = a.tiles > 0 ? a.tiles : fused_tiles(a.M, fused_tiles_n(a));
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributePriority;
    attr[0].val.priority = greatest;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    if (static_cast<int64_t>(a.ctas) == tiles)
        return cudaLaunchKernelEx(&cfg, fused_nf4_gemm<kTransW, false>, act, codes, cT, lact, lw, a, tab);
    return cudaLaunchKernelEx(&cfg, fused_nf4_gemm<kTransW, true>, act, codes, cT, lact, lw, a, tab);
}

template <bool kTransW>
cudaError_t launch_pair(const CUtensorMap& act, const CUtensorMap& codes, const CUtensorMap& cT,
                        const CUtensorMap& lact, const CUtensorMap& lw, const FusedArgs& a, const Nf4Tables& tab,
                        bool pdl, cudaStream_t st) {
    int least = 0, greatest = 0;
    cudaError_t e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
    if (e != cudaSuccess) return e;
    const int64_t tiles_m = (a.M + kFusedBM - 1) / kFusedBM;
    if (a.ctas <= 0 || (a.ctas & 1) || a.ctas > 2 * fused_tiles_n(a) * ((tiles_m + 1) / 2) || a.tile_first != 0)
        return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(a.ctas));
    cfg.blockDim = dim3(kFusedThreads);
    cfg.dynamicSmemBytes = kPSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributePriority;
    attr[0].val.priority = greatest;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, fused_nf4_gemm_pair<kTransW>, act, codes, cT, lact, lw, a, tab);
}

}  // namespace

size_t fused_smem_bytes() { return kSmemBytes; }

cudaError_t launch_fused_pair_fwd(const CUtensorMap& act, const CUtensorMap& codes_half, const CUtensorMap& cT_half,
                                  const CUtensorMap& lora_act, const CUtensorMap& lora_w, const FusedArgs& a,
                                  const Nf4Tables& tab, bool pdl, cudaStream_t st) {
    return launch_pair<false>(act, codes_half, cT_half, lora_act, lora_w, a, tab, pdl, st);
}

cudaError_t launch_fused_pair_dx(const CUtensorMap& act, const CUtensorMap& codes_half, const CUtensorMap& cT_half,
                                 const CUtensorMap& lora_act, const CUtensorMap& lora_w, const FusedArgs& a,
                                 const Nf4Tables& tab, bool pdl, cudaStream_t st) {
    return launch_pair<true>(act, codes_half, cT_half, lora_act, lora_w, a, tab, pdl, st);
}

cudaError_t fused_init_device() {
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(fused_nf4_gemm<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(kSmemBytes))) != cudaSuccess ||
        (e = cudaFuncSetAttribute(fused_nf4_gemm<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(kSmemBytes))) != cudaSuccess ||
        (e = cudaFuncSetAttribute(fused_nf4_gemm<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(kSmemBytes))) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(fused_nf4_gemm<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(kSmemBytes))) != cudaSuccess ||
        (e = cudaFuncSetAttribute(fused_nf4_gemm_pair<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(kPSmemBytes))) != cudaSuccess)
        return e;
    return cudaFuncSetAttribute(fused_nf4_gemm_pair<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(kPSmemBytes));
}

cudaError_t launch_fused_fwd(const CUtensorMap& act, const CUtensorMap& codes, const CUtensorMap& cT,
                             const CUtensorMap& lora_act, const CUtensorMap& lora_w, const FusedArgs& a,
                             const Nf4Tables& tab, bool pdl, cudaStream_t st) {
    return launch_fused<false>(act, codes, cT, lora_act, lora_w, a, tab, pdl, st);
}

cudaError_t launch_fused_dx(const CUtensorMap& act, const CUtensorMap& codes, const CUtensorMap& cT,
                            const CUtensorMap& lora_act, const CUtensorMap& lora_w, const FusedArgs& a,
                            const Nf4Tables& tab, bool pdl, cudaStream_t st) {
    return launch_fused<true>(act, codes, cT, lora_act, lora_w, a, tab, pdl, st);
}

}  // namespace qlora
