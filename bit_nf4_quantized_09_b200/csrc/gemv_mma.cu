// Small-batch forward for up to 64 tokens: Y = X . deq(W)^T + sT . B^T.
//
// With a few tokens every weight is used a few times only, so the step is
// bound by streaming the packed weight (about half a byte per weight);
// "ta-paperlens QLoRA explainer", 落とし穴, names this small-batch regime as
// the one where 4-bit weights pay off. The kernel is shaped so that the
// decode and its bookkeeping stay a few instructions per weight: per two
// weights one byte permute and one shared-memory load from a table.
//
// Factored dequantisation. Within a 64-weight block every weight is
// level[code] * c'_b, so for output row n
//   Y[m, n] = sum_b c'_{n,b} * sum_{k in b} level[code_{n,k}] * X[m, k].
// The inner sums run on the tensor core (mma.m16n8k16, bf16 operands, fp32
// accumulation) over the unscaled levels rounded to bf16, one block at a time
// into a zeroed fragment; c'_{n,b} (fp32) is applied with one FMA per
// accumulator per block. The weight the product sees is bf16(level) * c', not
// the exactly dequantised bf16(level * c'): at most 2^-8 relative apart per
// weight, far inside the forward's tolerance.
//
// Decoding. A code byte holds two consecutive weights (the first in the high
// nibble), so one 256-entry table of bf16 pairs turns a byte into the 32-bit
// operand register of two weights. The table lives in shared memory with one
// copy per lane (entry e of lane l at byte 256 e + 4 l): every lookup of a
// warp hits 32 distinct banks, and the offset 256 e + 4 l is a single byte
// permute of the code word and 4 l, so a lookup is that permute and a
// shared-memory load at the offset from the table's address. The other 128
// bytes of each 256-byte entry hold the stages' block constants.
//
// Data movement. A producer warp stages, per pipeline step of four block
// columns (aligned: the step's first column is a multiple of four), the
// packed codes of the CTA's 256 weight rows (one 128 x 256-byte TMA box:
// 128 contiguous bytes of every row, so each DRAM access is a whole line;
// 128-byte swizzle) and the matching X columns of every token (one 64 x M
// box per block column, 128-byte swizzle) into a ring of stages guarded by
// mbarriers; every wait is bounded. Four producer warps take the steps in
// turn: each issues its step's copies and decodes the step's block constants
// c' (E4M3 code, second-level scale and mean, or the fp32 constant; every
// load issued before the first use) beside the table, so four steps' load
// latencies overlap and a consumer reads the four constants of a row with
// one 16-byte load. Since steps are aligned, a row's four constants of a step
// are one aligned 4-byte word (or float4) when K/64 is a multiple of four, so
// each row costs one load, not four scattered ones.
//
// Fragment layout. A consumer warp owns 32 weight rows as two 16-row MMA
// tiles, which share every X fragment it loads. In each tile, lane (g, q)
// reads the 8 code bytes 8q .. 8q + 7 of each block of two rows, its
// fragment rows g and g + 8 (tile rows frag_row(g) and frag_row(g) + 8, an
// order chosen so that the code loads meet no bank conflict).
// Inside MMA step s (0..3) of a block its A-operand slots 2q, 2q + 1 hold
// weights 16q + 4s, +1 (code byte 8q + 2s) and slots 2q + 8, 2q + 9 hold
// weights 16q + 4s + 2, +3 (byte 8q + 2s + 1); its X fragment uses the same
// order, X[m][16q .. 16q + 15] of the block (two swizzled 16-byte chunks),
// loaded only by lanes of existing tokens (with one token, 4 lanes of 32:
// every quarter-warp phase of a 16-byte load costs a shared-memory
// wavefront, so loads of columns that are never written are left out).
//
// Work split. A CTA of 8 consumer warps owns 256 weight rows; the (row tile,
// block column) units are dealt out in equal contiguous ranges, one per CTA,
// one CTA per SM (stream-K), so no wave is left part-empty; a range may cross
// into the next row tile. Every CTA that touches a tile writes its fp32
// partial sums for it; the last one to finish (atomic ticket, no waiting)
// adds them in CTA order, adds the rank-r term and writes Y in bf16. The
// rank-r input sT comes from the preceding launch; the kernel may be launched
// as its programmatic dependent and waits for it (griddepcontrol.wait) only
// in that epilogue, so the weight stream overlaps the down-projection.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace qlora {

namespace {

constexpr int kTilesW = 2;                    // 16-row MMA tiles per consumer warp (sharing its X fragments)
constexpr int kWarps = 16 / kTilesW;          // consumer warps
constexpr int kProdWarps = 4;                 // producer warps: TMA (one lane) and the block constants
constexpr int kThreads = (kWarps + kProdWarps) * 32;
constexpr int kRowsCta = kWarps * 16 * kTilesW;  // 256 weight rows
constexpr int kStep = 4;                      // block columns per pipeline step
constexpr int kMaxStages = 6;  // at most 8: the constants of 8 stages fill the table's free halves
// The pair table: entry e at byte 256 e, its 32 lane copies in the first 128
// bytes; the second 128 bytes of the entries hold the stages' block constants.
constexpr uint32_t kLutBytes = 256 * 256;
constexpr uint32_t kCodeStage = 32 * kStep * kRowsCta;  // 128 contiguous bytes of each of the 256 rows

__host__ __device__ constexpr uint32_t x_box_bytes(int64_t M) {
    return static_cast<uint32_t>((M * 128 + 1023) / 1024 * 1024);  // 1024-aligned for the 128-byte swizzle
}
__host__ __device__ constexpr uint32_t stage_bytes(int64_t M) {
    return kCodeStage + kStep * x_box_bytes(M);
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void consumer_bar() { asm volatile("bar.sync 1, %0;" ::"n"(kWarps * 32) : "memory"); }

// The bf16 pair of code byte k of w, from this lane's copy of the table at
// `base`: one byte permute forms the offset 256 e + 4 lane (e in byte 1,
// lane4 = 4 lane in byte 0) and the load adds the table's address.
__device__ __forceinline__ uint32_t lut(uint32_t base, uint32_t lane4, uint32_t w, uint32_t k) {
    return lds32(base + __byte_perm(w, lane4, 0x5504u + (k << 4)));
}

// Address of the block constants (4 x fp32) of weight row r (0..255) of
// stage s, in the free half of table entry 32 s + r / 8.
__device__ __forceinline__ uint32_t const_addr(uint32_t base, int s, int r) {
    return base + static_cast<uint32_t>(32 * s + (r >> 3)) * 256u + 128u + static_cast<uint32_t>(r & 7) * 16u;
}

// The rank-r term of two 8-row halves of a warp's 16 rows, added to the
// warp's accumulators: for each 16-column rank step, A fragment = the rows'
// B entries (row g in slots 0 and 2, row g + 8 in slots 1 and 3), X fragment =
// the tokens' sT entries at the rows' sT columns; columns from `cols` on read
// as zero. `use_a` / `use_b` keep one half (the other's A slots zero) when the
// two halves read different sT columns (projections of a group).
template <int MT>
__device__ __forceinline__ void rank_mma(const GemvMmaArgs& a, float (&acc)[MT][4], int64_t rowA, int64_t rowB,
                                         int col, bool use_a, bool use_b, int g, int q) {
    const int cols = a.rank_cols, M = static_cast<int>(a.M);
    const uint16_t* bA = a.B + rowA * a.B_ld;
    const uint16_t* bB = a.B + rowB * a.B_ld;
    for (int k0 = 0; k0 < cols; k0 += 16) {
        const int j0 = k0 + 2 * q, j1 = j0 + 8;
        uint32_t af[4];
        af[0] = use_a && j0 < cols ? __ldg(reinterpret_cast<const uint32_t*>(bA + j0)) : 0u;
        af[1] = use_b && j0 < cols ? __ldg(reinterpret_cast<const uint32_t*>(bB + j0)) : 0u;
        af[2] = use_a && j1 < cols ? __ldg(reinterpret_cast<const uint32_t*>(bA + j1)) : 0u;
        af[3] = use_b && j1 < cols ? __ldg(reinterpret_cast<const uint32_t*>(bB + j1)) : 0u;
#pragma unroll
        for (int t = 0; t < MT; ++t) {
            const int m = min(8 * t + g, M - 1);  // tokens past M: copies, never written
            const uint16_t* xs = a.sT + static_cast<int64_t>(m) * a.sT_ld + col;
            const uint32_t x0 = j0 < cols ? __ldg(reinterpret_cast<const uint32_t*>(xs + j0)) : 0u;
            const uint32_t x1 = j1 < cols ? __ldg(reinterpret_cast<const uint32_t*>(xs + j1)) : 0u;
            mma_bf16(acc[t], af, x0, x1);
        }
    }
}

// Column of sT holding the rank-r input of output row n.
__device__ __forceinline__ int rank_col(const GemvMmaArgs& a, int64_t n) {
    for (int g = 0; g < a.ngroups - 1; ++g)
        if (n < a.group_end[g]) return a.group_rank_x[g];
    return a.group_rank_x[a.ngroups - 1];
}

// The work is the list of (row tile, NF4 block column) units in tile-major
// order, U = tiles * KB; CTA c takes units [c U / P, (c + 1) U / P) (stream-K).
// With P >= tiles a range touches at most two row tiles: its segments. The
// CTAs that touch a tile are consecutive, so a segment's partial-sum slot is
// its CTA index minus that of the tile's first CTA.
struct Sched {
    int U, P, KB;  // U < 2^31 and P >= tiles are ensured on the host
    __device__ int cta_of(int unit) const {
        return static_cast<int>((static_cast<int64_t>(unit + 1) * P - 1) / U);
    }
    __device__ int slot(int tile, int c) const { return c - cta_of(tile * KB); }
    __device__ int parts(int tile) const { return cta_of(min((tile + 1) * KB, U) - 1) - cta_of(tile * KB) + 1; }
};

// Pipeline steps are the aligned groups of kStep block columns (first column
// a multiple of kStep) that meet a segment's column range; step k of a CTA's
// range: its segment, first block column and the blocks [b0, b1) of the step
// inside the segment (the first and last step of a segment may be partial).
struct Step {
    int seg, col0, b0, b1;
};
__device__ __forceinline__ int steps_in(int lo, int hi) { return (hi + kStep - 1) / kStep - lo / kStep; }
__device__ __forceinline__ Step step_of(int k, int nst0, int blo0, int len0, int len1) {
    Step s;
    s.seg = k >= nst0 ? 1 : 0;
    const int lo = s.seg ? 0 : blo0, hi = s.seg ? len1 : blo0 + len0;
    s.col0 = (lo / kStep + (s.seg ? k - nst0 : k)) * kStep;
    s.b0 = max(lo - s.col0, 0);
    s.b1 = min(hi - s.col0, kStep);
    return s;
}

// Warp-local weight row of MMA fragment row g (0..7; g + 8 maps to this + 8).
// Lanes 0-15 (g < 4) then read rows 0, 2, 4, 6 and lanes 16-31 rows 1, 3, 5, 7,
// whose 128-byte-swizzled chunk pairs are disjoint: a half-warp's 8-byte code
// loads meet no bank twice.
__device__ __forceinline__ int frag_row(int g) { return ((g & 3) << 1) | (g >> 2); }

template <int MT, bool kNoDq>
__global__ void __launch_bounds__(kThreads, 1)
    gemv_mma_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_x,
                    const GemvMmaArgs a, const Nf4Tables tab) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    // the table first (16-byte alignment suffices), then the stages on a
    // 1024-byte boundary for the 128-byte swizzle
    uint8_t* stages_mem =
        reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw + kLutBytes) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[kMaxStages], empty[kMaxStages];
    __shared__ int last_of[2];
    __shared__ float levels[16];
    __shared__ volatile int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int M = static_cast<int>(a.M);
    const int N = static_cast<int>(a.N), KB = static_cast<int>(a.K / kBlock);
    const Sched sc{static_cast<int>(a.units), static_cast<int>(gridDim.x), KB};
    const int c = blockIdx.x;
    const int u0 = static_cast<int>(static_cast<int64_t>(c) * sc.U / sc.P);
    const int u1 = static_cast<int>(static_cast<int64_t>(c + 1) * sc.U / sc.P);
    const int t0 = u0 / KB;
    // segment 0: tile t0, block columns [blo0, blo0 + len0); segment 1 (if
    // the range crosses a tile boundary): tile t0 + 1, columns [0, len1)
    const int blo0 = u0 - t0 * KB;
    const int len0 = min(u1, (t0 + 1) * KB) - u0;
    const int len1 = u1 - u0 - len0;
    const int nst0 = steps_in(blo0, blo0 + len0), nst = nst0 + (len1 > 0 ? steps_in(0, len1) : 0);
    const int S = a.stages;
    const uint32_t xbox = x_box_bytes(M), stage = stage_bytes(M);
    const uint32_t lut_base = smem_u32(smem_raw);
    const uint32_t st_base = smem_u32(stages_mem);
    const uint64_t tmo = a.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full + s, 32);       // one arrive per lane of the step's producer warp
            mbar_init(empty + s, kWarps);  // one arrive per consumer warp
        }
        abort_flag = 0;
#pragma unroll
        for (int k = 0; k < 16; ++k) levels[k] = tab.level[k];
        fence_mbar_init();
    }
    __syncthreads();

    if (warp >= kWarps) {
        // ----------------------------------------------------- producers --
        if (warp == kWarps && lane == 0) {
            tma_prefetch_desc(&tm_codes);
            tma_prefetch_desc(&tm_x);
        }
        const float mean = kNoDq ? 0.0f : __ldg(a.mean);
        const uint32_t tx = kCodeStage + kStep * static_cast<uint32_t>(M) * 128u;
        const int pw = warp - kWarps;  // producer warp pw owns steps pw, pw + kProdWarps, ...
        constexpr int kRowsPerLane = kRowsCta / 32;
        int last_k = -1;  // this warp's last step whose copies were issued
        for (int k = pw; k < nst; k += kProdWarps) {
            const int s = k % S;
            const uint32_t u = static_cast<uint32_t>(k / S);
            if (k >= S && !__all_sync(0xFFFFFFFFu, mbar_wait_sleep(empty + s, (u - 1) & 1u, tmo, a.status))) {
                abort_flag = 1;
                break;
            }
            if (abort_flag) break;
            const Step sp = step_of(k, nst0, blo0, len0, len1);
            const int row0 = (t0 + sp.seg) * kRowsCta;
            uint8_t* st = stages_mem + s * stage;
            if (lane == 0) {
                mbar_expect_tx(full + s, tx);
                // whole steps even past a segment's end: the extra columns are
                // valid memory or zero-filled past K, and never used
                tma_load_2d(st, &tm_codes, full + s, sp.col0 * 32, row0);
#pragma unroll
                for (int b = 0; b < kStep; ++b)
                    tma_load_2d(st + kCodeStage + b * xbox, &tm_x, full + s, (sp.col0 + b) * kBlock, 0);
            }
            last_k = k;
            // the step's constants: lane l decodes rows l, l + 32, ... (clamped
            // to valid rows and columns; unused ones are never read); every
            // load is issued before the first use
            if (a.const_vec) {
                // the step's four constants of a row are one aligned word (E4M3)
                // or float4, and with double quantisation lie in one group of 256
                constexpr int kVBatch = 4;  // rows whose loads are in flight together
#pragma unroll 1
                for (int j0 = 0; j0 < kRowsPerLane; j0 += kVBatch) {
                    uint32_t qw[kVBatch];
                    float sv[kVBatch];
                    float4 av[kVBatch];
#pragma unroll
                    for (int j = 0; j < kVBatch; ++j) {
                        const int64_t ib =
                            static_cast<int64_t>(min(row0 + lane + 32 * (j0 + j), N - 1)) * KB + sp.col0;
                        if (kNoDq) {
                            av[j] = __ldg(reinterpret_cast<const float4*>(a.absmax + ib));
                        } else {
                            qw[j] = __ldg(reinterpret_cast<const uint32_t*>(a.qabsmax + ib));
                            sv[j] = __ldg(a.s2 + (ib >> 8));
                        }
                    }
#pragma unroll
                    for (int j = 0; j < kVBatch; ++j) {
                        if (!kNoDq)
                            av[j] = make_float4(__fmaf_rn(e4m3_to_f32(qw[j]), sv[j], mean),
                                                __fmaf_rn(e4m3_to_f32(qw[j] >> 8), sv[j], mean),
                                                __fmaf_rn(e4m3_to_f32(qw[j] >> 16), sv[j], mean),
                                                __fmaf_rn(e4m3_to_f32(qw[j] >> 24), sv[j], mean));
                    {
                        const float4 v = av[j];
                        sts128(const_addr(lut_base, s, lane + 32 * (j0 + j)), __float_as_uint(v.x), __float_as_uint(v.y),
                               __float_as_uint(v.z), __float_as_uint(v.w));
                    }
                    }
                }
            } else {
            constexpr int kBatch = 4;  // rows whose loads are in flight together
#pragma unroll 1
            for (int j0 = 0; j0 < kRowsPerLane; j0 += kBatch) {
                uint32_t qv[kBatch][kStep];
                float sv[kBatch][kStep];
#pragma unroll
                for (int j = 0; j < kBatch; ++j) {
                    const int64_t rb = static_cast<int64_t>(min(row0 + lane + 32 * (j0 + j), N - 1)) * KB;
#pragma unroll
                    for (int b = 0; b < kStep; ++b) {
                        const int64_t ib = rb + min(sp.col0 + b, KB - 1);
                        if (kNoDq) {
                            sv[j][b] = __ldg(a.absmax + ib);
                        } else {
                            qv[j][b] = __ldg(a.qabsmax + ib);
                            sv[j][b] = __ldg(a.s2 + (ib >> 8));
                        }
                    }
                }
#pragma unroll
                for (int j = 0; j < kBatch; ++j) {
                    float c4[kStep];
#pragma unroll
                    for (int b = 0; b < kStep; ++b)
                        c4[b] = kNoDq ? sv[j][b] : __fmaf_rn(e4m3_to_f32(qv[j][b]), sv[j][b], mean);
                    sts128(const_addr(lut_base, s, lane + 32 * (j0 + j)), __float_as_uint(c4[0]), __float_as_uint(c4[1]),
                           __float_as_uint(c4[2]), __float_as_uint(c4[3]));
                }
            }
            }
            mbar_arrive(full + s);  // release this lane's constants (the copies complete the phase)
        }
        // make sure no copy of this warp's is still landing in shared memory at exit
        if (lane == 0)
            for (int k = last_k; k >= 0 && k > last_k - S; k -= kProdWarps)
                mbar_wait(full + k % S, static_cast<uint32_t>(k / S) & 1u, tmo, nullptr);
        __syncwarp();
    } else {
        // ------------------------------------------------------ consumers --
        const int g = lane >> 2, q = lane & 3;
        const uint32_t lane4 = 4u * static_cast<uint32_t>(lane);
        // the table: entry e = bf16(level[e >> 4]) | bf16(level[e & 15]) << 16,
        // four lane copies per 16-byte store
        for (int i = threadIdx.x; i < 256 * 8; i += kWarps * 32) {
            const int e = i >> 3;
            const uint32_t v = pack_bf16x2(levels[e >> 4], levels[e & 15]);
            sts128(lut_base + static_cast<uint32_t>(e) * 256u + static_cast<uint32_t>(i & 7) * 16u, v, v, v, v);
        }
        consumer_bar();

        float acc[kTilesW][MT][4];
#pragma unroll
        for (int h = 0; h < kTilesW; ++h)
#pragma unroll
            for (int t = 0; t < MT; ++t) acc[h][t][0] = acc[h][t][1] = acc[h][t][2] = acc[h][t][3] = 0.0f;
        // X fragment rows in a stage's box: token g + 8t, chunks 2q and 2q + 1
        // of its 128-byte row, swizzled; lanes of tokens past M load nothing
        // and feed zeros (their MMA columns are never written)
        uint32_t xoff[MT][2];
#pragma unroll
        for (int t = 0; t < MT; ++t) {
            const uint32_t m = static_cast<uint32_t>(min(g + 8 * t, M - 1));
            xoff[t][0] = m * 128u + (((2u * q) ^ (m & 7u)) << 4);
            xoff[t][1] = m * 128u + (((2u * q + 1u) ^ (m & 7u)) << 4);
        }
        // this lane's code bytes in a stage's box: in MMA tile h of the warp,
        // rows frag_row(g) and frag_row(g) + 8 (a row past N is decoded from
        // zero-filled codes and its sums dropped); the 8 bytes of block b sit
        // in 16-byte chunk 2b + q/2 of the row's 128, stored at chunk
        // (2b + q/2) ^ (row & 7)
        const int fr = frag_row(g);
        const int wrow = warp * 16 * kTilesW + fr;  // CTA row of tile 0's fragment row g; tile h adds 16 h
        const uint32_t crow_sw = static_cast<uint32_t>(fr & 7);
        const uint32_t coff = static_cast<uint32_t>(wrow) * 128u + 8u * (q & 1);
        auto flush = [&](int seg) {
            // segment done: its partial sums, acc[h][t][0..1] = (row wrow +
            // 16 h, tokens 8t + 2q, +1) and acc[h][t][2..3] = (that row + 8,
            // the same tokens)
            const int tile = t0 + seg;
            const int sl = sc.slot(tile, c);
#pragma unroll
            for (int h = 0; h < kTilesW; ++h) {
                const int rowA = tile * kRowsCta + wrow + 16 * h, rowB = rowA + 8;
#pragma unroll
                for (int t = 0; t < MT; ++t) {
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int tok = 8 * t + 2 * q + e;
                        if (tok < M) {
                            float* pt = a.part + (static_cast<int64_t>(sl) * M + tok) * N;
                            if (rowA < N) pt[rowA] = acc[h][t][e];
                            if (rowB < N) pt[rowB] = acc[h][t][2 + e];
                        }
                    }
                    acc[h][t][0] = acc[h][t][1] = acc[h][t][2] = acc[h][t][3] = 0.0f;
                }
            }
        };

        // the rank-r term of the warp's rows, added by the CTA whose segment
        // ends at the tile's last block column (exactly one per tile); each
        // MMA tile's two 8-row halves lie inside one projection of a group
        auto add_rank = [&](int seg) {
            griddep_wait();  // sT from the preceding launch
#pragma unroll
            for (int h = 0; h < kTilesW; ++h) {
                const int64_t ra = static_cast<int64_t>(t0 + seg) * kRowsCta + wrow + 16 * h;
                const int64_t rA = ra < N ? ra : N - 1, rB = ra + 8 < N ? ra + 8 : N - 1;
                const int cA = rank_col(a, rA), cB = rank_col(a, rB);  // uniform over the warp
                if (cA == cB) {
                    rank_mma<MT>(a, acc[h], rA, rB, cA, true, true, g, q);
                } else {
                    rank_mma<MT>(a, acc[h], rA, rB, cA, true, false, g, q);
                    rank_mma<MT>(a, acc[h], rA, rB, cB, false, true, g, q);
                }
            }
        };

        bool ok = true;
        for (int k = 0; k < nst && ok; ++k) {
            const int s = k % S;
            const uint32_t u = static_cast<uint32_t>(k / S);
            const Step sp = step_of(k, nst0, blo0, len0, len1);
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(full + s, u & 1u, tmo, a.status));
            if (!ok) break;
            const uint32_t stc = st_base + static_cast<uint32_t>(s) * stage;
            // the step's block constants of each tile's rows fr and fr + 8
            float cA[kTilesW][kStep], cB[kTilesW][kStep];
#pragma unroll
            for (int h = 0; h < kTilesW; ++h) {
                const uint4 ca4 = lds128(const_addr(lut_base, s, wrow + 16 * h));
                const uint4 cb4 = lds128(const_addr(lut_base, s, wrow + 16 * h + 8));
                cA[h][0] = __uint_as_float(ca4.x);
                cA[h][1] = __uint_as_float(ca4.y);
                cA[h][2] = __uint_as_float(ca4.z);
                cA[h][3] = __uint_as_float(ca4.w);
                cB[h][0] = __uint_as_float(cb4.x);
                cB[h][1] = __uint_as_float(cb4.y);
                cB[h][2] = __uint_as_float(cb4.z);
                cB[h][3] = __uint_as_float(cb4.w);
            }
#pragma unroll
            for (int b = 0; b < kStep; ++b) {
                if (b < sp.b0 || b >= sp.b1) continue;
                const uint32_t ch = ((2u * b + (q >> 1)) ^ crow_sw) << 4;
                // A fragments of the block's four MMA steps of each tile
                // (unscaled levels)
                uint32_t af[kTilesW][4][4];
#pragma unroll
                for (int h = 0; h < kTilesW; ++h) {
                    const uint32_t ca = stc + coff + static_cast<uint32_t>(h) * 2048u + ch;
                    const uint2 wa = lds64(ca), wb = lds64(ca + 1024u);
#pragma unroll
                    for (int st4 = 0; st4 < 4; ++st4) {
                        const uint32_t xa = st4 < 2 ? wa.x : wa.y, xb = st4 < 2 ? wb.x : wb.y;
                        const uint32_t kk = (st4 & 1) * 2;
                        af[h][st4][0] = lut(lut_base, lane4, xa, kk);
                        af[h][st4][1] = lut(lut_base, lane4, xb, kk);
                        af[h][st4][2] = lut(lut_base, lane4, xa, kk + 1);
                        af[h][st4][3] = lut(lut_base, lane4, xb, kk + 1);
                    }
                }
                const uint32_t xb0 = stc + kCodeStage + b * xbox;
#pragma unroll
                for (int t = 0; t < MT; ++t) {
                    uint4 x0 = make_uint4(0u, 0u, 0u, 0u), x1 = x0;
                    if (t < MT / 2 || g + 8 * t < M) {  // tiles below MT / 2 are full
                        x0 = lds128(xb0 + xoff[t][0]);
                        x1 = lds128(xb0 + xoff[t][1]);
                    }
                    const uint32_t xw[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                    // per tile, the block's four MMA steps in one chain, then
                    // one FMA per accumulator with the block constants
#pragma unroll
                    for (int h = 0; h < kTilesW; ++h) {
                        float tv[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                        mma_bf16(tv, af[h][0], xw[0], xw[1]);
                        mma_bf16(tv, af[h][1], xw[2], xw[3]);
                        mma_bf16(tv, af[h][2], xw[4], xw[5]);
                        mma_bf16(tv, af[h][3], xw[6], xw[7]);
                        acc[h][t][0] = __fmaf_rn(tv[0], cA[h][b], acc[h][t][0]);
                        acc[h][t][1] = __fmaf_rn(tv[1], cA[h][b], acc[h][t][1]);
                        acc[h][t][2] = __fmaf_rn(tv[2], cB[h][b], acc[h][t][2]);
                        acc[h][t][3] = __fmaf_rn(tv[3], cB[h][b], acc[h][t][3]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + s);
            if (k == nst0 - 1) {
                if (blo0 + len0 == KB) add_rank(0);
                flush(0);
            } else if (k == nst - 1) {
                if (len1 == KB) add_rank(1);
                flush(1);
            }
        }
        if (!ok) abort_flag = 1;
    }

    // ---- tickets: the last CTA to finish a row tile reduces it
    const int nseg = len1 > 0 ? 2 : 1;
    __threadfence();  // publish this CTA's partials before taking tickets
    __syncthreads();
    if (abort_flag) return;  // a wait ran out (status recorded): no tickets, no output
    if (threadIdx.x == 0) {
        for (int j = 0; j < nseg; ++j) {
            const int tile = t0 + j;
            last_of[j] = (atomicAdd(a.counter + tile, 1) == sc.parts(tile) - 1) ? 1 : 0;
        }
    }
    __syncthreads();
    for (int j = 0; j < nseg; ++j) {
        if (!last_of[j]) continue;
        __threadfence();  // see the other CTAs' partials
        const int tile = t0 + j;
        const int n0 = tile * kRowsCta;
        const int np = sc.parts(tile);
        // four consecutive rows of one token per item; every partial of an
        // item is loaded before the first add (N is a multiple of 8)
        for (int i = threadIdx.x; i < M * (kRowsCta / 4); i += kThreads) {
            const int m = i / (kRowsCta / 4), n = n0 + 4 * (i % (kRowsCta / 4));
            if (n >= N) continue;
            float4 s4 = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            for (int s0 = 0; s0 < np; s0 += 8) {
                float4 v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    v[u] = s0 + u < np
                               ? __ldcg(reinterpret_cast<const float4*>(a.part + (static_cast<int64_t>(s0 + u) * M + m) * N + n))
                               : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    s4.x += v[u].x;
                    s4.y += v[u].y;
                    s4.z += v[u].z;
                    s4.w += v[u].w;
                }
            }
            *reinterpret_cast<uint2*>(a.Y + static_cast<int64_t>(m) * N + n) =
                make_uint2(pack_bf16x2(s4.x, s4.y), pack_bf16x2(s4.z, s4.w));
        }
        if (threadIdx.x == 0) a.counter[tile] = 0;  // ready for the next call
    }
}

// dynamic shared memory of one CTA: the 227 KB per block less room for the
// kernel's static shared variables
constexpr size_t kSmemLimit = 226 * 1024;

size_t smem_bytes(int64_t M, int stages) { return kLutBytes + static_cast<size_t>(stages) * stage_bytes(M) + 1024; }
static_assert(kMaxStages <= 8, "block constants of at most 8 stages fit in the table's free halves");
static_assert(kRowsCta == 256, "the codes tensor map's box is 256 rows");

template <int MT, bool kNoDq>
cudaError_t launch_mt(const CUtensorMap& codes, const CUtensorMap& x, const GemvMmaArgs& a, const Nf4Tables& tab,
                      bool pdl, cudaStream_t st) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(a.ctas));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem_bytes(a.M, a.stages);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, gemv_mma_kernel<MT, kNoDq>, codes, x, a, tab);
}

// n8 token tiles of the instantiation that serves M tokens
int token_tiles(int64_t M) { return M <= 8 ? 1 : (M <= 16 ? 2 : (M <= 32 ? 4 : 8)); }

}  // namespace

GemvMmaPlan gemv_mma_plan(int64_t M, int64_t N, int64_t K, int num_sms) {
    const int64_t KB = K / kBlock, tiles = (N + kRowsCta - 1) / kRowsCta, U = tiles * KB;
    const int64_t slots = std::max(num_sms, 1);  // one CTA per SM
    // whole waves, at least one CTA per row tile (so a range touches at most
    // two tiles), at most one CTA per unit
    const int64_t P = std::min(U, (tiles + slots - 1) / slots * slots);
    GemvMmaPlan plan;
    plan.ctas = static_cast<int>(P);
    plan.units = U;
    plan.stages = static_cast<int>(std::min<size_t>(kMaxStages, (kSmemLimit - kLutBytes - 1024) / stage_bytes(M)));
    plan.max_parts = static_cast<int>((KB + U / P - 1) / (U / P) + 1);
    return plan;
}

namespace {
template <int MT>
cudaError_t opt_in(int smax) {
    cudaError_t e = cudaFuncSetAttribute(gemv_mma_kernel<MT, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         smax);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(gemv_mma_kernel<MT, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smax);
}
}  // namespace

cudaError_t gemv_mma_init_device() {
    const int smax = static_cast<int>(kSmemLimit);
    cudaError_t e;
    if ((e = opt_in<1>(smax)) != cudaSuccess || (e = opt_in<2>(smax)) != cudaSuccess ||
        (e = opt_in<4>(smax)) != cudaSuccess)
        return e;
    return opt_in<8>(smax);
}

cudaError_t launch_gemv_mma(const CUtensorMap& codes, const CUtensorMap& x, const GemvMmaArgs& a,
                            const Nf4Tables& tab, bool pdl, cudaStream_t st) {
    if (a.M < 1 || a.M > kGemvMmaMaxM || a.ctas < 1 || a.stages < 2 || a.stages > kMaxStages)
        return cudaErrorInvalidValue;
    if (smem_bytes(a.M, a.stages) > kSmemLimit) return cudaErrorInvalidValue;
    const int mt = token_tiles(a.M);
    static_assert(8 * 8 == kGemvMmaMaxM, "token tiles");
    if (a.absmax) {
        if (mt == 1) return launch_mt<1, true>(codes, x, a, tab, pdl, st);
        if (mt == 2) return launch_mt<2, true>(codes, x, a, tab, pdl, st);
        if (mt == 4) return launch_mt<4, true>(codes, x, a, tab, pdl, st);
        return launch_mt<8, true>(codes, x, a, tab, pdl, st);
    }
    if (mt == 1) return launch_mt<1, false>(codes, x, a, tab, pdl, st);
    if (mt == 2) return launch_mt<2, false>(codes, x, a, tab, pdl, st);
    if (mt == 4) return launch_mt<4, false>(codes, x, a, tab, pdl, st);
    return launch_mt<8, false>(codes, x, a, tab, pdl, st);
}

}  // namespace qlora
