// Host-side launchers of the library's kernels (internal to libqlora_nf4.so).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace qlora {

// The first-level block constants of a quantised weight: with double
// quantisation c'_b = fmaf(E4M3(qabsmax[b]), s2[b / 256], *mean); without
// (absmax != nullptr) c_b = absmax[b] and the other three are not read.
struct BlockConstants {
    const uint8_t* qabsmax;
    const float* s2;
    const float* mean;
    const float* absmax;
};

// ----------------------------------------------------------- quantisation --
// W: fp32 [N, K], or bf16 [N, K] when bf16 is true. zero_word: a word the
// encoder sets to zero (the mean kernel's ticket), or nullptr.
cudaError_t launch_nf4_encode(const void* W, bool bf16, int64_t N, int64_t K, uint8_t* codes, float* absmax,
                              int* zero_word, const Nf4Tables& tab, int num_sms, cudaStream_t st);
// The double quantisation's mean: the fp64 pairwise tree over the nb
// constants (zero-padded to a power of two), built from aligned runs of
// kMeanRun by one launch. Scratch (16-byte aligned): the runs' fp64 sums, then
// the launch's ticket (dq_mean_ticket), which must be zero before it.
constexpr int kMeanPerThread = 16;
constexpr int64_t kMeanRun = 1024 * kMeanPerThread;  // 16384 constants per CTA
constexpr size_t dq_mean_scratch_bytes(int64_t nb) {
    return ((nb + kMeanRun - 1) / kMeanRun * 8 + 255) / 256 * 256 + 256;
}
int* dq_mean_ticket(void* scratch, int64_t nb);
cudaError_t launch_dq_mean(const float* absmax, int64_t nb, void* scratch, float* mean, cudaStream_t st);
// The E4M3 codes and second-level scales of the centred constants (after the
// encoder has written absmax and the mean).
cudaError_t launch_dq_groups(const float* absmax, int64_t nb, const float* mean, uint8_t* q, float* s2,
                             cudaStream_t st);
// out_map: the bf16 output viewed as [N*K/64 rows, 64], box {64, 128}, SW128.
constexpr size_t kDequantSmem = 2 * 128 * 128 + 1024;
cudaError_t launch_nf4_dequant(const CUtensorMap& out_map, const uint8_t* codes, const BlockConstants& c, int64_t N,
                               int64_t K, const Nf4Tables& tab, int num_sms, cudaStream_t st);
// c'ᵀ: cT[kb * ldc + n] = c'(row n, block kb) for n < N, 0 for N <= n < cols
// (columns from cols on are left alone: a group writes each projection's
// constants at its own column offset).
cudaError_t launch_decode_constants_t(const BlockConstants& c, int64_t N, int64_t K, int64_t ldc, int64_t cols,
                                      float* cT, cudaStream_t st);
// c'_b of the nb blocks in block order, fp32.
cudaError_t launch_decode_constants(const BlockConstants& c, int64_t nb, float* out, int num_sms, cudaStream_t st);
cudaError_t launch_e4m3_encode(const float* x, uint8_t* q, int64_t n, cudaStream_t st);

// ------------------------------------------------------ fused NF4 GEMMs --
// Tile of the fused kernels: 256 output rows (two M=128 MMAs) x 256 columns,
// 64-deep reduction steps, 3 pipeline stages.
constexpr int kFusedBM = 256;
constexpr int kFusedBN = 256;
constexpr int kFusedBK = 64;
constexpr int kFusedStages = 3;
constexpr int kFusedThreads = 320;  // 8 dequant/epilogue warps, 1 TMA warp, 1 MMA warp
size_t fused_smem_bytes();
cudaError_t fused_init_device();  // opt in to the large shared-memory carve-out

constexpr int kMaxGroups = 4;  // projections sharing one input in one fused launch

struct FusedArgs {
    int64_t M;          // tokens
    int64_t out_cols;   // N (forward) or K (dX): the output row pitch
    int64_t red;        // reduction length: K (forward) or N (dX)
    int rank_cols;      // columns of the low-rank term (UMMA K of the rank steps; 0 = none)
    int rank_steps;     // 64-column rank steps a tile's owner runs after its reduction steps
    // Output column groups (forward of projections that share one input):
    // group g owns out columns [group_end[g-1], group_end[g]) and its tiles
    // never straddle two groups; its rank step reads the act-side rank input
    // from column group_rank_x[g]. A single weight is one group.
    int ngroups;
    int64_t group_end[kMaxGroups];
    int group_rank_x[kMaxGroups];
    int ctas;           // CTAs (ranges of (tile, step) units): fused_ctas(); pair launches: 2 * pairs
    // Tiles of this launch: ids [tile_first, tile_first + tiles) (tiles = 0:
    // all of them). With pair_order, id 2p + h is row tile 2 (p % pairs_m) + h
    // of column tile p / pairs_m (pairs_m = ceil(row tiles / 2)), the order the
    // CTA-pair launch takes them in, so a stream-K launch can finish the tiles
    // a shorter pair launch left; otherwise id t is row tile t / tiles_n of
    // column tile t % tiles_n.
    int64_t tile_first;
    int64_t tiles;
    int pair_order;
    uint16_t* out;      // bf16 [M, out_cols]
    float* part;        // fp32 [fused_partial_ctas()][256][256] partial tiles of contributing CTAs
    int* flags;         // [fused_partial_ctas()] partial-ready flags, zero before the launch
    int* status;        // device status word
    uint64_t timeout_ns;
    int stall_producer; // test hook: load nothing
};

// Output tiles along the columns: 256-column tiles per group.
inline int64_t fused_tiles_n(const FusedArgs& a) {
    int64_t t = 0, start = 0;
    for (int g = 0; g < a.ngroups; ++g) {
        t += (a.group_end[g] - start + kFusedBN - 1) / kFusedBN;
        start = a.group_end[g];
    }
    return t;
}

// CTAs of a fused launch. With at least as many output tiles as SMs
// (max_ctas), one CTA per tile: no tile is split. With fewer, one CTA per SM
// (at most one per reduction step) and the tiles' steps dealt out in equal
// ranges, so every SM works; split tiles then go through fp32 partials.
inline int64_t fused_tiles(int64_t M, int64_t tiles_n) { return ((M + kFusedBM - 1) / kFusedBM) * tiles_n; }
inline int fused_ctas(int64_t M, int64_t tiles_n, int64_t red, int max_ctas) {
    const int64_t tiles = fused_tiles(M, tiles_n);
    if (tiles >= max_ctas) return static_cast<int>(tiles);
    const int64_t units = tiles * ((red + kFusedBK - 1) / kFusedBK);
    return static_cast<int>(units < max_ctas ? units : max_ctas);
}
// CTAs that may write a partial tile (0 when no tile is split).
inline int fused_partial_ctas(int64_t M, int64_t tiles_n, int64_t red, int max_ctas) {
    return fused_tiles(M, tiles_n) >= max_ctas ? 0 : fused_ctas(M, tiles_n, red, max_ctas);
}
// CTAs of a stream-K launch over `tiles` tiles (split when fewer than max_ctas).
inline int fused_ctas_for(int64_t tiles, int64_t red, int max_ctas) {
    if (tiles >= max_ctas) return static_cast<int>(tiles);
    const int64_t units = tiles * ((red + kFusedBK - 1) / kFusedBK);
    return static_cast<int>(units < max_ctas ? units : max_ctas);
}

// Forward: out = A_op . deq(W)^T + lora_a . lora_b^T, A_op = X [M, K].
// Maps: act {K, M} box {64, 256} SW128; codes {K/2, N} box {32, 256} SW32;
// cT {ldc, K/64} box {256, 1}; lora_act = sT {R, M} box {64, 256} SW128;
// lora_w = B {R', N} box {64, 256} SW128 (rank step c of a tile in group g
// reads lora_act at column group_rank_x[g] + 64c and lora_w at column 64c).
// pdl: launch as the programmatic dependent of the previous launch on st (the
// rank-r input, its output, is waited for only before the rank-r step).
cudaError_t launch_fused_fwd(const CUtensorMap& act, const CUtensorMap& codes, const CUtensorMap& cT,
                             const CUtensorMap& lora_act, const CUtensorMap& lora_w, const FusedArgs& a,
                             const Nf4Tables& tab, bool pdl, cudaStream_t st);
// dX: out = dY . deq(W) + sU . A.
// Maps: act = dY {N, M} box {64, 256} SW128; codes {K/2, N} box {128, 64} SW128;
// cT {ldc, K/64} box {64, 4}; lora_act = sU {R, M} box {64, 256} SW128;
// lora_w = A {K, R} box {64, 64} SW128 (four boxes per step; rank step c
// reads rows 64c.. of A and columns 64c.. of sU).
cudaError_t launch_fused_dx(const CUtensorMap& act, const CUtensorMap& codes, const CUtensorMap& cT,
                            const CUtensorMap& lora_act, const CUtensorMap& lora_w, const FusedArgs& a,
                            const Nf4Tables& tab, bool pdl, cudaStream_t st);

// CTA-pair forms of the two launches (whole tiles, clusters of two CTAs along
// M that share each dequantised weight tile; each CTA decodes its half). The
// grid is a.ctas: 2 per pair, pairs 0 .. a.ctas / 2 - 1 of the pair order
// (at most ceil(row tiles / 2) * column tiles).
// Maps as above except: forward codes box {32, 128}, cT box {128, 1}; dX
// codes box {64, 64} SW64, cT box {64, 2}.
cudaError_t launch_fused_pair_fwd(const CUtensorMap& act, const CUtensorMap& codes_half, const CUtensorMap& cT_half,
                                  const CUtensorMap& lora_act, const CUtensorMap& lora_w, const FusedArgs& a,
                                  const Nf4Tables& tab, bool pdl, cudaStream_t st);
cudaError_t launch_fused_pair_dx(const CUtensorMap& act, const CUtensorMap& codes_half, const CUtensorMap& cT_half,
                                 const CUtensorMap& lora_act, const CUtensorMap& lora_w, const FusedArgs& a,
                                 const Nf4Tables& tab, bool pdl, cudaStream_t st);

// ------------------------------------- small-batch register-fed MMA GEMV --
constexpr int kGemvMmaMaxM = 64;  // tokens: up to eight n8 MMA tiles

struct GemvMmaArgs {
    const uint8_t* qabsmax;  // E4M3 [N*K/64]
    const float* s2;         // [groups]
    const float* mean;       // [1]
    const float* absmax;     // fp32 [N*K/64] when stored without double quantisation (then the three above are unused)
    int64_t M, N, K;
    int rank_cols;           // columns of the rank-r dot of one output (a multiple of 8)
    int sT_ld, B_ld;         // row pitches of sT and B
    // Output row groups (projections sharing one input): output row n in
    // group g (group_end[g-1] <= n < group_end[g]) takes its rank-r input
    // from column group_rank_x[g] of sT. A single weight is one group.
    int ngroups;
    int64_t group_end[kMaxGroups];
    int group_rank_x[kMaxGroups];
    int ctas;                // grid size (from the plan)
    int64_t units;           // (row tiles) * (K/64 block columns)
    int stages;              // shared-memory pipeline stages (from the plan)
    int const_vec;           // K/64 % 4 == 0 and the constants aligned (qabsmax 4 B, absmax 16 B): one vector load per row and step
    float* part;             // fp32 [max_parts][M][N] partial sums
    int* counter;            // [row tiles] tickets, zero before the launch; left zero
    const uint16_t* sT;      // bf16 [M, sT_ld], read only in the epilogue
    const uint16_t* B;       // bf16 [N, B_ld]
    uint16_t* Y;             // bf16 [M, N]
    int* status;             // device status word
    uint64_t timeout_ns;
};

struct GemvMmaPlan {
    int ctas;
    int64_t units;
    int stages;
    int max_parts;  // partial-sum slots per row tile
};

GemvMmaPlan gemv_mma_plan(int64_t M, int64_t N, int64_t K, int num_sms);
cudaError_t gemv_mma_init_device();
// Maps: codes {K/2, N} box {128, 256} SW128; x = X {K, M} box {64, M} SW128. pdl: launch as the programmatic dependent of the previous launch on
// the stream (the kernel waits for it before reading sT).
cudaError_t launch_gemv_mma(const CUtensorMap& codes, const CUtensorMap& x, const GemvMmaArgs& a,
                            const Nf4Tables& tab, bool pdl, cudaStream_t st);

// ---------------------------------------------------------- skinny GEMMs --
// D[rows, NR] = sum over the reduction of A_op[rows, red] * B_op[NR, red]^T,
// split over the reduction (grid.y); the last CTA of each 128-row tile adds
// the fp32 partials in split order and writes the output. Up to
// kSkinnyMaxProblems independent problems share one launch (blockIdx.z): the
// 64-column chunks of a wider rank, or the gradients of several adapters.
constexpr int kSkinnyMaxStages = 8;  // stages x chunks: 24 KB each
constexpr int kSkinnyThreads = 192;  // TMA warp, MMA warp, 4 epilogue warps
size_t skinny_smem_bytes(int stages, int chunks);
cudaError_t skinny_init_device();

constexpr int kSkinnyOutBf16 = 0;           // out_bf16[row * out_ld + j] = bf16(scale * D)
constexpr int kSkinnyOutF32Transposed = 1;  // out_f32[j * out_ld + row] = D
constexpr int kSkinnyOutF32 = 2;            // out_f32[row * out_ld + j] = D
constexpr int kSkinnyMaxProblems = 8;

struct SkinnyProblem {
    int64_t rows;        // output rows (tiles of 128)
    int64_t red;         // reduction length (steps of 64)
    int a_mn_major;      // A_op rows-contiguous: two 64-wide TMA boxes per step
    int b_mn_major;      // B_op stored [red, NR] (box {NR, 64}, swizzle = NR*2 bytes)
    int mode;            // kSkinnyOut*
    int ncols;           // output columns (<= NR, even; a multiple of 4 for fp32)
    int64_t out_ld;      // output pitch in elements
    float scale;         // bf16 output scale
    uint16_t* out_bf16;
    float* out_f32;
    // bf16 output only: with row_ids set, output column j of row `row` is
    // kept iff row_ids[row] == (ids_col0 + j) / ids_r and written as zero
    // otherwise (the rank-r columns of the adapters a token does not use)
    const int* row_ids;
    int ids_col0;
    int ids_r;
};

struct SkinnyArgs {
    int NR;              // 16, 32 or 64: UMMA N of every problem
    int splits;          // reduction splits = cluster size along grid.y: 1, 2, 4 or 8
    int stages;          // pipeline stages; stages * chunks in 2 .. kSkinnyMaxStages
    int chunks;          // 64-deep reduction chunks per stage: 1, 2 or 4
    SkinnyProblem p[kSkinnyMaxProblems];
    int* status;
    uint64_t timeout_ns;
};

// The operand maps of each problem (A_op: K-major box {64, 128}, MN-major box
// {64, 64}, 128-byte swizzle; B_op: K-major box {64, NR}, 128-byte swizzle,
// MN-major box {NR, 64} with the NR*2-byte swizzle). A problem's row and
// column ranges are those of its maps: a map over a slice of a larger array
// (a base pointer inside it, the full row pitch) makes the slice's edge an
// out-of-bounds edge that TMA fills with zeros.
struct SkinnyMaps {
    CUtensorMap a[kSkinnyMaxProblems];
    CUtensorMap b[kSkinnyMaxProblems];
};

// pdl: launch as the programmatic dependent of the previous launch on st (it
// may start once every CTA of that launch has started; it completes after it).
cudaError_t launch_skinny(const SkinnyMaps& maps, const SkinnyArgs& args, int nproblems, cudaStream_t st,
                          bool pdl = false);

// ---------------------------------------------------------- adapter merge --
struct MergeArgs {
    const uint8_t* codes;  // packed NF4 [N, K/2]
    BlockConstants c;
    const uint16_t* A;     // bf16 [r, K]
    const uint16_t* B;     // bf16 [N, r]
    float scale;           // alpha / r
    int64_t N, K;
    uint16_t* W_out;       // bf16 [N, K]
    int* status;           // device status word (a bounded wait that ran out)
    uint64_t timeout_ns;
};

// W_out = bf16(deq(W) + scale . B . A); r in {8, 16, 32, 64}, on tcgen05.
// Maps: b_map = B [N, r] bf16 box {64, 128} SW128; a_map = A [r, K] bf16 box
// {64, 64} SW128; codes_map = codes [N, K/2] uint8 box {128, 128} SW128;
// out_map = W_out [N, K] bf16 box {64, 32} SW128.
cudaError_t launch_merge_tc(const CUtensorMap& b_map, const CUtensorMap& a_map, const CUtensorMap& codes_map,
                            const CUtensorMap& out_map, const MergeArgs& a, int r, const Nf4Tables& tab, int num_sms,
                            cudaStream_t st);
cudaError_t merge_tc_init_device();

}  // namespace qlora
