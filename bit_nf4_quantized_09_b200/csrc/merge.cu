// Adapter merge: W_out = bf16( deq(W) + (alpha/r) . B . A ).
//
// "waylandz LLM book ch.26", 26.2.2 (LoRAの学習設定, inference): the adapter
// is folded into the weight once, W_merged = W + (alpha/r) B A, and the
// merged weight is then used like the original one. "ta-paperlens QLoRA
// explainer", 落とし穴: a 4-bit base cannot absorb the small update (added
// to the NF4 weight and re-quantised, most of it is lost), so the merge goes
// to the 16-bit weight; re-quantising that is the caller's choice.
//
// Per element: w_hat = bf16(level[code] * c) exactly as the dequantiser
// computes it, then out = bf16_rn(fmaf(s, sum_j B[n, j] A[j, k], w_hat)) with
// the rank-r sum on the tensor cores (bf16 products, fp32 accumulation).
//
// The rank-r product is a dense contraction, so it runs on mma.m16n8k16: a
// warp unit is 16 weight rows (MMA rows) by one 64-column NF4 block column
// (eight n8 MMA tiles), r/16 MMA steps over the rank (r = 8 pads the upper
// half of its one step with zeros). The A operand is B's rows (row-major,
// rank pairs contiguous); the B operand is columns of A, gathered with 16-bit
// loads once per block column and kept in registers while the warp walks
// down the rows (units are ordered block column first, row group second, and
// each warp takes one contiguous range).
//
// The columns of the eight tiles are permuted so that lane (g, q), which
// holds the sums of rows g and g + 8 at MMA columns 2q and 2q + 1 of every
// tile, owns block columns 8q .. 8q + 7 (tiles 0-3) and 32 + 8q .. 39 + 8q
// (tiles 4-7): MMA column c of tile t is block column
//   8 (c / 2) + 32 (t / 4) + 2 (t % 4) + c % 2.
// So the lane's codes are two whole 32-bit words of the block's 32 packed
// bytes (words q and 4 + q), decoded by the per-block lookup table into the
// bf16 pairs of w_hat in tile order, and its results leave as two 16-byte
// stores per row: one warp store covers 64 contiguous bytes of each of 8
// rows (whole 32-byte sectors). The next unit's codes, constants and rank
// rows are loaded while the current one is computed.
//
// The kernel is bound by HBM: 0.5 B of codes, 1/64 B of constants and 2 B of
// output per weight; A and B are read from L2.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace qlora {

namespace {

constexpr int kMergeWarps = 8;
constexpr int kMergeThreads = kMergeWarps * 32;
// CTAs per SM the register budget is set for (the B-operand cache grows
// with r: 64 registers at r = 64)
template <int R>
constexpr int kMergeMinBlocks = R >= 64 ? 1 : 2;

// A[j, kk] | A[j + 1, kk] << 16: a bf16 pair of consecutive rank rows
__device__ __forceinline__ uint32_t rank_pair(const uint16_t* A, int j, int64_t kk, int64_t K) {
    return static_cast<uint32_t>(__ldg(A + j * K + kk)) | (static_cast<uint32_t>(__ldg(A + (j + 1) * K + kk)) << 16);
}

// Loads of one unit that do not depend on the block column's A fragments.
template <int S, bool kNoDq>
struct UnitLoads {
    uint32_t codes[2][2];  // rows g, g + 8: words q and 4 + q of the block
    uint32_t qa[2];        // E4M3 constants (or, kNoDq, fp32 constants as bits)
    float s2[2];
    uint32_t af[S][4];     // A operand: rows g, g + 8 of B, rank pairs 2q (+8)
};

template <int R, bool kNoDq>
__device__ __forceinline__ void load_unit(const MergeArgs& a, int64_t kb, int64_t rg, int g, int q,
                                          UnitLoads<(R >= 16 ? R / 16 : 1), kNoDq>& L) {
    constexpr int S = R >= 16 ? R / 16 : 1;
    const int64_t N = a.N, K = a.K, KB = K / kBlock;
    // rows past N read row N - 1; their results are not stored
    const int64_t rows[2] = {min(rg * 16 + g, N - 1), min(rg * 16 + g + 8, N - 1)};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t* cw = reinterpret_cast<const uint32_t*>(a.codes + rows[h] * (K / 2) + kb * 32);
        L.codes[h][0] = __ldg(cw + q);
        L.codes[h][1] = __ldg(cw + 4 + q);
        const int64_t b = rows[h] * KB + kb;
        if (kNoDq) {
            L.qa[h] = __float_as_uint(__ldg(a.c.absmax + b));
            L.s2[h] = 0.0f;
        } else {
            L.qa[h] = __ldg(a.c.qabsmax + b);
            L.s2[h] = __ldg(a.c.s2 + (b >> 8));
        }
#pragma unroll
        for (int s = 0; s < S; ++s) {
            const uint16_t* p = a.B + rows[h] * R + 16 * s + 2 * q;
            L.af[s][h] = __ldg(reinterpret_cast<const uint32_t*>(p));
            L.af[s][2 + h] = R >= 16 ? __ldg(reinterpret_cast<const uint32_t*>(p + 8)) : 0u;
        }
    }
}

template <int R, bool kNoDq>
__global__ void __launch_bounds__(kMergeThreads, kMergeMinBlocks<R>) merge_lora_kernel(const MergeArgs a, const Nf4Tables tab) {
    constexpr int S = R >= 16 ? R / 16 : 1;  // k16 MMA steps over the rank
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int64_t N = a.N, K = a.K, KB = K / kBlock, RG = (N + 15) / 16, U = RG * KB;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * kMergeWarps;
    const int64_t w = static_cast<int64_t>(blockIdx.x) * kMergeWarps + (threadIdx.x >> 5);
    const int64_t u_begin = U * w / warps, u_end = U * (w + 1) / warps;
    if (u_begin >= u_end) return;
    const float mu = kNoDq ? 0.0f : __ldg(a.c.mean);

    uint32_t bf[8][S][2];  // B operand of tile t, step s (columns of A)
    int64_t kb_loaded = -1;
    UnitLoads<S, kNoDq> cur;
    load_unit<R, kNoDq>(a, u_begin / RG, u_begin % RG, g, q, cur);
#pragma unroll 1
    for (int64_t u = u_begin; u < u_end; ++u) {
        const int64_t kb = u / RG, rg = u - kb * RG, k0 = kb * kBlock;
        // the next unit's loads (the last unit reloads itself)
        const int64_t un = u + 1 < u_end ? u + 1 : u;
        UnitLoads<S, kNoDq> nxt;
        load_unit<R, kNoDq>(a, un / RG, un % RG, g, q, nxt);
        if (kb != kb_loaded) {
            kb_loaded = kb;
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                const int64_t kk = k0 + 8 * (g >> 1) + 32 * (t >> 2) + 2 * (t & 3) + (g & 1);
#pragma unroll
                for (int s = 0; s < S; ++s) {
                    bf[t][s][0] = rank_pair(a.A, 16 * s + 2 * q, kk, K);
                    bf[t][s][1] = R >= 16 ? rank_pair(a.A, 16 * s + 2 * q + 8, kk, K) : 0u;
                }
            }
        }

        float acc[8][4];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.0f;
#pragma unroll
            for (int s = 0; s < S; ++s) mma_bf16(acc[t], cur.af[s], bf[t][s][0], bf[t][s][1]);
        }

        const float sc = a.scale;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t n = rg * 16 + g + 8 * h;
            const float c = kNoDq ? __uint_as_float(cur.qa[h]) : __fmaf_rn(e4m3_to_f32(cur.qa[h]), cur.s2[h], mu);
            const Nf4BlockLut lut = make_block_lut(tab.level, c);
            uint32_t wh[8];  // w_hat pairs of tile t: columns of MMA columns 2q, 2q + 1
            lut_decode8(lut, cur.codes[h][0], *reinterpret_cast<uint32_t(*)[4]>(wh));
            lut_decode8(lut, cur.codes[h][1], *reinterpret_cast<uint32_t(*)[4]>(wh + 4));
            uint32_t v[8];
#pragma unroll
            for (int t = 0; t < 8; ++t)
                v[t] = pack_bf16x2(__fmaf_rn(sc, acc[t][2 * h], __uint_as_float(wh[t] << 16)),
                                   __fmaf_rn(sc, acc[t][2 * h + 1], __uint_as_float(wh[t] & 0xFFFF0000u)));
            if (n < N) {
                uint4* o = reinterpret_cast<uint4*>(a.W_out + n * K + k0 + 8 * q);
                o[0] = make_uint4(v[0], v[1], v[2], v[3]);  // columns 8q .. 8q + 7
                o[4] = make_uint4(v[4], v[5], v[6], v[7]);  // columns 32 + 8q .. 39 + 8q
            }
        }
        cur = nxt;
    }
}

template <int R, bool kNoDq>
cudaError_t launch_r(const MergeArgs& a, const Nf4Tables& tab, int num_sms, cudaStream_t st) {
    int per_sm = 0;
    const cudaError_t e =
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, merge_lora_kernel<R, kNoDq>, kMergeThreads, 0);
    if (e != cudaSuccess) return e;
    const int64_t units = (a.N + 15) / 16 * (a.K / kBlock);
    const int64_t want = (units + kMergeWarps - 1) / kMergeWarps;
    const int64_t cap = static_cast<int64_t>(std::max(per_sm, 1)) * std::max(num_sms, 1);
    const int grid = static_cast<int>(std::max<int64_t>(1, std::min(want, cap)));
    merge_lora_kernel<R, kNoDq><<<grid, kMergeThreads, 0, st>>>(a, tab);
    return cudaGetLastError();
}

template <bool kNoDq>
cudaError_t launch_storage(const MergeArgs& a, int r, const Nf4Tables& tab, int num_sms, cudaStream_t st) {
    switch (r) {
        case 8: return launch_r<8, kNoDq>(a, tab, num_sms, st);
        case 16: return launch_r<16, kNoDq>(a, tab, num_sms, st);
        case 32: return launch_r<32, kNoDq>(a, tab, num_sms, st);
        case 64: return launch_r<64, kNoDq>(a, tab, num_sms, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_merge_lora(const MergeArgs& a, int r, const Nf4Tables& tab, int num_sms, cudaStream_t st) {
    if (a.N < 1 || a.K < kBlock || a.K % kBlock != 0) return cudaErrorInvalidValue;
    return a.c.absmax ? launch_storage<true>(a, r, tab, num_sms, st) : launch_storage<false>(a, r, tab, num_sms, st);
}

}  // namespace qlora
