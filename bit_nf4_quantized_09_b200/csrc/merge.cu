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
// (eight n8 MMA tiles, tile t covering columns 8t .. 8t + 7), r/16 MMA steps
// over the rank (r = 8 pads the upper half of its one step with zeros). The
// A operand is B's rows (row-major, rank pairs contiguous); the B operand is
// columns of A, gathered with 16-bit loads once per block column and kept in
// registers while the warp walks down the rows (units are ordered block
// column first, row group second, and each warp takes one contiguous range).
// Lane (g, q) holds the sums of rows g and g + 8 at columns 8t + 2q, 8t + 2q
// + 1, whose codes are byte q of each 32-bit word of the block's 32 packed
// bytes: two byte permutes per pair of words gather them, and the per-block
// lookup table turns them into the bf16 pairs of w_hat. The bf16 results go
// straight to global memory, 4 bytes per lane and tile; a warp's stores
// cover 128 contiguous bytes of each of its 16 rows.
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

// A[j, kk] | A[j + 1, kk] << 16: a bf16 pair of consecutive rank rows
__device__ __forceinline__ uint32_t rank_pair(const uint16_t* A, int j, int64_t kk, int64_t K) {
    return static_cast<uint32_t>(__ldg(A + j * K + kk)) | (static_cast<uint32_t>(__ldg(A + (j + 1) * K + kk)) << 16);
}

template <bool kNoDq>
__device__ __forceinline__ float block_constant(const BlockConstants& c, int64_t b, float mu) {
    if (kNoDq) return __ldg(c.absmax + b);
    return __fmaf_rn(e4m3_to_f32(__ldg(c.qabsmax + b)), __ldg(c.s2 + (b >> 8)), mu);
}

template <int R, bool kNoDq>
__global__ void __launch_bounds__(kMergeThreads) merge_lora_kernel(const MergeArgs a, const Nf4Tables tab) {
    constexpr int S = R >= 16 ? R / 16 : 1;  // k16 MMA steps over the rank
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int64_t N = a.N, K = a.K, KB = K / kBlock, RG = (N + 15) / 16, U = RG * KB;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * kMergeWarps;
    const int64_t w = static_cast<int64_t>(blockIdx.x) * kMergeWarps + (threadIdx.x >> 5);
    const int64_t u_end = U * (w + 1) / warps;
    const float mu = kNoDq ? 0.0f : __ldg(a.c.mean);
    const uint32_t sel = static_cast<uint32_t>(q) | (static_cast<uint32_t>(q + 4) << 4);  // byte q of two words

    uint32_t bf[8][S][2];  // B operand of tile t, step s (columns of A)
    int64_t kb_loaded = -1;
#pragma unroll 1
    for (int64_t u = U * w / warps; u < u_end; ++u) {
        const int64_t kb = u / RG, rg = u - kb * RG, k0 = kb * kBlock;
        if (kb != kb_loaded) {
            kb_loaded = kb;
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                const int64_t kk = k0 + 8 * t + g;
#pragma unroll
                for (int s = 0; s < S; ++s) {
                    bf[t][s][0] = rank_pair(a.A, 16 * s + 2 * q, kk, K);
                    bf[t][s][1] = R >= 16 ? rank_pair(a.A, 16 * s + 2 * q + 8, kk, K) : 0u;
                }
            }
        }
        // rows g and g + 8 of the group; loads of rows past N read row N - 1
        // and their results are not stored
        const int64_t nA = rg * 16 + g, nB = nA + 8;
        const int64_t rA = nA < N ? nA : N - 1, rB = nB < N ? nB : N - 1;
        uint32_t af[S][4];
#pragma unroll
        for (int s = 0; s < S; ++s) {
            const uint16_t* pa = a.B + rA * R + 16 * s + 2 * q;
            const uint16_t* pb = a.B + rB * R + 16 * s + 2 * q;
            af[s][0] = __ldg(reinterpret_cast<const uint32_t*>(pa));
            af[s][1] = __ldg(reinterpret_cast<const uint32_t*>(pb));
            af[s][2] = R >= 16 ? __ldg(reinterpret_cast<const uint32_t*>(pa + 8)) : 0u;
            af[s][3] = R >= 16 ? __ldg(reinterpret_cast<const uint32_t*>(pb + 8)) : 0u;
        }
        const uint4* pcA = reinterpret_cast<const uint4*>(a.codes + rA * (K / 2) + kb * 32);
        const uint4* pcB = reinterpret_cast<const uint4*>(a.codes + rB * (K / 2) + kb * 32);
        const uint4 cA0 = __ldg(pcA), cA1 = __ldg(pcA + 1), cB0 = __ldg(pcB), cB1 = __ldg(pcB + 1);
        const float cvA = block_constant<kNoDq>(a.c, rA * KB + kb, mu);
        const float cvB = block_constant<kNoDq>(a.c, rB * KB + kb, mu);

        float acc[8][4];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.0f;
#pragma unroll
            for (int s = 0; s < S; ++s) mma_bf16(acc[t], af[s], bf[t][s][0], bf[t][s][1]);
        }

        // byte q of words 0..3 and 4..7: the codes of columns 8t + 2q (high
        // nibble) and 8t + 2q + 1 (low nibble) for t = 0..3 and 4..7
        auto gather = [sel](uint32_t x, uint32_t y, uint32_t z, uint32_t v) {
            return __byte_perm(__byte_perm(x, y, sel), __byte_perm(z, v, sel), 0x5410);
        };
        uint32_t hA[8], hB[8];  // w_hat pairs of tile t (column 8t + 2q in the low half)
        {
            const Nf4BlockLut lA = make_block_lut(tab.level, cvA);
            uint32_t o0[4], o1[4];
            lut_decode8(lA, gather(cA0.x, cA0.y, cA0.z, cA0.w), o0);
            lut_decode8(lA, gather(cA1.x, cA1.y, cA1.z, cA1.w), o1);
#pragma unroll
            for (int i = 0; i < 4; ++i) hA[i] = o0[i], hA[i + 4] = o1[i];
        }
        {
            const Nf4BlockLut lB = make_block_lut(tab.level, cvB);
            uint32_t o0[4], o1[4];
            lut_decode8(lB, gather(cB0.x, cB0.y, cB0.z, cB0.w), o0);
            lut_decode8(lB, gather(cB1.x, cB1.y, cB1.z, cB1.w), o1);
#pragma unroll
            for (int i = 0; i < 4; ++i) hB[i] = o0[i], hB[i + 4] = o1[i];
        }

        const float sc = a.scale;
        uint16_t* outA = a.W_out + nA * K + k0 + 2 * q;
        uint16_t* outB = a.W_out + nB * K + k0 + 2 * q;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const uint32_t vA = pack_bf16x2(__fmaf_rn(sc, acc[t][0], __uint_as_float(hA[t] << 16)),
                                            __fmaf_rn(sc, acc[t][1], __uint_as_float(hA[t] & 0xFFFF0000u)));
            const uint32_t vB = pack_bf16x2(__fmaf_rn(sc, acc[t][2], __uint_as_float(hB[t] << 16)),
                                            __fmaf_rn(sc, acc[t][3], __uint_as_float(hB[t] & 0xFFFF0000u)));
            if (nA < N) *reinterpret_cast<uint32_t*>(outA + 8 * t) = vA;
            if (nB < N) *reinterpret_cast<uint32_t*>(outB + 8 * t) = vB;
        }
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
