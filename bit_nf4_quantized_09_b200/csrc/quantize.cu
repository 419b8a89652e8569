// NF4 quantiser (blockwise absmax + nearest-level codes + nibble packing),
// double quantisation of the absmax constants, and dequantisation.
//
// Sources: "ta-paperlens QLoRA explainer", sections 量子化を1段落で (c = max|x|
// over blocks of 64; store the index of the nearest level of x/c), NF4
// (16 normal-quantile levels, exact zero, ends +-1) and 二重量子化 (constants
// centred by their mean, 8-bit floats in groups of 256, one fp32 per group);
// "QLoRA" glossary (ultralytics), NF4 construction and nearest-level argmin.
#include <cuda_fp16.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace qlora {

// ---------------------------------------------------------------------------
// K1: absmax + encode + pack. Eight threads per 64-weight block, eight
// consecutive weights per thread (two 16-byte loads), four packed bytes out.
// The code of v = w / c is the number of decision thresholds strictly below
// v. It is read from a table over a uniform grid of 129 cells of width 1/64
// on [-1, 1]: cell j = RN(64 v + 64) covers [(j - 64.5)/64, (j - 63.5)/64],
// holds the number of thresholds below the cell and the one threshold inside
// it, if any (neighbouring thresholds are more than 1/64 apart), so the code
// is base_j + [v > t_j]. RN(64 v + 64) is the low bits of one fma with
// 1.5 * 2^23 + 64; at a cell edge either cell gives the same code. The table
// is replicated 16 times so that a half warp reads it without bank
// conflicts.
//
// v is the correctly rounded quotient, computed without a division per
// weight by Markstein's method (P. Markstein, IBM J. Res. Dev. 34(1), 1990;
// Muller et al., Handbook of Floating-Point Arithmetic, 2nd ed., sec. 4.9):
// with y = RN(1/c) and q0 = RN(w*y), the remainder w - c*q0 is exact in one
// fma and RN(q0 + (w - c*q0)*y) = RN(w/c). The theorem needs the quotient and
// the remainder to stay in the normal range; blocks with c < 2^-96 take the
// IEEE division instead (so no remainder of a value near a threshold can be
// subnormal), and values far below every threshold code to the zero level
// either way.
// The quotient's three roundings and the cell index's fma run on pairs of
// weights in the packed fp32x2 instructions of sm_100 (each half an IEEE
// fp32 operation with round-to-nearest, so every result is bit for bit the
// scalar one), halving their issue slots.
// Loads of the next block run ahead of the current block's arithmetic.
// ---------------------------------------------------------------------------
constexpr int kCells = 129;
constexpr int kCellCopies = 16;

// The code of q, given jbits = the bits of fma(q, 64, 1.5 * 2^23 + 64).
__device__ __forceinline__ uint32_t nf4_code_j(float q, uint32_t jbits, const float2* sLut, int copy) {
    const int j = static_cast<int>(jbits - 0x4B400000u);  // RN(64 q + 64), 0..128
    const float2 e = sLut[j * kCellCopies + copy];  // {threshold in the cell (2 if none), thresholds below}
    return static_cast<uint32_t>(__float_as_int(e.y)) + (q > e.x ? 1u : 0u);
}

__device__ __forceinline__ uint32_t nf4_code(float q, const float2* sLut, int copy) {
    return nf4_code_j(q, __float_as_uint(__fmaf_rn(q, 64.0f, 12582976.0f)), sLut, copy);
}

// Packed fp32 pairs: lo in bits 0..31, hi in bits 32..63.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// One thread's eight consecutive weights of a block, as loaded: two float4
// of fp32 input, or one uint4 of bf16 input (every bf16 value is an fp32
// value, so a bf16 weight codes exactly as its fp32 upcast).
template <bool kBf16>
struct Raw8 {
    float4 a, b;
};
template <>
struct Raw8<true> {
    uint4 a;
};

template <bool kBf16>
__device__ __forceinline__ Raw8<kBf16> load8(const void* W, int64_t blk, int sub) {
    Raw8<kBf16> r;
    if constexpr (kBf16) {
        r.a = __ldcs(reinterpret_cast<const uint4*>(W) + blk * 8 + sub);
    } else {
        r.a = __ldcs(reinterpret_cast<const float4*>(W) + blk * 16 + sub * 2);
        r.b = __ldcs(reinterpret_cast<const float4*>(W) + blk * 16 + sub * 2 + 1);
    }
    return r;
}

template <bool kBf16>
__device__ __forceinline__ void unpack8(const Raw8<kBf16>& r, float (&v)[8]) {
    if constexpr (kBf16) {
        const uint32_t w[4] = {r.a.x, r.a.y, r.a.z, r.a.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);  // element 2i in the low half
            v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    } else {
        v[0] = r.a.x, v[1] = r.a.y, v[2] = r.a.z, v[3] = r.a.w;
        v[4] = r.b.x, v[5] = r.b.y, v[6] = r.b.z, v[7] = r.b.w;
    }
}

template <bool kBf16>
__global__ void __launch_bounds__(256) nf4_encode_kernel(const void* __restrict__ W, int64_t nblocks,
                                                         uint32_t* __restrict__ codes, float* __restrict__ absmax,
                                                         Nf4Tables tab, int* __restrict__ zero_word) {
    asm volatile("griddepcontrol.launch_dependents;");  // the mean launch may be scheduled; it waits for this grid
    __shared__ float2 sLut[kCells * kCellCopies];
    if (zero_word && blockIdx.x == 0 && threadIdx.x == 0) *zero_word = 0;  // the mean kernel's ticket
    for (int j = threadIdx.x; j < kCells; j += blockDim.x) {
        const float lo = (static_cast<float>(j) - 64.5f) * 0.015625f, hi = lo + 0.015625f;  // exact
        int below = 0;
        float inside = 2.0f;
#pragma unroll
        for (int k = 0; k < 15; ++k) {
            below += tab.thresh[k] < lo ? 1 : 0;
            if (tab.thresh[k] >= lo && tab.thresh[k] < hi) inside = tab.thresh[k];
        }
        const float2 e = make_float2(inside, __int_as_float(below));
#pragma unroll
        for (int c = 0; c < kCellCopies; ++c) sLut[j * kCellCopies + c] = e;
    }
    __syncthreads();
    const int copy = threadIdx.x & (kCellCopies - 1);

    const int sub = threadIdx.x & 7;               // position inside the block
    const int lane_blk = (threadIdx.x & 31) >> 3;  // which of the warp's 4 blocks
    const int64_t stride = ((static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5) * 4;
    int64_t bw = ((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5) * 4;

    // warp-uniform loop: every lane takes part in the shuffles of every pass
    Raw8<kBf16> x{};
    if (bw + lane_blk < nblocks) x = load8<kBf16>(W, bw + lane_blk, sub);
    for (; bw < nblocks; bw += stride) {
        const int64_t b = bw + lane_blk;
        const bool valid = b < nblocks;
        const int64_t nb = b + stride;
        Raw8<kBf16> nx{};
        if (nb < nblocks) nx = load8<kBf16>(W, nb, sub);
        float v[8];
        unpack8<kBf16>(x, v);
        float c = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) c = fmaxf(c, fabsf(v[i]));
        c = fmaxf(c, __shfl_xor_sync(0xFFFFFFFFu, c, 1));
        c = fmaxf(c, __shfl_xor_sync(0xFFFFFFFFu, c, 2));
        c = fmaxf(c, __shfl_xor_sync(0xFFFFFFFFu, c, 4));
        uint32_t word = 0;
        if (c == 0.0f) {
            word = 0x77777777u;  // all-zero block: every element is the exact-zero level
        } else if (c >= 0x1p-96f) {
            const float y = __frcp_rn(c);
            const uint64_t y2 = f2_pack(y, y), nc2 = f2_pack(-c, -c);
            const uint64_t k64 = f2_pack(64.0f, 64.0f), kmagic = f2_pack(12582976.0f, 12582976.0f);
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                // weights i and i + 1: q = RN(v / c) and the cell fma, in pairs
                const uint64_t v2 = f2_pack(v[i], v[i + 1]);
                const uint64_t q0 = f2_mul(v2, y2);
                const uint64_t rem = f2_fma(nc2, q0, v2);
                const uint64_t q = f2_fma(rem, y2, q0);
                const uint64_t jb = f2_fma(q, k64, kmagic);
                float qa, qb, ja, jbf;
                f2_unpack(q, qa, qb);
                f2_unpack(jb, ja, jbf);
                const uint32_t ca = nf4_code_j(qa, __float_as_uint(ja), sLut, copy);
                const uint32_t cb = nf4_code_j(qb, __float_as_uint(jbf), sLut, copy);
                word |= ((ca << 4) | cb) << (4 * i);  // element i in the high nibble of byte i / 2
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                word |= nf4_code(__fdiv_rn(v[i], c), sLut, copy) << (8 * (i >> 1) + ((i & 1) ? 0 : 4));
        }
        // element 2j sits in the high nibble of byte j; bytes little-endian in the word
        if (valid) {
            __stcs(codes + b * 8 + sub, word);
            if (sub == 0) absmax[b] = c;
        }
        x = nx;
    }
}

// ---------------------------------------------------------------------------
// The fp64 pairwise tree over 1024 values, one per thread: lane l holds value
// l of its warp and `x += shfl_down(x, s)` for s = 1, 2, 4, 8, 16 leaves in
// lane 0 exactly the tree ((x0 + x1) + (x2 + x3)) + ...; the same step then
// runs over the 32 warp sums. The result is valid in thread 0.
// ---------------------------------------------------------------------------
__device__ __forceinline__ double tree_sum_1024(double x, double* warp_sums) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int s = 1; s < 32; s <<= 1) x += __shfl_down_sync(0xFFFFFFFFu, x, s);
    if (lane == 0) warp_sums[warp] = x;
    __syncthreads();
    double y = 0.0;
    if (warp == 0) {
        y = warp_sums[lane];
#pragma unroll
        for (int s = 1; s < 32; s <<= 1) y += __shfl_down_sync(0xFFFFFFFFu, y, s);
    }
    return y;  // valid in thread 0
}


// K2a: the mean's fp64 pairwise tree (over the nb constants, zero-padded to a
// power of two). Its subtrees over aligned runs nest: a CTA of 1024 threads
// sums one aligned run of 16384 constants, thread i its 16 consecutive ones in
// tree order (((c0 + c1) + (c2 + c3)) + ...), then the 1024 values by
// tree_sum_1024; the last CTA to finish (an atomic ticket that the encoder has
// set to zero) sums the run sums 1024 at a time, level by level, and writes
// mean = fp32(sum / nb).
__global__ void __launch_bounds__(1024) dq_mean_kernel(const float* __restrict__ absmax, int64_t nb,
                                                        double* __restrict__ run_sums, int* __restrict__ ticket,
                                                        float* __restrict__ mean) {
    __shared__ double ws[32];
    __shared__ int last;
    asm volatile("griddepcontrol.launch_dependents;");
    asm volatile("griddepcontrol.wait;" ::: "memory");  // absmax and the zeroed ticket of the encoder
    const int64_t b0 = (static_cast<int64_t>(blockIdx.x) * 1024 + threadIdx.x) * kMeanPerThread;
    double q[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int64_t bj = b0 + 4 * j;
        float4 f;
        if (bj + 3 < nb) {
            f = __ldcg(reinterpret_cast<const float4*>(absmax + bj));  // kept in L2 for the group pass
        } else {
            f.x = bj < nb ? absmax[bj] : 0.0f;
            f.y = bj + 1 < nb ? absmax[bj + 1] : 0.0f;
            f.z = bj + 2 < nb ? absmax[bj + 2] : 0.0f;
            f.w = 0.0f;  // bj + 3 >= nb
        }
        q[j] = (static_cast<double>(f.x) + static_cast<double>(f.y)) + (static_cast<double>(f.z) + static_cast<double>(f.w));
    }
    const double x = (q[0] + q[1]) + (q[2] + q[3]);  // the thread's 16 consecutive constants in tree order
    const double s = tree_sum_1024(x, ws);
    if (threadIdx.x == 0) {
        run_sums[blockIdx.x] = s;
        __threadfence();  // the run sum, before the ticket
        last = atomicAdd(ticket, 1) == static_cast<int>(gridDim.x) - 1;
    }
    __syncthreads();
    if (!last) return;
    __threadfence();  // every run sum, filed before its ticket
    double total = s;
    for (int64_t n = gridDim.x; n > 1; n = (n + 1023) / 1024) {
        // level: node c sums run_sums[1024 c .. 1024 c + 1023] into run_sums[c]
        for (int64_t c = 0; c * 1024 < n; ++c) {
            const int64_t i = c * 1024 + threadIdx.x;
            const double v = i < n ? __ldcg(run_sums + i) : 0.0;
            total = tree_sum_1024(v, ws);  // thread 0; ends its reads before the barrier below
            __syncthreads();
            if (threadIdx.x == 0) run_sums[c] = total;
            __syncthreads();
        }
        __threadfence_block();
    }
    if (threadIdx.x == 0) {
        *mean = __double2float_rn(__ddiv_rn(total, static_cast<double>(nb)));
        *ticket = 0;
    }
}

// ---------------------------------------------------------------------------
// K2b: one warp per group of 256 constants, eight per lane.
// d = c - mean, s2 = max|d| / 448, code = E4M3_rn_satfinite(d / s2).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) dq_groups_kernel(const float* __restrict__ c, int64_t nb,
                                                         const float* __restrict__ mean, uint8_t* __restrict__ q,
                                                         float* __restrict__ s2) {
    asm volatile("griddepcontrol.wait;" ::: "memory");  // the mean of the preceding launch
    const int lane = threadIdx.x & 31;
    const int64_t g = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t ng = (nb + kGroup - 1) / kGroup;
    if (g >= ng) return;
    const float mu = *mean;
    const int64_t b0 = g * kGroup + lane * 8;
    float d[8];
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t b = b0 + i;
        d[i] = (b < nb) ? __fsub_rn(c[b], mu) : 0.0f;
        m = fmaxf(m, fabsf(d[i]));
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, s));
    const float sg = __fdiv_rn(m, 448.0f);
    if (lane == 0) s2[g] = sg;
    uint8_t out[8];
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        uint32_t pair = 0;
        if (sg != 0.0f) pair = f32x2_to_e4m3x2(__fdiv_rn(d[i], sg), __fdiv_rn(d[i + 1], sg));
        out[i] = static_cast<uint8_t>(pair & 0xFFu);
        out[i + 1] = static_cast<uint8_t>((pair >> 8) & 0xFFu);
    }
    if (b0 + 8 <= nb) {
        uint2 w;
        w.x = out[0] | (out[1] << 8) | (out[2] << 16) | (static_cast<uint32_t>(out[3]) << 24);
        w.y = out[4] | (out[5] << 8) | (out[6] << 16) | (static_cast<uint32_t>(out[7]) << 24);
        *reinterpret_cast<uint2*>(q + b0) = w;
    } else {
        for (int i = 0; i < 8; ++i)
            if (b0 + i < nb) q[b0 + i] = out[i];
    }
}

// Decoded first-level constant of block b: c' = E4M3(q_b) * s2_g + mean, one
// fp32 rounding.
__device__ __forceinline__ float decode_constant(const uint8_t* q, const float* s2, float mu, int64_t b) {
    return __fmaf_rn(e4m3_to_f32(q[b]), s2[b / kGroup], mu);
}

// ---------------------------------------------------------------------------
// K3: standalone dequantisation to bf16. A CTA of 128 threads walks chunks of
// 128 consecutive 64-weight blocks, one block per thread. kNoDq: the weight
// keeps one fp32 absmax per block (no double quantisation) and q, s2, mean
// are not read. The next chunk's
// codes are loaded while the current one is decoded; the 16 KB of bf16 output
// go to a 128-byte-swizzled shared tile (conflict-free 16-byte stores) that a
// TMA tensor store writes to global memory as 128 rows of 128 bytes, with two
// tiles in flight.
// ---------------------------------------------------------------------------
constexpr int kDeqChunk = 128;

template <bool kNoDq>
__global__ void __launch_bounds__(kDeqChunk) nf4_dequant_kernel(const __grid_constant__ CUtensorMap tm_out,
                                                                 const uint4* __restrict__ codes,
                                                                 const uint8_t* __restrict__ q,
                                                                 const float* __restrict__ s2,
                                                                 const float* __restrict__ mean,
                                                                 const float* __restrict__ absmax, int64_t nblocks,
                                                                 Nf4Tables tab) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int t = threadIdx.x;
    const float mu = kNoDq ? 0.0f : *mean;
    const int64_t nchunks = (nblocks + kDeqChunk - 1) / kDeqChunk;

    // this thread's block of the first chunk: codes, then the 8-bit constant
    // and group scale (or, kNoDq, the fp32 constant in ps2)
    int64_t ch = blockIdx.x;
    uint4 p0 = make_uint4(0, 0, 0, 0), p1 = p0;
    uint32_t pq = 0;
    float ps2 = 0.0f;
    if (ch < nchunks && ch * kDeqChunk + t < nblocks) {
        const int64_t b = ch * kDeqChunk + t;
        p0 = __ldcs(codes + 2 * b);
        p1 = __ldcs(codes + 2 * b + 1);
        if (kNoDq) {
            ps2 = absmax[b];
        } else {
            pq = q[b];
            ps2 = s2[b / kGroup];
        }
    }
    for (int it = 0; ch < nchunks; ch += gridDim.x, ++it) {
        const int64_t b = ch * kDeqChunk + t;
        const int64_t nb = b + static_cast<int64_t>(gridDim.x) * kDeqChunk;
        // the next chunk's loads are in flight while this one is decoded
        uint4 n0 = make_uint4(0, 0, 0, 0), n1 = n0;
        uint32_t nq = 0;
        float ns2 = 0.0f;
        if (nb < nblocks) {
            n0 = __ldcs(codes + 2 * nb);
            n1 = __ldcs(codes + 2 * nb + 1);
            if (kNoDq) {
                ns2 = absmax[nb];
            } else {
                nq = q[nb];
                ns2 = s2[nb / kGroup];
            }
        }
        const float cprime = (b < nblocks) ? (kNoDq ? ps2 : __fmaf_rn(e4m3_to_f32(pq), ps2, mu)) : 0.0f;
        const Nf4BlockLut lut = make_block_lut(tab.level, cprime);

        uint8_t* tile = tiles + (it & 1) * (kDeqChunk * 128);
        if (t == 0) bulk_wait_read<1>();  // the store issued two chunks ago has left this tile
        __syncthreads();
        const uint32_t row = smem_u32(tile) + t * 128;
        const uint32_t words[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            uint32_t o[4];
            lut_decode8(lut, words[j], o);
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(row + ((j ^ (t & 7)) << 4)), "r"(o[0]),
                         "r"(o[1]), "r"(o[2]), "r"(o[3])
                         : "memory");
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (t == 0) {
            tma_store_2d(&tm_out, tile, 0, static_cast<int>(ch * kDeqChunk));
            bulk_commit();
        }
        p0 = n0;
        p1 = n1;
        pq = nq;
        ps2 = ns2;
    }
    if (t == 0) bulk_wait<0>();
}

// ---------------------------------------------------------------------------
// Decoded constants transposed for the matmul kernels: cT[kb * ldc + n] =
// c' of block (n, kb), so a run of consecutive output rows n for one k-block
// is contiguous (one TMA box). 32 x 32 tiles through shared memory. kNoDq:
// the constants are the weight's fp32 absmax values, transposed unchanged.
// ---------------------------------------------------------------------------
template <bool kNoDq>
__global__ void __launch_bounds__(256) decode_constants_t_kernel(const uint8_t* __restrict__ q,
                                                                  const float* __restrict__ s2,
                                                                  const float* __restrict__ mean,
                                                                  const float* __restrict__ absmax, int64_t N,
                                                                  int64_t KB, int64_t ldc, int64_t cols,
                                                                  float* __restrict__ cT) {
    // a CTA takes 64 rows n by 64 block columns kb; thread t decodes the 16
    // constants of row n0 + t / 4, block columns kb0 + 16 (t % 4) .. + 15
    // (one 16-byte load of E4M3 codes, or four of fp32 absmax, when the row's
    // constants are 16-aligned) into a padded shared tile, which leaves as
    // float4 stores of four consecutive n per block column
    __shared__ float tile[64][65];
    const float mu = kNoDq ? 0.0f : *mean;
    const int64_t n0 = static_cast<int64_t>(blockIdx.y) * 64, kb0 = static_cast<int64_t>(blockIdx.x) * 64;
    const int t = threadIdx.x, nl = t >> 2, k16 = (t & 3) * 16;
    const int64_t n = n0 + nl;
    float c[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) c[j] = 0.0f;
    if (n < N) {
        const int64_t base = n * KB + kb0 + k16;
        if ((KB & 15) == 0 && kb0 + k16 < KB) {
            // 16 whole constants, in one group of 256 (base is a multiple of 16)
            if (kNoDq) {
                const float4* src = reinterpret_cast<const float4*>(absmax + base);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 v = src[i];
                    c[4 * i] = v.x, c[4 * i + 1] = v.y, c[4 * i + 2] = v.z, c[4 * i + 3] = v.w;
                }
            } else {
                const uint4 w = *reinterpret_cast<const uint4*>(q + base);
                const float sg = s2[base / kGroup];
                const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    c[i] = __fmaf_rn(e4m3_to_f32(static_cast<uint8_t>(words[i >> 2] >> (8 * (i & 3)))), sg, mu);
            }
        } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int64_t kb = kb0 + k16 + j;
                if (kb < KB) c[j] = kNoDq ? absmax[n * KB + kb] : decode_constant(q, s2, mu, n * KB + kb);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) tile[k16 + j][nl] = c[j];
    __syncthreads();
    // cols is a multiple of 4, as are ldc and the rows' offset, so each
    // float4 lies inside the written range and is 16-byte aligned
    for (int i = t; i < 64 * 16; i += 256) {
        const int kl = i >> 4, n4 = (i & 15) * 4;
        const int64_t kb = kb0 + kl, nn = n0 + n4;
        if (kb < KB && nn < cols) {
            float4 v;
            v.x = nn < N ? tile[kl][n4] : 0.0f;
            v.y = nn + 1 < N ? tile[kl][n4 + 1] : 0.0f;
            v.z = nn + 2 < N ? tile[kl][n4 + 2] : 0.0f;
            v.w = nn + 3 < N ? tile[kl][n4 + 3] : 0.0f;
            *reinterpret_cast<float4*>(cT + kb * ldc + nn) = v;
        }
    }
}

// c'_b of every block, in block order (fp32 [nb]).
template <bool kNoDq>
__global__ void __launch_bounds__(256) decode_constants_kernel(const uint8_t* __restrict__ q,
                                                                const float* __restrict__ s2,
                                                                const float* __restrict__ mean,
                                                                const float* __restrict__ absmax, int64_t nb,
                                                                float* __restrict__ c) {
    const float mu = kNoDq ? 0.0f : *mean;
    for (int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b < nb;
         b += static_cast<int64_t>(gridDim.x) * blockDim.x)
        c[b] = kNoDq ? absmax[b] : decode_constant(q, s2, mu, b);
}

// Test hook: the double quantisation's E4M3 conversion on arbitrary floats.
__global__ void e4m3_encode_kernel(const float* __restrict__ x, uint8_t* __restrict__ q, int64_t n) {
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        q[i] = static_cast<uint8_t>(f32x2_to_e4m3x2(x[i], 0.0f) & 0xFFu);
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------

static int grid_for(int64_t work_items, int threads, int max_ctas) {
    int64_t g = (work_items + threads - 1) / threads;
    if (g > max_ctas) g = max_ctas;
    return static_cast<int>(g < 1 ? 1 : g);
}

cudaError_t launch_nf4_encode(const void* W, bool bf16, int64_t N, int64_t K, uint8_t* codes, float* absmax,
                              int* zero_word, const Nf4Tables& tab, int num_sms, cudaStream_t st) {
    const int64_t nb = N * K / kBlock;
    const int grid = grid_for(nb * 8, 256, num_sms * 8);
    if (bf16)
        nf4_encode_kernel<true><<<grid, 256, 0, st>>>(W, nb, reinterpret_cast<uint32_t*>(codes), absmax, tab,
                                                       zero_word);
    else
        nf4_encode_kernel<false><<<grid, 256, 0, st>>>(W, nb, reinterpret_cast<uint32_t*>(codes), absmax, tab,
                                                        zero_word);
    return cudaGetLastError();
}

int* dq_mean_ticket(void* scratch, int64_t nb) {
    return reinterpret_cast<int*>(static_cast<uint8_t*>(scratch) + dq_mean_scratch_bytes(nb) - 256);
}

// programmatic dependent launches: each waits (griddepcontrol.wait) for its
// predecessor before it reads, so only the launch latency overlaps
static cudaLaunchConfig_t pdl_config(unsigned grid, unsigned block, cudaStream_t st, cudaLaunchAttribute* attr) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.stream = st;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

cudaError_t launch_dq_mean(const float* absmax, int64_t nb, void* scratch, float* mean, cudaStream_t st) {
    const int64_t runs = (nb + kMeanRun - 1) / kMeanRun;
    if (runs > 0x7FFFFFFF) return cudaErrorInvalidValue;
    cudaLaunchAttribute attr[1];
    const cudaLaunchConfig_t cfg = pdl_config(static_cast<unsigned>(runs), 1024, st, attr);
    return cudaLaunchKernelEx(&cfg, dq_mean_kernel, absmax, nb, static_cast<double*>(scratch),
                              dq_mean_ticket(scratch, nb), mean);
}

cudaError_t launch_dq_groups(const float* absmax, int64_t nb, const float* mean, uint8_t* q, float* s2,
                             cudaStream_t st) {
    const int64_t ng = (nb + kGroup - 1) / kGroup;
    cudaLaunchAttribute attr[1];
    const cudaLaunchConfig_t cfg = pdl_config(static_cast<unsigned>((ng * 32 + 255) / 256), 256, st, attr);
    return cudaLaunchKernelEx(&cfg, dq_groups_kernel, absmax, nb, static_cast<const float*>(mean), q, s2);
}
cudaError_t launch_nf4_dequant(const CUtensorMap& out_map, const uint8_t* codes, const BlockConstants& c, int64_t N,
                               int64_t K, const Nf4Tables& tab, int num_sms, cudaStream_t st) {
    const int64_t nb = N * K / kBlock;
    const int64_t nchunks = (nb + kDeqChunk - 1) / kDeqChunk;
    const int grid = static_cast<int>(std::min<int64_t>(nchunks, static_cast<int64_t>(num_sms) * 6));
    const uint4* cw = reinterpret_cast<const uint4*>(codes);
    if (c.absmax)
        nf4_dequant_kernel<true><<<grid, kDeqChunk, kDequantSmem, st>>>(out_map, cw, nullptr, nullptr, nullptr,
                                                                         c.absmax, nb, tab);
    else
        nf4_dequant_kernel<false><<<grid, kDeqChunk, kDequantSmem, st>>>(out_map, cw, c.qabsmax, c.s2, c.mean,
                                                                          nullptr, nb, tab);
    return cudaGetLastError();
}

cudaError_t launch_decode_constants_t(const BlockConstants& c, int64_t N, int64_t K, int64_t ldc, int64_t cols,
                                      float* cT, cudaStream_t st) {
    const int64_t KB = K / kBlock;
    if ((cols & 3) || (ldc & 3) || (reinterpret_cast<uintptr_t>(cT) & 15)) return cudaErrorInvalidValue;
    dim3 grid(static_cast<unsigned>((KB + 63) / 64), static_cast<unsigned>((cols + 63) / 64));
    if (c.absmax)
        decode_constants_t_kernel<true><<<grid, 256, 0, st>>>(nullptr, nullptr, nullptr, c.absmax, N, KB, ldc, cols, cT);
    else
        decode_constants_t_kernel<false><<<grid, 256, 0, st>>>(c.qabsmax, c.s2, c.mean, nullptr, N, KB, ldc, cols,
                                                               cT);
    return cudaGetLastError();
}

cudaError_t launch_decode_constants(const BlockConstants& c, int64_t nb, float* out, int num_sms, cudaStream_t st) {
    const int grid = grid_for(nb, 256, 8 * num_sms);
    if (c.absmax)
        decode_constants_kernel<true><<<grid, 256, 0, st>>>(nullptr, nullptr, nullptr, c.absmax, nb, out);
    else
        decode_constants_kernel<false><<<grid, 256, 0, st>>>(c.qabsmax, c.s2, c.mean, nullptr, nb, out);
    return cudaGetLastError();
}

cudaError_t launch_e4m3_encode(const float* x, uint8_t* q, int64_t n, cudaStream_t st) {
    e4m3_encode_kernel<<<grid_for(n, 256, 4096), 256, 0, st>>>(x, q, n);
    return cudaGetLastError();
}

}  // namespace qlora
