// Rank-r ("skinny") matmuls of the LoRA path on the sm_100 tensor core.
//
// "waylandz ch.26" 26.2.4: y = W x + (alpha/r) B (A x). The down-projections
// X A^T (forward) and dY B (backward) and the adapter gradients
//   dA = s (dY B)^T X,  dB = s dY^T (X A^T)
// ("ta-paperlens QLoRA explainer", 勾配は実際どこへ行くのか: only A and B keep
// a gradient) all have one side of width r <= 64. Each is computed as
// D[rows, NR] = A_op[rows, red] . B_op[NR, red]^T with NR = max(16, r) on
// the UMMA N side, split over the reduction into fp32 partials that a second,
// deterministic pass adds in a fixed order.
//   warp 0 TMA producer, warp 1 TMEM owner + UMMA issuer, warps 2-5 epilogue.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace qlora {

namespace {

constexpr uint32_t kABytes = 128 * 64 * 2;  // 16 KB
constexpr uint32_t kBBytes = 64 * 64 * 2;   // up to 64 rows of 128 B
constexpr uint32_t kStage = kABytes + kBBytes;
constexpr uint32_t kBarOff = kSkinnyStages * kStage;
constexpr uint32_t kSmem = kBarOff + 256 + 1024;
constexpr uint32_t kTmemCols = 64;

__global__ void __launch_bounds__(kSkinnyThreads, 1)
    skinny_gemm(const __grid_constant__ CUtensorMap tm_a0, const __grid_constant__ CUtensorMap tm_b0,
                const __grid_constant__ CUtensorMap tm_a1, const __grid_constant__ CUtensorMap tm_b1,
                const SkinnyArgs args) {
    const int prob = blockIdx.z;
    const SkinnyProblem& P = args.p[prob];
    const int64_t row0 = static_cast<int64_t>(blockIdx.x) * 128;
    if (row0 >= P.rows || static_cast<int>(blockIdx.y) >= P.splits) return;  // whole CTA idle
    const CUtensorMap* ta = prob ? &tm_a1 : &tm_a0;
    const CUtensorMap* tb = prob ? &tm_b1 : &tm_b0;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOff);
    uint64_t* empty = full + kSkinnyStages;
    uint64_t* acc = empty + kSkinnyStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int NR = args.NR;
    const int KT = static_cast<int>((P.red + 63) / 64);
    const int k_begin = blockIdx.y * P.steps_per_split;
    const int k_end = min(k_begin + P.steps_per_split, KT);
    const int steps = max(k_end - k_begin, 0);
    const uint64_t tmo = args.timeout_ns;
    const uint32_t b_bytes = static_cast<uint32_t>(NR) * 128u;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSkinnyStages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        mbar_init(acc, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            int last_use[kSkinnyStages];
            for (int s = 0; s < kSkinnyStages; ++s) last_use[s] = -1;
            for (int i = 0; i < steps; ++i) {
                const int s = i % kSkinnyStages;
                const uint32_t u = static_cast<uint32_t>(i / kSkinnyStages);
                if (i >= kSkinnyStages && !mbar_wait(empty + s, (u - 1) & 1u, tmo, args.status)) {
                    *abort_flag = 1;
                    break;
                }
                if (*abort_flag) break;
                const int k = (k_begin + i) * 64;
                uint8_t* st = smem + s * kStage;
                mbar_arrive_expect_tx(full + s, kABytes + b_bytes);
                if (!args.a_mn_major) {
                    tma_load_2d(st, ta, full + s, k, static_cast<int>(row0));
                } else {
                    tma_load_2d(st, ta, full + s, static_cast<int>(row0), k);
                    tma_load_2d(st + 8192, ta, full + s, static_cast<int>(row0) + 64, k);
                }
                tma_load_2d(st + kABytes, tb, full + s, k, 0);
                last_use[s] = static_cast<int>(u);
            }
            for (int s = 0; s < kSkinnyStages; ++s)
                if (last_use[s] >= 0) mbar_wait(full + s, static_cast<uint32_t>(last_use[s]) & 1u, tmo, nullptr);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, NR, args.a_mn_major != 0, false);
            bool ok = true;
            for (int i = 0; i < steps; ++i) {
                const int s = i % kSkinnyStages;
                const uint32_t u = static_cast<uint32_t>(i / kSkinnyStages);
                if (!mbar_wait(full + s, u & 1u, tmo, args.status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t a = smem_u32(smem + s * kStage), b = a + kABytes;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t adesc = args.a_mn_major ? sw128_desc(a + kk * 2048, 8192, 1024)
                                                           : sw128_desc(a + kk * 32, 16, 1024);
                    const uint64_t bdesc = sw128_desc(b + kk * 32, 16, 1024);
                    umma_f16(tmem, adesc, bdesc, idesc, (i > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(empty + s);
            }
            if (!ok) {
                *abort_flag = 1;
                __threadfence_block();
            }
            umma_commit(acc);
            mbar_wait(acc, 0, tmo, args.status);
        }
        __syncwarp();
    } else {
        // epilogue warps 2..5 -> TMEM lane quarters 2, 3, 0, 1
        const bool ok = mbar_wait(acc, 0, tmo, args.status);
        tc_fence_after();
        const int q = warp & 3;
        const int64_t row = row0 + q * 32 + lane;
        float* out = P.part + (static_cast<int64_t>(blockIdx.y) * P.rows + row) * NR;
        for (int c0 = 0; c0 < NR; c0 += 16) {
            uint32_t r[16];
            tmem_ld16(tmem + (static_cast<uint32_t>(q * 32) << 16) + c0, r);
            tmem_ld_wait();
            if (row < P.rows) {
                float4* dst = reinterpret_cast<float4*>(out + c0);
                const bool good = ok && !*abort_flag && steps > 0;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float4 v = good ? make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                                  __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]))
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
                    dst[i] = v;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------- reductions --

__global__ void reduce_lora_down_kernel(const float* __restrict__ part, int splits, int64_t M, int NR, int r,
                                        float scale, uint16_t* __restrict__ out_rm, uint16_t* __restrict__ out_t,
                                        int64_t ldt) {
    const int64_t total = M * r;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t m = i / r;
        const int j = static_cast<int>(i % r);
        float acc = 0.0f;
        for (int s = 0; s < splits; ++s) acc += part[(s * M + m) * NR + j];
        const uint16_t b = static_cast<uint16_t>(pack_bf16x2(__fmul_rn(scale, acc), 0.0f) & 0xFFFFu);
        out_rm[m * r + j] = b;
        if (out_t) out_t[static_cast<int64_t>(j) * ldt + m] = b;
    }
}

__global__ void reduce_lora_grads_kernel(const float* __restrict__ partA, int splitsA, int64_t K,
                                         const float* __restrict__ partB, int splitsB, int64_t N, int NR, int r,
                                         float* __restrict__ dA, float* __restrict__ dB) {
    const int64_t totalA = static_cast<int64_t>(r) * K, totalB = N * r;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < totalA + totalB;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        if (i < totalA) {
            const int j = static_cast<int>(i / K);
            const int64_t k = i % K;
            float acc = 0.0f;
            for (int s = 0; s < splitsA; ++s) acc += partA[(s * K + k) * NR + j];
            dA[i] = acc;
        } else {
            const int64_t t = i - totalA;
            const int64_t n = t / r;
            const int j = static_cast<int>(t % r);
            float acc = 0.0f;
            for (int s = 0; s < splitsB; ++s) acc += partB[(s * N + n) * NR + j];
            dB[t] = acc;
        }
    }
}

__global__ void transpose_bf16_kernel(const uint16_t* __restrict__ in, int64_t rows, int64_t cols,
                                      uint16_t* __restrict__ out, int64_t ldo) {
    __shared__ uint16_t tile[32][33];
    const int64_t r0 = static_cast<int64_t>(blockIdx.y) * 32, c0 = static_cast<int64_t>(blockIdx.x) * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    for (int i = ty; i < 32; i += 8) {
        const int64_t rr = r0 + i, cc = c0 + tx;
        tile[i][tx] = (rr < rows && cc < cols) ? in[rr * cols + cc] : 0;
    }
    __syncthreads();
    for (int i = ty; i < 32; i += 8) {
        const int64_t cc = c0 + i, rr = r0 + tx;
        if (cc < cols && rr < rows) out[cc * ldo + rr] = tile[tx][i];
    }
}

}  // namespace

size_t skinny_smem_bytes() { return kSmem; }

cudaError_t launch_skinny(const CUtensorMap& a0, const CUtensorMap& b0, const CUtensorMap& a1, const CUtensorMap& b1,
                          const SkinnyArgs& args, int nproblems, cudaStream_t st) {
    int64_t max_tiles = 0;
    int max_splits = 0;
    for (int p = 0; p < nproblems; ++p) {
        max_tiles = std::max<int64_t>(max_tiles, (args.p[p].rows + 127) / 128);
        max_splits = std::max(max_splits, args.p[p].splits);
    }
    dim3 grid(static_cast<unsigned>(max_tiles), static_cast<unsigned>(max_splits), static_cast<unsigned>(nproblems));
    skinny_gemm<<<grid, kSkinnyThreads, kSmem, st>>>(a0, b0, a1, b1, args);
    return cudaGetLastError();
}

cudaError_t skinny_init_device() {
    return cudaFuncSetAttribute(skinny_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmem));
}

cudaError_t launch_reduce_lora_down(const float* part, int splits, int64_t M, int NR, int r, float scale,
                                    uint16_t* out_rm, uint16_t* out_t, int64_t ldt, cudaStream_t st) {
    const int64_t total = M * r;
    const int grid = static_cast<int>(std::min<int64_t>((total + 255) / 256, 4096));
    reduce_lora_down_kernel<<<std::max(grid, 1), 256, 0, st>>>(part, splits, M, NR, r, scale, out_rm, out_t, ldt);
    return cudaGetLastError();
}

cudaError_t launch_reduce_lora_grads(const float* partA, int splitsA, int64_t K, const float* partB, int splitsB,
                                     int64_t N, int NR, int r, float* dA, float* dB, cudaStream_t st) {
    const int64_t total = static_cast<int64_t>(r) * K + N * r;
    const int grid = static_cast<int>(std::min<int64_t>((total + 255) / 256, 8192));
    reduce_lora_grads_kernel<<<std::max(grid, 1), 256, 0, st>>>(partA, splitsA, K, partB, splitsB, N, NR, r, dA,
                                                                dB);
    return cudaGetLastError();
}

cudaError_t launch_transpose_bf16(const uint16_t* in, int64_t rows, int64_t cols, uint16_t* out, int64_t ldo,
                                  cudaStream_t st) {
    dim3 grid(static_cast<unsigned>((cols + 31) / 32), static_cast<unsigned>((rows + 31) / 32));
    transpose_bf16_kernel<<<grid, 256, 0, st>>>(in, rows, cols, out, ldo);
    return cudaGetLastError();
}

}  // namespace qlora
