// Small-batch forward (a few tokens): the weight-streaming, memory-bound
// regime. "ta-paperlens QLoRA explainer", 落とし穴: 4-bit weights pay off in
// small-batch, token-at-a-time generation because far fewer bytes are read.
//
// Swap-AB on the tensor core: D[128 weight rows, Mp tokens] accumulates
// deq(W)[rows, k] . X[tokens, k]^T, so the dequantised weight tile fills the
// UMMA M = 128 side and the tokens (padded to Mp = 16..64) the N side.
// Each CTA streams one 128-row tile over a slice of K (split-K for SM fill);
// fp32 partials go to the workspace and a second pass adds them in a fixed
// order together with the rank-r term sT . B^T and rounds Y to bf16.
//   warps 0-3  dequantisers (one weight row each per 64-step), then epilogue
//   warp 4     TMA producer (codes, decoded constants, X tile)
//   warp 5     TMEM owner + UMMA issuer
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace qlora {

namespace {

constexpr uint32_t kWTile = 128 * 64 * 2;   // 16 KB dequantised bf16
constexpr uint32_t kXTile = 64 * 64 * 2;    // up to 64 tokens x 64
constexpr uint32_t kCodeTile = 128 * 32;    // 4 KB packed
constexpr uint32_t kCTile = 128 * 4;        // 512 B constants
constexpr uint32_t kOffX = kWTile;
constexpr uint32_t kOffCodes = kOffX + kXTile;
constexpr uint32_t kOffC = kOffCodes + kCodeTile;
constexpr uint32_t kStage = 29 * 1024;      // kOffC + kCTile rounded up to 1 KB
constexpr int kStages = kGemvStages;
constexpr uint32_t kBarOff = kStages * kStage;
constexpr uint32_t kSmem = kBarOff + 256 + 1024;
constexpr uint32_t kTmemCols = 64;
constexpr int kDeqThreads = 128;

static_assert(kOffC + kCTile <= kStage, "stage layout");

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ void sts128(uint32_t addr, const uint32_t (&v)[4]) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3])
                 : "memory");
}

__global__ void __launch_bounds__(kGemvThreads, 2)
    gemv_nf4_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_codes,
                    const __grid_constant__ CUtensorMap tm_c, const GemvArgs args, const Nf4Tables tab) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOff);
    uint64_t* deq = full + kStages;
    uint64_t* empty = deq + kStages;
    uint64_t* acc = empty + kStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n0 = static_cast<int64_t>(blockIdx.x) * 128;
    const int KT = static_cast<int>(args.K / 64);
    const int k_begin = blockIdx.y * args.steps_per_split;
    const int k_end = min(k_begin + args.steps_per_split, KT);
    const int steps = max(k_end - k_begin, 0);
    const int Mp = args.Mp;
    const uint32_t x_bytes = static_cast<uint32_t>(Mp) * 128u;
    const uint64_t tmo = args.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(deq + s, kDeqThreads);
            mbar_init(empty + s, 1);
        }
        mbar_init(acc, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        if (lane == 0) {
            int last_use[kStages];
            for (int s = 0; s < kStages; ++s) last_use[s] = -1;
            for (int i = 0; i < steps; ++i) {
                const int s = i % kStages;
                const uint32_t u = static_cast<uint32_t>(i / kStages);
                if (i >= kStages && !mbar_wait(empty + s, (u - 1) & 1u, tmo, args.status)) {
                    *abort_flag = 1;
                    break;
                }
                if (*abort_flag) break;
                const int kt = k_begin + i;
                uint8_t* st = smem + s * kStage;
                mbar_arrive_expect_tx(full + s, x_bytes + kCodeTile + kCTile);
                tma_load_2d(st + kOffX, &tm_x, full + s, kt * 64, 0);
                tma_load_2d(st + kOffCodes, &tm_codes, full + s, kt * 32, static_cast<int>(n0));
                tma_load_2d(st + kOffC, &tm_c, full + s, static_cast<int>(n0), kt);
                last_use[s] = static_cast<int>(u);
            }
            for (int s = 0; s < kStages; ++s)
                if (last_use[s] >= 0) mbar_wait(full + s, static_cast<uint32_t>(last_use[s]) & 1u, tmo, nullptr);
        }
        __syncwarp();
    } else if (warp == 5) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, Mp, false, false);
            bool ok = true;
            for (int i = 0; i < steps; ++i) {
                const int s = i % kStages;
                const uint32_t u = static_cast<uint32_t>(i / kStages);
                if (!mbar_wait(full + s, u & 1u, tmo, args.status)) { ok = false; break; }
                if (!mbar_wait(deq + s, u & 1u, tmo, args.status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t wt = smem_u32(smem + s * kStage), xt = wt + kOffX;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16(tmem, sw128_desc(wt + kk * 32, 16, 1024), sw128_desc(xt + kk * 32, 16, 1024), idesc,
                             (i > 0 || kk > 0) ? 1u : 0u);
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
        // ---------------------------------------------------- dequantise --
        const int t = threadIdx.x;  // weight row n0 + t
        bool ok = true;
        for (int i = 0; i < steps; ++i) {
            const int s = i % kStages;
            const uint32_t u = static_cast<uint32_t>(i / kStages);
            if (!mbar_wait(full + s, u & 1u, tmo, args.status)) { ok = false; break; }
            uint8_t* st = smem + s * kStage;
            const uint32_t crow = smem_u32(st + kOffCodes) + t * 32;
            const uint32_t sw = (t >> 2) & 1;  // 32-byte swizzle of the code rows
            const uint32_t wrow = smem_u32(st) + t * 128;
            const float cprime = reinterpret_cast<const float*>(st + kOffC)[t];
            const Nf4BlockLut lut = make_block_lut(tab.level, cprime);
            const uint4 a = lds128(crow + ((0 ^ sw) << 4)), b = lds128(crow + ((1 ^ sw) << 4));
            const uint32_t words[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                uint32_t o[4];
                lut_decode8(lut, words[j], o);
                sts128(wrow + ((static_cast<uint32_t>(j) ^ (t & 7)) << 4), o);
            }
            fence_proxy_async_smem();
            mbar_arrive(deq + s);
        }
        if (!ok) *abort_flag = 1;

        // ------------------------------------------------------ epilogue --
        const bool acc_ok = mbar_wait(acc, 0, tmo, args.status);
        tc_fence_after();
        const bool good = acc_ok && !*abort_flag && steps > 0;
        const int64_t n = n0 + warp * 32 + lane;
        float* part = args.part + static_cast<int64_t>(blockIdx.y) * args.M * args.N;
        for (int c0 = 0; c0 < Mp; c0 += 16) {
            uint32_t r[16];
            tmem_ld16(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c0, r);
            tmem_ld_wait();
            if (n < args.N) {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int64_t m = c0 + i;
                    if (m < args.M) part[m * args.N + n] = good ? __uint_as_float(r[i]) : 0.0f;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Y[m][n] = bf16( sum_s part[s][m][n] + sum_j sT[m][j] * B[n][j] ).
template <int R>
__global__ void __launch_bounds__(256) gemv_reduce_kernel(const float* __restrict__ part, int splits, int64_t M,
                                                          int64_t N, const uint16_t* __restrict__ sT,
                                                          const uint16_t* __restrict__ Bw, uint16_t* __restrict__ Y) {
    __shared__ float s_sT[64 * R];
    for (int i = threadIdx.x; i < M * R; i += blockDim.x) s_sT[i] = __uint_as_float(static_cast<uint32_t>(sT[i]) << 16);
    __syncthreads();
    const int64_t n = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (n >= N) return;
    float b[R];
#pragma unroll
    for (int j = 0; j < R; ++j) b[j] = __uint_as_float(static_cast<uint32_t>(Bw[n * R + j]) << 16);
    for (int64_t m = 0; m < M; ++m) {
        float acc = 0.0f;
        for (int s = 0; s < splits; ++s) acc += part[(s * M + m) * N + n];
        float lora = 0.0f;
#pragma unroll
        for (int j = 0; j < R; ++j) lora = __fmaf_rn(s_sT[m * R + j], b[j], lora);
        Y[m * N + n] = static_cast<uint16_t>(pack_bf16x2(acc + lora, 0.0f) & 0xFFFFu);
    }
}

}  // namespace

size_t gemv_smem_bytes() { return kSmem; }

cudaError_t gemv_init_device() {
    return cudaFuncSetAttribute(gemv_nf4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmem));
}

cudaError_t launch_gemv(const CUtensorMap& x, const CUtensorMap& codes, const CUtensorMap& cT, const GemvArgs& a,
                        const Nf4Tables& tab, cudaStream_t st) {
    dim3 grid(static_cast<unsigned>((a.N + 127) / 128), static_cast<unsigned>(a.splits));
    gemv_nf4_kernel<<<grid, kGemvThreads, kSmem, st>>>(x, codes, cT, a, tab);
    return cudaGetLastError();
}

cudaError_t launch_gemv_reduce(const float* part, int splits, int64_t M, int64_t N, const uint16_t* sT,
                               const uint16_t* B, int r, uint16_t* Y, cudaStream_t st) {
    const unsigned grid = static_cast<unsigned>((N + 255) / 256);
    switch (r) {
        case 8: gemv_reduce_kernel<8><<<grid, 256, 0, st>>>(part, splits, M, N, sT, B, Y); break;
        case 16: gemv_reduce_kernel<16><<<grid, 256, 0, st>>>(part, splits, M, N, sT, B, Y); break;
        case 32: gemv_reduce_kernel<32><<<grid, 256, 0, st>>>(part, splits, M, N, sT, B, Y); break;
        case 64: gemv_reduce_kernel<64><<<grid, 256, 0, st>>>(part, splits, M, N, sT, B, Y); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace qlora
