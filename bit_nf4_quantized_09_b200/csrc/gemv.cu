// Small-batch forward (a few tokens) on the tcgen05 tensor core: the
// weight-streaming, memory-bound regime. "ta-paperlens QLoRA explainer",
// 落とし穴: 4-bit weights pay off in small-batch, token-at-a-time generation
// because far fewer bytes are read. The default routing sends up to 16 tokens
// to the register-fed kernel (gemv_mma.cu) and more to the tiled GEMM (split
// over K when its tiles are fewer than the SMs), which measured faster; this
// kernel serves up to 64 tokens when QLORA_OPT_SMALL_M_MAX and
// QLORA_OPT_REG_GEMV_MAX_M select it.
//
// Swap-AB on the tensor core: D[128 weight rows, Mp tokens] accumulates
// deq(W)[rows, k] . X[tokens, k]^T, so the dequantised weight tile fills the
// UMMA M = 128 side and the tokens (padded to Mp = 16..64) the N side.
// Each CTA streams one 128-row tile over a slice of K (split-K for SM fill).
// The split CTAs of a row tile write fp32 partials; the last one to finish
// (atomic ticket, no waiting) adds them in split order, adds the rank-r term
// sT . B^T and writes Y in bf16.
//   warps 0-7  dequantisers: weight row t & 127, half (t >> 7) of each
//              64-weight block, so every row has two threads; warps 0-3
//              then run the epilogue (TMEM lane = weight row)
//   warp 8     TMA producer: X tile, packed codes, decoded constants
//   warp 9     TMEM owner + UMMA issuer
// Input stages (TMA) and dequantised-tile stages are separate rings, so the
// producer can run several steps ahead of the dequantisers.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace qlora {

namespace {

// Input stage (one 64-deep step): X tile [Mp x 64] bf16 (128-byte rows,
// 1 KB aligned), packed codes [128 rows x 32 B], decoded constants [128].
// Its size depends on Mp, so as many stages as fit the input budget are used
// (up to kMaxInStages), to keep enough loads in flight on long K.
constexpr uint32_t kCodeTile = 128 * 32;    // 4 KB packed
constexpr uint32_t kCTile = 128 * 4;        // 512 B constants
constexpr int kMaxInStages = 10;
constexpr uint32_t kInBudget = 40 * 1024;  // with the 32 KB ring: three CTAs per SM
constexpr uint32_t kWTile = 128 * 64 * 2;   // 16 KB dequantised bf16
constexpr int kWStages = 2;
constexpr uint32_t kWOff = kInBudget;
constexpr uint32_t kBarOff = kWOff + kWStages * kWTile;
constexpr uint32_t kSmem = kBarOff + 512 + 1024;
constexpr uint32_t kTmemCols = 64;
constexpr int kDeqWarps = 8;

static_assert(kGemvThreads == 320, "warp roles");

__host__ __device__ constexpr uint32_t gemv_in_stage_bytes(int Mp) {
    return (static_cast<uint32_t>(Mp) * 128u + kCodeTile + kCTile + 1023u) & ~1023u;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ void sts128(uint32_t addr, const uint32_t (&v)[4]) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3])
                 : "memory");
}

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// sum_j sT[j] * B[j] over bf16 operands, fp32 products and sums in order.
__device__ __forceinline__ float lora_dot(const uint16_t* sT, const uint16_t* b, int r) {
    const uint32_t* t2 = reinterpret_cast<const uint32_t*>(sT);
    const uint32_t* b2 = reinterpret_cast<const uint32_t*>(b);
    float acc = 0.0f;
#pragma unroll 4
    for (int j = 0; j < r / 2; ++j) {
        const uint32_t tj = __ldg(t2 + j), bj = __ldg(b2 + j);
        acc = __fmaf_rn(__uint_as_float(tj << 16), __uint_as_float(bj << 16), acc);
        acc = __fmaf_rn(__uint_as_float(tj & 0xFFFF0000u), __uint_as_float(bj & 0xFFFF0000u), acc);
    }
    return acc;
}

__global__ void __launch_bounds__(kGemvThreads, 3)
    gemv_nf4_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_codes,
                    const __grid_constant__ CUtensorMap tm_c, const GemvArgs args, const Nf4Tables tab) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* in_full = reinterpret_cast<uint64_t*>(smem + kBarOff);
    uint64_t* in_empty = in_full + kMaxInStages;
    uint64_t* w_full = in_empty + kMaxInStages;
    uint64_t* w_empty = w_full + kWStages;
    uint64_t* acc = w_empty + kWStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n0 = static_cast<int64_t>(blockIdx.x) * 128;
    const int KT = static_cast<int>(args.K / 64);
    const int k_begin = blockIdx.y * args.steps_per_split;
    const int k_end = min(k_begin + args.steps_per_split, KT);
    const int steps = max(k_end - k_begin, 0);
    const int Mp = args.Mp;
    const uint32_t x_bytes = static_cast<uint32_t>(Mp) * 128u;
    const uint32_t in_stage = gemv_in_stage_bytes(Mp);
    const uint32_t off_codes = x_bytes, off_c = x_bytes + kCodeTile;
    const int n_in = min(kMaxInStages, static_cast<int>(kInBudget / in_stage));
    const uint64_t tmo = args.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kMaxInStages; ++s) {
            mbar_init(in_full + s, 1);
            mbar_init(in_empty + s, 1);
        }
        for (int s = 0; s < kWStages; ++s) {
            mbar_init(w_full + s, kDeqWarps);  // one arrive per dequant warp
            mbar_init(w_empty + s, 1);
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
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_codes);
        tma_prefetch_desc(&tm_c);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 8) {
        // ---------------------------------------------------- producer --
        if (lane == 0) {
            int last_use[kMaxInStages];
            for (int s = 0; s < kMaxInStages; ++s) last_use[s] = -1;
            for (int i = 0; i < steps; ++i) {
                const int s = i % n_in;
                const uint32_t u = static_cast<uint32_t>(i / n_in);
                if (i >= n_in && !mbar_wait(in_empty + s, (u - 1) & 1u, tmo, args.status)) {
                    *abort_flag = 1;
                    break;
                }
                if (*abort_flag) break;
                const int kt = k_begin + i;
                uint8_t* st = smem + s * in_stage;
                mbar_arrive_expect_tx(in_full + s, x_bytes + kCodeTile + kCTile);
                tma_load_2d(st, &tm_x, in_full + s, kt * 64, 0);
                tma_load_2d(st + off_codes, &tm_codes, in_full + s, kt * 32, static_cast<int>(n0));
                tma_load_2d(st + off_c, &tm_c, in_full + s, static_cast<int>(n0), kt);
                last_use[s] = static_cast<int>(u);
            }
            for (int s = 0; s < n_in; ++s)
                if (last_use[s] >= 0) mbar_wait(in_full + s, static_cast<uint32_t>(last_use[s]) & 1u, tmo, nullptr);
        }
        __syncwarp();
    } else if (warp == 9) {
        // --------------------------------------------------------- MMA --
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, Mp, false, false);
            bool ok = true;
            for (int i = 0; i < steps; ++i) {
                const int s = i % n_in, ws = i % kWStages;
                if (!mbar_wait(in_full + s, static_cast<uint32_t>(i / n_in) & 1u, tmo, args.status)) {
                    ok = false;
                    break;
                }
                if (!mbar_wait(w_full + ws, static_cast<uint32_t>(i / kWStages) & 1u, tmo, args.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t xt = smem_u32(smem + s * in_stage), wt = smem_u32(smem + kWOff + ws * kWTile);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16(tmem, sw128_desc(wt + kk * 32, 16, 1024), sw128_desc(xt + kk * 32, 16, 1024), idesc,
                             (i > 0 || kk > 0) ? 1u : 0u);
                umma_commit(in_empty + s);
                umma_commit(w_empty + ws);
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
        // -------------------------------------------------- dequantise --
        const int row = threadIdx.x & 127;  // weight row n0 + row
        const int half = threadIdx.x >> 7;  // weights [32 half, 32 half + 32) of each block
        bool ok = true;
        for (int i = 0; i < steps; ++i) {
            const int s = i % n_in, ws = i % kWStages;
            bool got = mbar_wait(in_full + s, static_cast<uint32_t>(i / n_in) & 1u, tmo, args.status);
            if (got && i >= kWStages)
                got = mbar_wait(w_empty + ws, static_cast<uint32_t>(i / kWStages - 1) & 1u, tmo, args.status);
            ok = __all_sync(0xFFFFFFFFu, got);
            if (!ok) break;
            uint8_t* st = smem + s * in_stage;
            // 32-byte rows of codes, 32-byte swizzle: logical chunk `half` of row `row`
            const uint32_t code_addr = smem_u32(st + off_codes) + row * 32 + ((half ^ ((row >> 2) & 1)) << 4);
            const float cprime = reinterpret_cast<const float*>(st + off_c)[row];
            const Nf4BlockLut lut = make_block_lut(tab.level, cprime);
            const uint4 a = lds128(code_addr);
            const uint32_t words[4] = {a.x, a.y, a.z, a.w};
            const uint32_t wrow = smem_u32(smem + kWOff + ws * kWTile) + row * 128;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t o[4];
                lut_decode8(lut, words[j], o);
                const uint32_t chunk = static_cast<uint32_t>(4 * half + j);
                sts128(wrow + ((chunk ^ (row & 7)) << 4), o);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(w_full + ws);
        }
        if (!ok) *abort_flag = 1;

        if (warp < 4) {
            // -------------------------------------------------- epilogue --
            // thread = weight row n; TMEM columns = tokens, 16 at a time
            const bool acc_ok = __all_sync(0xFFFFFFFFu, mbar_wait(acc, 0, tmo, args.status));
            tc_fence_after();
            const bool good = acc_ok && !*abort_flag && steps > 0;
            const int64_t n = n0 + warp * 32 + lane;
            const int64_t M = args.M, N = args.N;
            const int r = args.r;
            const bool single = args.splits == 1;
            float* my_part = args.part + static_cast<int64_t>(blockIdx.y) * M * N;
#pragma unroll 1
            for (int c0 = 0; c0 < Mp; c0 += 16) {
                uint32_t v[16];
                tmem_ld16(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c0, v);
                tmem_ld_wait();
                if (n < N) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int64_t m = c0 + i;
                        if (m < M) {
                            const float x = good ? __uint_as_float(v[i]) : 0.0f;
                            if (single)
                                args.Y[m * N + n] =
                                    static_cast<uint16_t>(pack_bf16x2(x + lora_dot(args.sT + m * r, args.B + n * r, r),
                                                                      0.0f) & 0xFFFFu);
                            else
                                my_part[m * N + n] = x;
                        }
                    }
                }
            }
            if (!single) {
                __threadfence();  // publish this split's partials before taking a ticket
                epi_bar();
                if (threadIdx.x == 0) {
                    const int ticket = atomicAdd(args.counter + blockIdx.x, 1);
                    *last_flag = (ticket == args.splits - 1) ? 1 : 0;
                }
                epi_bar();
                if (*last_flag) {
                    __threadfence();  // see the other splits' partials
                    if (n < N) {
#pragma unroll 1
                        for (int64_t m = 0; m < M; ++m) {
                            // splits in order, four loads in flight at a time
                            float acc_m = 0.0f;
                            for (int s0 = 0; s0 < args.splits; s0 += 4) {
                                float x[4];
#pragma unroll
                                for (int u = 0; u < 4; ++u)
                                    x[u] = (s0 + u < args.splits)
                                               ? __ldcg(args.part + (static_cast<int64_t>(s0 + u) * M + m) * N + n)
                                               : 0.0f;
                                acc_m += x[0];
                                acc_m += x[1];
                                acc_m += x[2];
                                acc_m += x[3];
                            }
                            args.Y[m * N + n] = static_cast<uint16_t>(
                                pack_bf16x2(acc_m + lora_dot(args.sT + m * r, args.B + n * r, r), 0.0f) & 0xFFFFu);
                        }
                    }
                    if (threadIdx.x == 0) args.counter[blockIdx.x] = 0;  // ready for the next call
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
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

}  // namespace qlora
