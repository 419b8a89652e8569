// Rank-r ("skinny") matmuls of the LoRA path on the sm_100 tensor core.
//
// "waylandz ch.26" 26.2.4: y = W x + (alpha/r) B (A x). The down-projections
//   sT = s X A^T (forward),  sU = s dY B (backward)
// and the adapter gradients ("ta-paperlens QLoRA explainer",
// 勾配は実際どこへ行くのか: only A and B keep a gradient)
//   dA = sU^T X,  dB = dY^T sT
// all have one side of width r <= 64. Each is D[rows, NR] = A_op[rows, red] .
// B_op[NR, red]^T with NR = max(16, r) on the UMMA N side:
//   A_op  K-major (X, dY read along the reduction) or MN-major (X^T, dY^T
//         read by TMA straight out of X and dY with the 128-byte swizzle);
//   B_op  K-major (A [r, K]) or MN-major (B [N, r], sU and sT [M, r] read in
//         place with a 32/64/128-byte swizzle matching NR).
// The reduction is split over the S <= 8 CTAs of a thread-block cluster
// (grid.y). Each CTA leaves its fp32 accumulator in its own shared memory;
// after a cluster barrier CTA c sums rows [c 128/S, (c + 1) 128/S) of the
// tile over the S CTAs in rank order through distributed shared memory and
// writes them, so outputs are deterministic and no partials reach global
// memory. One launch carries up to eight such problems (grid.z), each with
// its own pair of operand maps: the 64-column chunks of a rank above 64
// (several adapters side by side), the projections of a group, or dA and dB
// together. A bf16 output may zero, per token row, the columns of the
// adapters that the row does not use.
//   warp 0 TMA producer, warp 1 TMEM owner + UMMA issuer, warps 2-5 epilogue.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace qlora {

namespace {

constexpr uint32_t kABytes = 128 * 64 * 2;  // 16 KB
constexpr uint32_t kBBytes = 64 * 64 * 2;   // up to 64 x 64 bf16
constexpr uint32_t kStage = kABytes + kBBytes;  // per 64-deep chunk of a stage
constexpr uint32_t kTmemCols = 64;
constexpr uint32_t kRowBytes = 256;  // one fp32 accumulator row of 64 columns in the reduction buffer
__host__ __device__ constexpr uint32_t smem_bytes(int stages, int chunks) {
    return stages * chunks * kStage + 256 + 1024;
}

// Shared-memory descriptor of an MN-major B tile [64 reduction rows, NR
// columns] written by TMA with the swizzle whose span is NR * 2 bytes: rows of
// NR*2 bytes, 8-row groups SBO = 8 * NR * 2 apart.
__device__ __forceinline__ uint64_t mn_b_desc(uint32_t addr, int NR) {
    const uint32_t row = static_cast<uint32_t>(NR) * 2u;
    const uint32_t layout = NR == 16 ? 6u : (NR == 32 ? 4u : 2u);  // SW32, SW64, SW128
    uint64_t d = 0;
    d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(1u) << 16;  // leading byte offset: one atom spans all NR columns
    d |= static_cast<uint64_t>(((8u * row) >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    d |= static_cast<uint64_t>(layout) << 61;
    return d;
}

__global__ void __launch_bounds__(kSkinnyThreads, 1)
    skinny_gemm(const __grid_constant__ SkinnyMaps maps, const __grid_constant__ SkinnyArgs args) {
    // a launch that depends on this one programmatically may be scheduled
    // now; it waits for this grid's completion before reading its output
    asm volatile("griddepcontrol.launch_dependents;");
    const int prob = blockIdx.z;
    const SkinnyProblem P = args.p[prob];
    const int64_t row0 = static_cast<int64_t>(blockIdx.x) * 128;
    if (row0 >= P.rows) return;  // the whole cluster (same row tile) is idle
    const CUtensorMap* ta = &maps.a[prob];
    const CUtensorMap* tb = &maps.b[prob];

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int stages = args.stages, C = args.chunks;
    const uint32_t stage_bytes = static_cast<uint32_t>(C) * kStage;  // C A chunks, then C B chunks
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + stages * stage_bytes);
    uint64_t* empty = full + kSkinnyMaxStages;
    uint64_t* acc = empty + kSkinnyMaxStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int NR = args.NR;
    // the splits interleave: split y takes steps y, y + S, y + 2S, ... (of C
    // chunks each), so the cluster's CTAs read neighbouring pieces of each row
    // at the same time
    const int KT = static_cast<int>((P.red + 64 * C - 1) / (64 * C));
    const int S = args.splits, y = static_cast<int>(blockIdx.y);
    const int steps = y < KT ? (KT - y + S - 1) / S : 0;
    const uint64_t tmo = args.timeout_ns;
    const uint32_t b_bytes = static_cast<uint32_t>(NR) * 128u;

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
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
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(ta);
        tma_prefetch_desc(tb);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            int last = -1;
            for (int i = 0; i < steps; ++i) {
                const int s = i % stages;
                const uint32_t u = static_cast<uint32_t>(i / stages);
                if (i >= stages && !mbar_wait(empty + s, (u - 1) & 1u, tmo, args.status)) {
                    *abort_flag = 1;
                    break;
                }
                if (*abort_flag) break;
                uint8_t* st = smem + s * stage_bytes;
                mbar_arrive_expect_tx(full + s, static_cast<uint32_t>(C) * (kABytes + b_bytes));
                const int ar = static_cast<int>(row0);
                // the A chunks first, back to back: C * 128 contiguous bytes of each row in flight together
                for (int j = 0; j < C; ++j) {
                    const int k = ((i * S + y) * C + j) * 64;
                    uint8_t* sa = st + j * kABytes;
                    if (!P.a_mn_major) {
                        tma_load_2d(sa, ta, full + s, k, ar);
                    } else {
                        tma_load_2d(sa, ta, full + s, ar, k);
                        tma_load_2d(sa + 8192, ta, full + s, ar + 64, k);
                    }
                }
                for (int j = 0; j < C; ++j) {
                    const int k = ((i * S + y) * C + j) * 64;
                    uint8_t* sb = st + C * kABytes + j * kBBytes;
                    if (!P.b_mn_major)
                        tma_load_2d(sb, tb, full + s, k, 0);
                    else
                        tma_load_2d(sb, tb, full + s, 0, k);
                }
                last = i;
            }
            // every copy in flight has landed before the stages are reused
            for (int i = max(0, last - stages + 1); i <= last; ++i)
                mbar_wait(full + i % stages, static_cast<uint32_t>(i / stages) & 1u, tmo, nullptr);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, NR, P.a_mn_major != 0, P.b_mn_major != 0);
            bool ok = true;
            for (int i = 0; i < steps; ++i) {
                const int s = i % stages;
                const uint32_t u = static_cast<uint32_t>(i / stages);
                if (!mbar_wait(full + s, u & 1u, tmo, args.status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t st = smem_u32(smem + s * stage_bytes);
                for (int j = 0; j < C; ++j) {
                    const uint32_t a = st + j * kABytes, b = st + C * kABytes + j * kBBytes;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t adesc = P.a_mn_major ? sw128_desc(a + kk * 2048, 8192, 1024)
                                                            : sw128_desc(a + kk * 32, 16, 1024);
                        const uint64_t bdesc = P.b_mn_major ? mn_b_desc(b + kk * 16 * NR * 2, NR)
                                                            : sw128_desc(b + kk * 32, 16, 1024);
                        umma_f16(tmem, adesc, bdesc, idesc, (i > 0 || j > 0 || kk > 0) ? 1u : 0u);
                    }
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
        // epilogue warps 2..5 -> TMEM lane quarters 2, 3, 0, 1; thread = tile
        // row t. The accumulator row goes to this CTA's reduction buffer in
        // the first stages (idle: every UMMA has completed and every copy has
        // landed): 16-byte chunk c of row t at t * 256 + ((c ^ (t & 7)) << 4),
        // so eight consecutive rows fill all banks.
        const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(acc, 0, tmo, args.status));
        tc_fence_after();
        const int q = warp & 3;
        const int t = q * 32 + lane;
        const bool good = ok && !*abort_flag && steps > 0;
        const uint32_t buf = smem_u32(smem) + static_cast<uint32_t>(t) * kRowBytes;
#pragma unroll
        for (int c0 = 0; c0 < 64; c0 += 16) {
            if (c0 < NR) {
                uint32_t r[16];
                tmem_ld16(tmem + (static_cast<uint32_t>(q * 32) << 16) + c0, r);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t w4[4] = {good ? r[4 * i] : 0u, good ? r[4 * i + 1] : 0u, good ? r[4 * i + 2] : 0u,
                                            good ? r[4 * i + 3] : 0u};
                    const uint32_t c = static_cast<uint32_t>(c0 / 4 + i);
                    sts128(buf + ((c ^ static_cast<uint32_t>(t & 7)) << 4), w4);
                }
            }
        }
    }

    // every CTA of the cluster has its accumulator in shared memory
    tc_fence_before();
    cluster_sync();

    // CTA `rank` sums its slice of rows over the cluster in rank order and
    // writes it. Items are (row, 4-column chunk) pairs: row-major outputs take
    // the chunks of a row on neighbouring threads, the transposed output the
    // rows of a chunk.
    {
        const int rank = static_cast<int>(cluster_ctarank());
        const int rows_per = 128 / S, chunks = NR / 4;
        const bool by_row = P.mode == kSkinnyOutF32Transposed;
        const uint32_t buf0 = smem_u32(smem);
        const int id_rows = P.row_ids != nullptr;
        for (int it = threadIdx.x; it < rows_per * chunks; it += kSkinnyThreads) {
            const int rl = by_row ? it % rows_per : it / chunks;
            const int c = by_row ? it / rows_per : it % chunks;
            const int t = rank * rows_per + rl;
            const int64_t row = row0 + t;
            if (row >= P.rows || 4 * c >= P.ncols) continue;
            const uint32_t off = static_cast<uint32_t>(t) * kRowBytes + ((static_cast<uint32_t>(c) ^ (t & 7)) << 4);
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int s = 0; s < S; ++s) {
                const float4 x = ld_cluster_f4(mapa_shared(buf0 + off, static_cast<uint32_t>(s)));
                v.x += x.x;
                v.y += x.y;
                v.z += x.z;
                v.w += x.w;
            }
            const int j = 4 * c;
            if (P.mode == kSkinnyOutBf16) {
                // the adapter of this token row (row_ids set): columns of
                // other adapters are written as zeros
                const int id = id_rows ? __ldg(P.row_ids + row) : 0;
                const bool keep = !id_rows || (P.ids_col0 + j) / P.ids_r == id;  // 4 columns, one adapter (r >= 8)
                uint2 o;
                o.x = keep ? pack_bf16x2(__fmul_rn(P.scale, v.x), __fmul_rn(P.scale, v.y)) : 0u;
                o.y = keep ? pack_bf16x2(__fmul_rn(P.scale, v.z), __fmul_rn(P.scale, v.w)) : 0u;
                *reinterpret_cast<uint2*>(P.out_bf16 + row * P.out_ld + j) = o;
            } else if (P.mode == kSkinnyOutF32Transposed) {
                P.out_f32[static_cast<int64_t>(j) * P.out_ld + row] = v.x;
                P.out_f32[static_cast<int64_t>(j + 1) * P.out_ld + row] = v.y;
                P.out_f32[static_cast<int64_t>(j + 2) * P.out_ld + row] = v.z;
                P.out_f32[static_cast<int64_t>(j + 3) * P.out_ld + row] = v.w;
            } else {
                *reinterpret_cast<float4*>(P.out_f32 + row * P.out_ld + j) = v;
            }
        }
    }

    // no CTA leaves while another may still read its shared memory
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    // launched as a programmatic dependent (beside a fused matmul), this
    // grid completes only after its primary, so later work on the stream
    // still sees the primary's results; otherwise a no-op
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace

size_t skinny_smem_bytes(int stages, int chunks) { return smem_bytes(stages, chunks); }

cudaError_t launch_skinny(const SkinnyMaps& maps, const SkinnyArgs& args, int nproblems, cudaStream_t st, bool pdl) {
    if (nproblems < 1 || nproblems > kSkinnyMaxProblems) return cudaErrorInvalidValue;
    const int S = args.splits;
    if (S != 1 && S != 2 && S != 4 && S != 8) return cudaErrorInvalidValue;
    // the reduction buffer (32 KB) lies in the stages
    if (args.chunks != 1 && args.chunks != 2 && args.chunks != 4) return cudaErrorInvalidValue;
    if (args.stages < 1 || args.stages * args.chunks < 2 || args.stages * args.chunks > kSkinnyMaxStages)
        return cudaErrorInvalidValue;
    int64_t max_tiles = 0;
    for (int p = 0; p < nproblems; ++p) max_tiles = std::max<int64_t>(max_tiles, (args.p[p].rows + 127) / 128);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(max_tiles), static_cast<unsigned>(S), static_cast<unsigned>(nproblems));
    cfg.blockDim = dim3(kSkinnyThreads);
    cfg.dynamicSmemBytes = smem_bytes(args.stages, args.chunks);
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = static_cast<unsigned>(S);
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, skinny_gemm, maps, args);
}

cudaError_t skinny_init_device() {
    return cudaFuncSetAttribute(skinny_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(smem_bytes(kSkinnyMaxStages, 1)));
}

}  // namespace qlora
