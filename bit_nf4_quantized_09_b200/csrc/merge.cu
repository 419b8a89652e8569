// Adapter merge on the tensor core: W_out = bf16(fmaf(s, (B A)[n, k], w_hat[n, k])).
//
// "waylandz LLM book ch.26", 26.2.2 (inference: the adapter is folded into the
// weight once, W_merged = W + (alpha/r) B A); "ta-paperlens QLoRA explainer",
// 落とし穴 (the merge goes to the 16-bit weight). w_hat is the dequantised
// weight exactly as the dequantiser computes it.
//
// The work is the dequantiser's stream (half a byte of codes in, two bytes of
// bf16 out per weight) with a rank-r contraction folded into its epilogue, so
// the contraction goes on tcgen05 and the kernel stays bound by HBM. Output
// tiles are 128 rows x 256 columns; a persistent CTA per SM takes a contiguous
// range of them in row-major order (measured 109 vs 134 us on 22016 x 8192
// against a column-major order):
//   warp 8     TMA producer: per tile, B's 128 rows (K-major, 128-byte
//              swizzle, columns past r zero-filled) and A's r x 256 tile
//              (MN-major, four 64-column boxes, rows past r zero-filled) into
//              a 2-stage operand ring, and the tile's packed codes into a
//              3-stage code ring;
//   warp 9     TMEM owner and UMMA issuer: ceil(r/16) tcgen05.mma
//              (M 128, N 256, K 16) per tile into one of two 256-column
//              accumulators, so the epilogue of one tile overlaps the next;
//   warps 0-7  epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 (its rows)
//              and columns 128 (w / 4) .. + 127, decodes the codes of those
//              columns through the per-block lookup, and writes
//              bf16(fmaf(s, acc, w_hat)) 64 columns at a time into a 128-byte
//              swizzled 32-row buffer (two per warp) that one TMA store sends
//              out.
// Every wait is bounded; a wait that runs out records QLORA_ERR_DEVICE_TIMEOUT
// in the status word, abandons the loop and still frees TMEM.
#include "common.cuh"
#include "kernels.h"

namespace qlora {

namespace {

constexpr int kRowsT = 128, kColsT = 256;
constexpr int kEpiWarps = 8;                      // 4 lane quarters x kEpiWarps / 4 column groups
constexpr int kEpiCols = kColsT / (kEpiWarps / 4);  // columns of one epilogue warp
constexpr int kThreadsM = 32 * (kEpiWarps + 2);
constexpr int kWarpProd = kEpiWarps, kWarpMma = kEpiWarps + 1;
constexpr uint32_t kOpB = kRowsT * 128;           // 16 KB: 128 rows x 64 rank columns, bf16
constexpr uint32_t kOpA = 4 * 64 * 128;           // 32 KB: 64 rank rows x 256 columns, bf16
constexpr uint32_t kOpStage = kOpB + kOpA;        // 48 KB
constexpr uint32_t kCodeStage = kRowsT * 128;     // 16 KB: 128 rows x 256 columns of codes
constexpr int kOpStages = 2, kCodeStages = 3;
constexpr uint32_t kOffCodes = kOpStages * kOpStage;
constexpr uint32_t kStageOut = 32 * 128;          // 4 KB: 32 rows x 64 bf16 columns, 128-byte swizzle
constexpr uint32_t kOffScratch = kOffCodes + kCodeStages * kCodeStage;  // 2 output buffers per epilogue warp
constexpr uint32_t kOffBar = kOffScratch + kEpiWarps * 2 * kStageOut;
constexpr uint32_t kSmemM = kOffBar + 256 + 1024;
constexpr uint32_t kTmemColsM = 512;

__global__ void __launch_bounds__(kThreadsM, 1)
    merge_tc_kernel(const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_a,
                    const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_out,
                    const MergeArgs a, const int ksteps, const Nf4Tables tab) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* op_full = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* op_empty = op_full + kOpStages;
    uint64_t* code_full = op_empty + kOpStages;
    uint64_t* code_empty = code_full + kCodeStages;
    uint64_t* acc_full = code_empty + kCodeStages;
    uint64_t* acc_empty = acc_full + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    __shared__ float levels[16];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t N = a.N, K = a.K, KB = K / kBlock;
    const int tiles_r = static_cast<int>((N + kRowsT - 1) / kRowsT);
    const int64_t tiles = static_cast<int64_t>(tiles_r) * ((K + kColsT - 1) / kColsT);
    const uint64_t tmo = a.timeout_ns;
    // this CTA's tiles: a contiguous range in row-major order, so it streams
    // along its rows (whole DRAM pages of codes and output per row)
    const int64_t t_lo = tiles * blockIdx.x / gridDim.x, t_hi = tiles * (blockIdx.x + 1) / gridDim.x;
    const int n_my = static_cast<int>(t_hi - t_lo);
    const int64_t tiles_c = tiles / tiles_r;
    auto tile_n0 = [&](int i) { return ((t_lo + i) / tiles_c) * kRowsT; };
    auto tile_k0 = [&](int i) { return ((t_lo + i) % tiles_c) * kColsT; };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kOpStages; ++s) {
            mbar_init(op_full + s, 1);
            mbar_init(op_empty + s, 1);  // the tile's UMMAs
        }
        for (int s = 0; s < kCodeStages; ++s) {
            mbar_init(code_full + s, 1);
            mbar_init(code_empty + s, kEpiWarps);  // one arrive per epilogue warp
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(acc_full + b, 1);
            mbar_init(acc_empty + b, kEpiWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (threadIdx.x == 0) {
#pragma unroll
        for (int k = 0; k < 16; ++k) levels[k] = tab.level[k];  // constant indices: the table stays in parameter space
    }
    if (warp == kWarpMma) {
        tmem_alloc(tmem_slot, kTmemColsM);
        tmem_relinquish();
    }
    if (warp == kWarpProd && lane == 0) {
        tma_prefetch_desc(&tm_b);
        tma_prefetch_desc(&tm_a);
        tma_prefetch_desc(&tm_codes);
        tma_prefetch_desc(&tm_out);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == kWarpProd) {
        // ----------------------------------------------------- producer --
        if (lane == 0) {
            int last_op = -1, last_code = -1;  // the last tiles whose copies were issued
            for (int i = 0; i < n_my; ++i) {
                const int64_t n0 = tile_n0(i), k0 = tile_k0(i);
                const int so = i % kOpStages, sc = i % kCodeStages;
                if (i >= kOpStages &&
                    !mbar_wait(op_empty + so, static_cast<uint32_t>(i / kOpStages - 1) & 1u, tmo, a.status)) {
                    *abort_flag = 1;
                    break;
                }
                if (*abort_flag) break;
                uint8_t* op = smem + so * kOpStage;
                mbar_arrive_expect_tx(op_full + so, kOpStage);
                tma_load_2d(op, &tm_b, op_full + so, 0, static_cast<int>(n0));
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    tma_load_2d(op + kOpB + c * 8192, &tm_a, op_full + so, static_cast<int>(k0) + 64 * c, 0);
                last_op = i;
                if (i >= kCodeStages &&
                    !mbar_wait(code_empty + sc, static_cast<uint32_t>(i / kCodeStages - 1) & 1u, tmo, a.status)) {
                    *abort_flag = 1;
                    break;
                }
                mbar_arrive_expect_tx(code_full + sc, kCodeStage);
                tma_load_2d(smem + kOffCodes + sc * kCodeStage, &tm_codes, code_full + sc, static_cast<int>(k0 / 2),
                            static_cast<int>(n0));
                last_code = i;
            }
            // every copy in flight lands before the CTA's shared memory is released
            for (int i = max(0, last_op - kOpStages + 1); i <= last_op; ++i)
                mbar_wait(op_full + i % kOpStages, static_cast<uint32_t>(i / kOpStages) & 1u, tmo, nullptr);
            for (int i = max(0, last_code - kCodeStages + 1); i <= last_code; ++i)
                mbar_wait(code_full + i % kCodeStages, static_cast<uint32_t>(i / kCodeStages) & 1u, tmo, nullptr);
        }
        __syncwarp();
    } else if (warp == kWarpMma) {
        // ---------------------------------------------------------- MMA --
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(kRowsT, kColsT, false, true);
            int last = -1;  // the last tile whose UMMAs were committed
            tc_fence_after();
            for (int i = 0; i < n_my; ++i) {
                const int so = i % kOpStages, b = i & 1;
                if (!mbar_wait(op_full + so, static_cast<uint32_t>(i / kOpStages) & 1u, tmo, a.status) ||
                    (i >= 2 && !mbar_wait(acc_empty + b, static_cast<uint32_t>(i / 2 - 1) & 1u, tmo, a.status))) {
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t ob = smem_u32(smem + so * kOpStage), oa = ob + kOpB;
                for (int kk = 0; kk < ksteps; ++kk)
                    umma_f16(tmem + b * kColsT, sw128_desc(ob + kk * 32, 16, 1024), sw128_desc(oa + kk * 2048, 8192, 1024),
                             idesc, kk > 0 ? 1u : 0u);
                umma_commit(op_empty + so);
                umma_commit(acc_full + b);
                last = i;
            }
            // the commit of the last tile arrives once every UMMA of this CTA
            // has completed: wait for it (bounded) before TMEM may be freed
            if (last >= 0) mbar_wait(acc_full + (last & 1), static_cast<uint32_t>(last / 2) & 1u, tmo, nullptr);
        }
        __syncwarp();
    } else {
        // ----------------------------------------------------- epilogue --
        const int q = warp & 3, h = warp >> 2;
        const int row_l = q * 32 + lane;
        const uint32_t outbuf = smem_u32(smem + kOffScratch) + warp * 2 * kStageOut;
        int nstore = 0;  // this warp's output stores so far: buffer nstore & 1
        const uint32_t swz = static_cast<uint32_t>(row_l & 7);
        const float mu = a.c.absmax ? 0.0f : __ldg(a.c.mean);
        for (int i = 0; i < n_my; ++i) {
            const int64_t n0 = tile_n0(i), k0 = tile_k0(i);
            const int b = i & 1, sc = i % kCodeStages;
            const int64_t n = n0 + row_l;
            // the row's two block constants of this half (loads before the waits)
            // the row's block constants of this warp's columns (loads before the waits)
            constexpr int kBlocksW = kEpiCols / kBlock;
            float cp[kBlocksW];
#pragma unroll
            for (int j = 0; j < kBlocksW; ++j) {
                const int64_t kb = (k0 + h * kEpiCols) / kBlock + j;
                const int64_t bk = n < N && kb < KB ? n * KB + kb : 0;
                cp[j] = a.c.absmax ? __ldg(a.c.absmax + bk)
                                   : __fmaf_rn(e4m3_to_f32(__ldg(a.c.qabsmax + bk)), __ldg(a.c.s2 + (bk >> 8)), mu);
            }
            const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(acc_full + b, static_cast<uint32_t>(i / 2) & 1u, tmo,
                                                              a.status)) &&
                            __all_sync(0xFFFFFFFFu, mbar_wait(code_full + sc, static_cast<uint32_t>(i / kCodeStages) & 1u,
                                                              tmo, a.status));
            if (!ok || *abort_flag) {
                *abort_flag = 1;
                break;
            }
            tc_fence_after();
            const uint32_t crow = smem_u32(smem + kOffCodes + sc * kCodeStage) + static_cast<uint32_t>(row_l) * 128u;
            const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16) + b * kColsT + h * kEpiCols;
            // one 64-column block at a time: 32 rows x 128 bytes into an output
            // buffer in the 128-byte swizzled layout, then one TMA store
#pragma unroll
            for (int jb = 0; jb < kBlocksW; ++jb) {
                const Nf4BlockLut lut = make_block_lut(levels, cp[jb]);
                const uint32_t buf = outbuf + (nstore & 1) * kStageOut;
                if (lane == 0) bulk_wait_read<1>();  // the store that last used this buffer has read it
                __syncwarp();
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t r[32];
                    tmem_ld32(trow + 64 * jb + 32 * half, r);
                    // 32 columns = one 16-byte chunk of the row's codes
                    const uint32_t chunk = static_cast<uint32_t>((h * kEpiCols + 64 * jb + 32 * half) / 32);
                    const uint4 cw = lds128(crow + ((chunk ^ swz) << 4));
                    const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t wh[4], o[4];
                        lut_decode8(lut, words[j], wh);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float lo =
                                __fmaf_rn(a.scale, __uint_as_float(r[8 * j + 2 * e]), __uint_as_float(wh[e] << 16));
                            const float hi = __fmaf_rn(a.scale, __uint_as_float(r[8 * j + 2 * e + 1]),
                                                       __uint_as_float(wh[e] & 0xFFFF0000u));
                            o[e] = pack_bf16x2(lo, hi);
                        }
                        const uint32_t c16 = static_cast<uint32_t>(4 * half + j);  // 16-byte chunk of the 128-byte row
                        sts128(buf + lane * 128u + ((c16 ^ static_cast<uint32_t>(lane & 7)) << 4), o);
                    }
                }
                fence_proxy_async_smem();  // the buffer, visible to the TMA store
                __syncwarp();
                if (lane == 0) {
                    const int64_t x = k0 + h * kEpiCols + 64 * jb, y = n0 + 32 * q;
                    if (x < K && y < N) tma_store_2d(&tm_out, smem + (buf - smem_u32(smem)), static_cast<int>(x),
                                                     static_cast<int>(y));
                    bulk_commit();
                }
                ++nstore;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(acc_empty + b);
                mbar_arrive(code_empty + sc);
            }
        }
        if (lane == 0) bulk_wait<0>();  // this warp's stores are complete before the CTA exits
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemColsM);
    }
}

}  // namespace

size_t merge_tc_smem_bytes() { return kSmemM; }

cudaError_t launch_merge_tc(const CUtensorMap& b_map, const CUtensorMap& a_map, const CUtensorMap& codes_map,
                            const CUtensorMap& out_map, const MergeArgs& a, int r, const Nf4Tables& tab, int num_sms,
                            cudaStream_t st) {
    if (a.N < 1 || a.K < kBlock || a.K % kBlock != 0 || r < 8 || r > 64 || r % 8 != 0) return cudaErrorInvalidValue;
    const int64_t tiles = (a.N + kRowsT - 1) / kRowsT * ((a.K + kColsT - 1) / kColsT);
    const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
    merge_tc_kernel<<<grid, kThreadsM, kSmemM, st>>>(b_map, a_map, codes_map, out_map, a, (r + 15) / 16, tab);
    return cudaGetLastError();
}

cudaError_t merge_tc_init_device() {
    return cudaFuncSetAttribute(merge_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(kSmemM));
}

}  // namespace qlora
