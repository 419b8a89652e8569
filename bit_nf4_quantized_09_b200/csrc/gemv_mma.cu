// Small-batch forward for up to 32 tokens: Y = X . deq(W)^T + sT . B^T.
//
// With a few tokens every weight is used a few times only, so the step is
// bound by streaming the packed weight (about half a byte per weight) and by
// decoding it; "ta-paperlens QLoRA explainer", 落とし穴, names this
// small-batch regime as the one where 4-bit weights pay off.
//
// Design: no shared-memory staging of the weight at all. Each warp owns 16
// weight rows and walks K in steps of four NF4 blocks (256 weights per row).
// Lane (g, q) loads the 32 packed bytes of block q of rows g and g + 8 with
// 16-byte global loads one step ahead, builds the two per-block bf16 lookup
// tables, decodes straight into the A fragments of mma.m16n8k16 (weight rows
// = MMA rows) and multiplies them with X fragments read from shared memory
// (tokens = MMA columns, n8 tiles). The reduction index inside an MMA is
// permuted: lane q's slots 2q, 2q + 1, 2q + 8, 2q + 9 of MMA step s hold
// weights 4s .. 4s + 3 of its block, and the X fragment uses the same order,
// so no data is moved between lanes.
//
// CTA = 8 warps = 128 weight rows. The (row tile, block column) units are
// dealt out in equal contiguous ranges, one per CTA slot (stream-K), so no
// wave is left part-empty; a range may cross into the next row tile. Every
// CTA that touches a tile writes its fp32 partial sums for it; the last one
// to finish (atomic ticket) adds them in CTA order, adds the rank-r term and
// writes Y in bf16. The rank-r input sT comes from the preceding launch;
// the kernel may be launched as its programmatic dependent and waits for it
// (griddepcontrol.wait) only before the epilogue, so the weight stream
// overlaps the down-projection.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace qlora {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kRowsCta = kWarps * 16;
constexpr uint32_t kChunk = 144;  // bytes per 64 X elements in shared memory (128 + 16 pad)

// Row pitch of the staged X slice: 144-byte chunks and a pitch congruent to
// 64 mod 128 bytes, so the 16-byte fragment reads of a quarter warp (2 token
// rows x 4 lanes q) fall on 8 distinct groups of 4 banks.
__host__ __device__ constexpr uint32_t x_pitch(int chunks) {
    const uint32_t raw = static_cast<uint32_t>(chunks) * kChunk;
    return (raw + 63u) / 128u * 128u + 64u;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ void sts64(uint32_t addr, uint32_t a, uint32_t b) {
    asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// sum_{j < cols} sT[j] * B[j] over bf16 operands, fp32 products and sums in
// order (cols a multiple of 8, both rows 16-byte aligned); the loads of each
// 32 columns are issued before their first product.
__device__ __forceinline__ float rank_dot(const uint16_t* sT, const uint16_t* b, int cols) {
    float acc = 0.0f;
    for (int c0 = 0; c0 < cols; c0 += 32) {
        uint4 tv[4], bv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const bool in = c0 + 8 * i < cols;
            tv[i] = in ? __ldg(reinterpret_cast<const uint4*>(sT + c0) + i) : make_uint4(0u, 0u, 0u, 0u);
            bv[i] = in ? __ldg(reinterpret_cast<const uint4*>(b + c0) + i) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (c0 + 8 * i >= cols) break;
            const uint32_t tw[4] = {tv[i].x, tv[i].y, tv[i].z, tv[i].w};
            const uint32_t bw[4] = {bv[i].x, bv[i].y, bv[i].z, bv[i].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                acc = __fmaf_rn(__uint_as_float(tw[j] << 16), __uint_as_float(bw[j] << 16), acc);
                acc = __fmaf_rn(__uint_as_float(tw[j] & 0xFFFF0000u), __uint_as_float(bw[j] & 0xFFFF0000u), acc);
            }
        }
    }
    return acc;
}

// Column of sT holding the rank-r input of output row n.
__device__ __forceinline__ int rank_col(const GemvMmaArgs& a, int64_t n) {
    for (int g = 0; g < a.ngroups - 1; ++g)
        if (n < a.group_end[g]) return a.group_rank_x[g];
    return a.group_rank_x[a.ngroups - 1];
}

// The weight stream goes through a per-lane ring of kStages step slots in
// shared memory, filled by cp.async kStages - 1 steps ahead. A slot holds one
// step's inputs for lane (g, q): the 32 packed bytes of rows g and g + 8, the
// aligned words holding their E4M3 constants, and their second-level scales.
// Only the lane that copies a slot reads it, so a per-thread wait_group is
// the only synchronisation. 80-byte slots keep the 16-byte reads of eight
// consecutive lanes on distinct banks.
constexpr uint32_t kSlot = 80;

// Per instantiation (MT n8 token tiles): ring depth and CTAs per SM. One
// token tile runs three CTAs per SM with a two-step ring; wider ones two
// CTAs with a three-step ring (their staged X slice is larger).
template <int MT>
struct Cfg {
    static constexpr int kStages = MT == 1 ? 2 : 3;
    static constexpr int kCtasPerSm = MT == 1 ? 3 : 2;
    static constexpr uint32_t kRing = kStages * kSlot * kThreads;  // bytes per CTA
};

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

template <int MT, bool kNoDq>
__global__ void __launch_bounds__(kThreads, Cfg<MT>::kCtasPerSm)
    gemv_mma_kernel(const GemvMmaArgs a, const Nf4Tables tab) {
    constexpr int kStages = Cfg<MT>::kStages;
    constexpr uint32_t kRing = Cfg<MT>::kRing;
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ int last_of[2];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int M = static_cast<int>(a.M);
    const int N = static_cast<int>(a.N), KB = static_cast<int>(a.K / kBlock);
    const int64_t K = a.K;
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
    const int it0 = (len0 + 3) / 4, it_all = it0 + (len1 + 3) / 4;
    const uint32_t PX = x_pitch(a.max_chunks);
    const uint32_t ring = smem_u32(smem) + threadIdx.x * kSlot;  // this lane's slot 0
    const uint32_t xs = smem_u32(smem) + kRing;

    // This lane's rows and first block column in each segment: unit indices
    // (row * KB + column) of rows g and g + 8, the last column offset, and the
    // bit offsets of the E4M3 constants in their aligned words (the same for
    // every step of a segment, since steps advance by 4 columns). A lane past
    // its segment's end or past N copies a valid neighbour (clamped row and
    // column) instead: its X chunk is zero or its output row is dropped, so
    // nothing it decodes reaches Y (decoded weights are always finite).
    struct LaneSeg {
        int64_t ia, ib;
        int kmax;
        uint32_t sh;  // byte offset of row g's constant * 8 | (row g + 8's) << 8
    };
    auto lane_seg = [&](int j) {
        const int r0 = (t0 + j) * kRowsCta + warp * 16 + g;
        LaneSeg ls;
        const int blo = j ? 0 : blo0;
        ls.ia = static_cast<int64_t>(min(r0, N - 1)) * KB + blo;
        ls.ib = static_cast<int64_t>(min(r0 + 8, N - 1)) * KB + blo;
        ls.kmax = (j ? len1 : len0) - 1;
        ls.sh = static_cast<uint32_t>((ls.ia + q) & 3) * 8 | static_cast<uint32_t>((ls.ib + q) & 3) * 8 << 8;
        return ls;
    };
    const LaneSeg seg0 = lane_seg(0), seg1 = lane_seg(1);

    // copies of step gi into slot gi % kStages
    auto issue = [&](int gi) {
        if (gi < it_all) {
            const bool s1 = gi >= it0;
            const int off = min(4 * (gi - (s1 ? it0 : 0)) + q, s1 ? seg1.kmax : seg0.kmax);
            const int64_t ia = (s1 ? seg1.ia : seg0.ia) + off, ib = (s1 ? seg1.ib : seg0.ib) + off;
            const uint32_t d = ring + (gi % kStages) * (kSlot * kThreads);
            cp_async16(d, a.codes + ia * 32);
            cp_async16(d + 16, a.codes + ia * 32 + 16);
            cp_async16(d + 32, a.codes + ib * 32);
            cp_async16(d + 48, a.codes + ib * 32 + 16);
            if (kNoDq) {  // the two fp32 constants
                cp_async4(d + 64, a.absmax + ia);
                cp_async4(d + 68, a.absmax + ib);
            } else {
                cp_async4(d + 64, a.qabsmax + (ia & ~int64_t(3)));
                cp_async4(d + 68, a.qabsmax + (ib & ~int64_t(3)));
                cp_async4(d + 72, a.s2 + (ia >> 8));
                cp_async4(d + 76, a.s2 + (ib >> 8));
            }
        }
        cp_async_commit();  // possibly empty: keeps one group per step
    };
    // ---- stage X (its loads go out ahead of the weight stream's): step i's
    // four 64-column chunks at chunk 4i .. 4i + 3, zeros for columns past a
    // segment's end
    for (int i = threadIdx.x; i < M * it_all * 32; i += kThreads) {
        const int cc = i & 7, ch = (i >> 3) % (4 * it_all), m = (i >> 3) / (4 * it_all);
        const int seg = ch >= 4 * it0;
        const int lb = ch - (seg ? 4 * it0 : 0);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (lb < (seg ? len1 : len0))
            v = __ldg(reinterpret_cast<const uint4*>(a.X + m * K + ((seg ? 0 : blo0) + lb) * kBlock) + cc);
        const uint32_t at = xs + m * PX + ch * kChunk + cc * 16;
        sts64(at, v.x, v.y);
        sts64(at + 8, v.z, v.w);
    }


#pragma unroll
    for (int i = 0; i < kStages - 1; ++i) issue(i);

    const float mean = kNoDq ? 0.0f : __ldg(a.mean);
    float acc[MT][4];
#pragma unroll
    for (int t = 0; t < MT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.0f;
    // X fragment rows: token g + 8t, clamped to the last token (the MMA
    // columns past M then hold copies whose sums are never written)
    uint32_t xtok[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) xtok[t] = kRing + min(g + 8 * t, M - 1) * PX + q * kChunk;
    __syncthreads();  // X staged

#pragma unroll 1
    for (int gi = 0; gi < it_all; ++gi) {
        issue(gi + kStages - 1);
        cp_async_wait<kStages - 1>();  // this lane's copies of step gi have landed
        const uint32_t d = ring + (gi % kStages) * (kSlot * kThreads);
        const uint4 a0 = lds128(d), a1 = lds128(d + 16), b0 = lds128(d + 32), b1 = lds128(d + 48);
        const uint4 cq = lds128(d + 64);  // q words A, B; s2 A, B (kNoDq: constants A, B)
        const uint32_t sh = gi >= it0 ? seg1.sh : seg0.sh;
        const float cpa = kNoDq ? __uint_as_float(cq.x)
                                : __fmaf_rn(e4m3_to_f32(cq.x >> (sh & 31u)), __uint_as_float(cq.z), mean);
        const float cpb = kNoDq ? __uint_as_float(cq.y)
                                : __fmaf_rn(e4m3_to_f32(cq.y >> (sh >> 8)), __uint_as_float(cq.w), mean);
        const Nf4BlockLut la = make_block_lut(tab.level, cpa);
        const Nf4BlockLut lb = make_block_lut(tab.level, cpb);
        const uint32_t wa[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const uint32_t wb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
        const uint8_t* xstep = smem + 4 * gi * kChunk;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            uint32_t oa[4], ob[4];
            lut_decode8_sx(la, wa[w], oa);
            lut_decode8_sx(lb, wb[w], ob);
            // X fragments of MMA steps 2w and 2w + 1: 16 contiguous bytes
            uint4 bx[MT];
#pragma unroll
            for (int t = 0; t < MT; ++t) bx[t] = *reinterpret_cast<const uint4*>(xstep + xtok[t] + 16 * w);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t af[4] = {oa[2 * h], ob[2 * h], oa[2 * h + 1], ob[2 * h + 1]};
#pragma unroll
                for (int t = 0; t < MT; ++t) mma_bf16(acc[t], af, h ? bx[t].z : bx[t].x, h ? bx[t].w : bx[t].y);
            }
        }
        if (gi == it0 - 1 || gi == it_all - 1) {
            // segment done: its partial sums, c0, c1 = (row g, tokens 2q,
            // 2q + 1) and c2, c3 = (row g + 8, the same tokens)
            const int tile = t0 + (gi >= it0);
            const int sl = sc.slot(tile, c);
            const int rowA = tile * kRowsCta + warp * 16 + g, rowB = rowA + 8;
#pragma unroll
            for (int t = 0; t < MT; ++t) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int tok = 8 * t + 2 * q + e;
                    if (tok < M) {
                        float* pt = a.part + (static_cast<int64_t>(sl) * M + tok) * N;
                        if (rowA < N) pt[rowA] = acc[t][e];
                        if (rowB < N) pt[rowB] = acc[t][2 + e];
                    }
                }
                acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.0f;
            }
        }
    }
    cp_async_wait<0>();

    // ---- tickets: the last CTA to finish a row tile reduces it
    const int nseg = len1 > 0 ? 2 : 1;
    __threadfence();  // publish this CTA's partials before taking tickets
    __syncthreads();
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
        griddep_wait();   // sT from the preceding launch
        const int tile = t0 + j;
        const int n0 = tile * kRowsCta;
        const int np = sc.parts(tile);
        for (int i = threadIdx.x; i < M * kRowsCta; i += kThreads) {
            const int m = i / kRowsCta, n = n0 + i % kRowsCta;
            if (n >= N) continue;
            // every load of this output goes out before the first use: the
            // rank-r operands, then the partials in CTA order, 16 at a time
            const float lr = rank_dot(a.sT + static_cast<int64_t>(m) * a.sT_ld + rank_col(a, n),
                                      a.B + static_cast<int64_t>(n) * a.B_ld, a.rank_cols);
            float s = 0.0f;
            for (int s0 = 0; s0 < np; s0 += 16) {
                float v[16];
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    v[u] = s0 + u < np ? __ldcg(a.part + (static_cast<int64_t>(s0 + u) * M + m) * N + n) : 0.0f;
#pragma unroll
                for (int u = 0; u < 16; ++u) s += v[u];
            }
            a.Y[static_cast<int64_t>(m) * N + n] = static_cast<uint16_t>(pack_bf16x2(s + lr, 0.0f) & 0xFFFFu);
        }
        if (threadIdx.x == 0) a.counter[tile] = 0;  // ready for the next call
    }
}

template <int MT, bool kNoDq>
cudaError_t launch_mt(const GemvMmaArgs& a, const Nf4Tables& tab, size_t smem, bool pdl, cudaStream_t st) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(a.ctas));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, gemv_mma_kernel<MT, kNoDq>, a, tab);
}

constexpr int kMaxMt = 4;

// n8 token tiles of the instantiation that serves M tokens (1, 2 or 4)
int token_tiles(int64_t M) { return M <= 8 ? 1 : (M <= 16 ? 2 : kMaxMt); }

}  // namespace

size_t gemv_mma_smem_bytes(int64_t M, int max_chunks) {
    const uint32_t ring = token_tiles(M) == 1 ? Cfg<1>::kRing : Cfg<2>::kRing;
    return ring + static_cast<size_t>(M) * x_pitch(max_chunks);
}

GemvMmaPlan gemv_mma_plan(int64_t M, int64_t N, int64_t K, int num_sms) {
    const int64_t KB = K / kBlock, tiles = (N + kRowsCta - 1) / kRowsCta, U = tiles * KB;
    const bool one = token_tiles(M) == 1;
    const int per_sm = one ? Cfg<1>::kCtasPerSm : Cfg<2>::kCtasPerSm;
    // staged X per CTA: what the SM's 227 KB leave beside the rings
    const size_t budget = (227 * 1024) / per_sm - 1024 - (one ? Cfg<1>::kRing : Cfg<2>::kRing);
    const int64_t slots = static_cast<int64_t>(per_sm) * std::max(num_sms, 1);
    // whole waves of CTA slots, at least one CTA per row tile (so a range
    // touches at most two tiles), at most one CTA per unit
    int64_t P = std::min(U, (tiles + slots - 1) / slots * slots);
    // staged X chunks: the range's blocks plus up to 3 pad blocks per segment
    auto chunks = [&](int64_t p) { return ((U + p - 1) / p + 6 + 3) / 4 * 4; };
    while (P < U && static_cast<size_t>(M) * x_pitch(static_cast<int>(chunks(P))) > budget) P = std::min(U, P + slots);
    GemvMmaPlan plan;
    plan.ctas = static_cast<int>(P);
    plan.units = U;
    plan.max_chunks = static_cast<int>(chunks(P));
    plan.max_parts = static_cast<int>((KB + U / P - 1) / (U / P) + 1);
    return plan;
}

namespace {
template <bool kNoDq>
cudaError_t gemv_mma_opt_in(int smax) {
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(gemv_mma_kernel<1, kNoDq>, cudaFuncAttributeMaxDynamicSharedMemorySize, smax)) !=
        cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(gemv_mma_kernel<2, kNoDq>, cudaFuncAttributeMaxDynamicSharedMemorySize, smax)) !=
        cudaSuccess)
        return e;
    return cudaFuncSetAttribute(gemv_mma_kernel<4, kNoDq>, cudaFuncAttributeMaxDynamicSharedMemorySize, smax);
}
}  // namespace

cudaError_t gemv_mma_init_device() {
    const int smax = 220 * 1024;  // above any plan (the plan keeps two or three CTAs per SM)
    const cudaError_t e = gemv_mma_opt_in<false>(smax);
    return e != cudaSuccess ? e : gemv_mma_opt_in<true>(smax);
}

cudaError_t launch_gemv_mma(const GemvMmaArgs& a, const Nf4Tables& tab, bool pdl, cudaStream_t st) {
    if (a.M < 1 || a.M > kGemvMmaMaxM || a.ctas < 1) return cudaErrorInvalidValue;
    const size_t smem = gemv_mma_smem_bytes(a.M, a.max_chunks);
    const int mt = token_tiles(a.M);
    static_assert(kMaxMt * 8 == kGemvMmaMaxM, "token tiles");
    if (a.absmax) {
        if (mt == 1) return launch_mt<1, true>(a, tab, smem, pdl, st);
        if (mt == 2) return launch_mt<2, true>(a, tab, smem, pdl, st);
        return launch_mt<4, true>(a, tab, smem, pdl, st);
    }
    if (mt == 1) return launch_mt<1, false>(a, tab, smem, pdl, st);
    if (mt == 2) return launch_mt<2, false>(a, tab, smem, pdl, st);
    return launch_mt<4, false>(a, tab, smem, pdl, st);
}

}  // namespace qlora
