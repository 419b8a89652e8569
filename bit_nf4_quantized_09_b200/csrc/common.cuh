// Device-side building blocks shared by the kernels of libqlora_nf4.so:
// NF4 tables, the per-block dequantisation lookup, and thin inline-PTX
// wrappers for mbarriers, TMA, and the sm_100 tensor core (tcgen05/TMEM).
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace qlora {

constexpr int kBlock = 64;    // weights per first-level absmax block
constexpr int kGroup = 256;   // first-level constants per second-level group

// Device status bits written by pipelined kernels when a bounded wait runs out.
constexpr int kStatusTimeout = 1;

// The NF4 levels and the 15 decision thresholds between neighbours, passed to
// kernels by value (they live in the kernel-parameter constant bank).
struct Nf4Tables {
    float level[16];
    float thresh[15];
    float pad_;
};

// ---------------------------------------------------------------------------
// Small helpers
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// E4M3 byte -> fp32 (exact: every E4M3 value is an fp16 value).
__device__ __forceinline__ float e4m3_to_f32(uint32_t q) {
    uint32_t h2;
    uint16_t in = static_cast<uint16_t>(q & 0xFFu);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

// Two fp32 -> two E4M3 bytes, round-to-nearest-even, saturating to +-448.
// Result: byte 0 = e4m3(lo), byte 1 = e4m3(hi).
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// ---------------------------------------------------------------------------
// NF4 dequantisation of one 64-weight block through a per-block lookup table.
//
// The restored value depends only on (code, block): w_hat = bf16(level[code]
// * c'). So each block builds its 16 bf16 entries once (16 fp32 multiplies,
// 8 paired conversions) and splits them into a low-byte table and a high-byte
// table, 16 bytes each (4 registers each). A 4-bit code then indexes them
// with byte permutes: its low 3 bits pick one of 8 bytes from a register pair
// and its top bit picks which pair.
// ---------------------------------------------------------------------------

struct Nf4BlockLut {
    uint32_t lo[4];   // low bytes of entries 0..15, 4 per register
    uint32_t hi[4];   // high bytes
};

__device__ __forceinline__ Nf4BlockLut make_block_lut(const float (&level)[16], float cprime) {
    Nf4BlockLut t;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t p0 = pack_bf16x2(__fmul_rn(level[4 * j + 0], cprime), __fmul_rn(level[4 * j + 1], cprime));
        uint32_t p1 = pack_bf16x2(__fmul_rn(level[4 * j + 2], cprime), __fmul_rn(level[4 * j + 3], cprime));
        // p0 bytes: [lo(4j), hi(4j), lo(4j+1), hi(4j+1)], p1 likewise for 4j+2, 4j+3
        t.lo[j] = __byte_perm(p0, p1, 0x6420);
        t.hi[j] = __byte_perm(p0, p1, 0x7531);
    }
    return t;
}

// Eight codes packed in one little-endian word (byte b holds element 2b in its
// high nibble and element 2b+1 in its low nibble) -> eight bf16 in code order,
// as four bf16x2 words (out[i] = elements 2i, 2i+1 with 2i in the low half).
__device__ __forceinline__ void lut_decode8(const Nf4BlockLut& t, uint32_t packed, uint32_t (&out)[4]) {
    const uint32_t idx = packed & 0x77777777u;         // low 3 bits of every code
    const uint32_t top = (packed >> 3) & 0x11111111u;  // top bit of every code
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t sel = h ? (idx >> 16) : idx;
        const uint32_t msel = h ? (top >> 16) : top;
        // per output byte: 0xFF where the code's top bit is set
        const uint32_t m = __byte_perm(0x0000FF00u, 0u, msel);
        const uint32_t loA = __byte_perm(t.lo[0], t.lo[1], sel);
        const uint32_t loB = __byte_perm(t.lo[2], t.lo[3], sel);
        const uint32_t hiA = __byte_perm(t.hi[0], t.hi[1], sel);
        const uint32_t hiB = __byte_perm(t.hi[2], t.hi[3], sel);
        const uint32_t lo = (loA & ~m) | (loB & m);   // bytes ordered [e1, e0, e3, e2]
        const uint32_t hi = (hiA & ~m) | (hiB & m);
        out[2 * h + 0] = __byte_perm(lo, hi, 0x4051);  // e0 | e1 << 16
        out[2 * h + 1] = __byte_perm(lo, hi, 0x6273);  // e2 | e3 << 16
    }
}

// D += A . B on the legacy tensor path, mma.m16n8k16 with bf16 operands and
// fp32 accumulation. Lane (g, q) = (lane / 4, lane % 4) holds
//   a[0] = A(g, 2q..2q+1), a[1] = A(g+8, 2q..2q+1), a[2] = A(g, 2q+8..2q+9),
//   a[3] = A(g+8, 2q+8..2q+9); b0 = B(2q..2q+1, g), b1 = B(2q+8..2q+9, g);
//   d[0..1] = D(g, 2q..2q+1), d[2..3] = D(g+8, 2q..2q+1)
// (the lower index in the low half of each 32-bit register).
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// prmt.b32 in its default mode: a selector nibble with bit 3 set yields the
// sign bit of the byte it picks, replicated over the whole output byte.
__device__ __forceinline__ uint32_t prmt_sx(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// lut_decode8 with the byte masks taken straight from the packed word: the
// top bit of a high-nibble code is bit 7 of its byte, and that of a
// low-nibble code is bit 7 of the same byte shifted left by 4, so one
// sign-replicating permute yields the four 0x00/0xFF masks of a half.
__device__ __forceinline__ void lut_decode8_sx(const Nf4BlockLut& t, uint32_t packed, uint32_t (&out)[4]) {
    const uint32_t idx = packed & 0x77777777u;
    const uint32_t p4 = packed << 4;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t sel = h ? (idx >> 16) : idx;
        // output bytes [e1, e0, e3, e2] (h = 0) or [e5, e4, e7, e6] (h = 1)
        const uint32_t m = prmt_sx(p4, packed, h ? 0xFBEAu : 0xD9C8u);
        const uint32_t loA = __byte_perm(t.lo[0], t.lo[1], sel);
        const uint32_t loB = __byte_perm(t.lo[2], t.lo[3], sel);
        const uint32_t hiA = __byte_perm(t.hi[0], t.hi[1], sel);
        const uint32_t hiB = __byte_perm(t.hi[2], t.hi[3], sel);
        const uint32_t lo = (loA & ~m) | (loB & m);
        const uint32_t hi = (hiA & ~m) | (hiB & m);
        out[2 * h + 0] = __byte_perm(lo, hi, 0x4051);
        out[2 * h + 1] = __byte_perm(lo, hi, 0x6273);
    }
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Announce `bytes` of asynchronous copies for the current phase without
// arriving (the phase still needs its arrivals).
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity to complete. Returns false
// (and records kStatusTimeout in *status) if it has not completed within
// timeout_ns; the caller then abandons its remaining work.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns, int* status) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(a, parity)) return true;
        if (global_timer_ns() - t0 > timeout_ns) {
            if (status) atomicOr(status, kStatusTimeout);
            return false;
        }
    }
}

// mbar_wait for a waiter that can take a little latency (a producer a few
// stages ahead of its consumers): between polls the warp sleeps, 32 ns at
// first, doubling up to 512 ns, so that it takes no issue slots from the
// warps that compute. Bounded the same way.
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity, uint64_t timeout_ns, int* status) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    uint32_t ns = 32;
    while (!mbar_try_wait(a, parity)) {
        if (global_timer_ns() - t0 > timeout_ns) {
            if (status) atomicOr(status, kStatusTimeout);
            return false;
        }
        __nanosleep(ns);
        ns = ns < 512 ? 2 * ns : 512;
    }
    return true;
}

// ---------------------------------------------------------------------------
// Thread-block clusters (two CTAs of one GPU sharing shared memory)
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// The shared::cluster address of the same shared-memory location in CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t local, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
    return r;
}

__device__ __forceinline__ void st_cluster128(uint32_t addr, const uint32_t (&v)[4]) {
    asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v[0]), "r"(v[1]), "r"(v[2]),
                 "r"(v[3])
                 : "memory");
}

// Arrive on an mbarrier of another CTA of the cluster (address from mapa),
// releasing this thread's earlier writes at cluster scope.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// mbar_wait for a barrier that other CTAs of the cluster arrive on: acquire
// at cluster scope. Bounded the same way.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, uint64_t timeout_ns, int* status) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait_cluster(a, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait_cluster(a, parity)) return true;
        if (global_timer_ns() - t0 > timeout_ns) {
            if (status) atomicOr(status, kStatusTimeout);
            return false;
        }
    }
}

// Bulk copy of `bytes` from this CTA's shared memory to another CTA's of the
// cluster (dst and the destination's mbarrier as mapa addresses), completing
// as transaction bytes on that mbarrier.
__device__ __forceinline__ void bulk_copy_to_cluster(uint32_t dst_cluster, uint32_t src, uint32_t bytes,
                                                     uint32_t mbar_cluster) {
    asm volatile(
        "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst_cluster),
        "r"(src), "r"(bytes), "r"(mbar_cluster)
        : "memory");
}

// 16-byte shared-memory load and store (shared-window addresses).
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ void sts128(uint32_t addr, const uint32_t (&v)[4]) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3])
                 : "memory");
}

// 16-byte load from shared memory of any CTA of the cluster (mapa address).
__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Generic-proxy writes to shared memory of any CTA of the cluster -> visible
// to the async proxy (the tensor core reading them as an operand).
__device__ __forceinline__ void fence_proxy_async_cluster() {
    asm volatile("fence.proxy.async.shared::cluster;" ::: "memory");
}

// ---------------------------------------------------------------------------
// TMA (tiled bulk tensor copies, global -> shared, no multicast)
// ---------------------------------------------------------------------------

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// Shared -> global tiled bulk store (TMA), tracked by bulk groups.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(smem_u32(src)), "r"(x), "r"(y)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until at most N committed bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

template <int N>
__device__ __forceinline__ void bulk_wait() {
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: TMEM allocation, UMMA (kind::f16 with bf16 operands, fp32 accum)
// ---------------------------------------------------------------------------

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {  // whole warp
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {  // whole warp
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {  // whole warp
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, one instruction, issued by one thread.
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on an mbarrier once all previously issued tcgen05.mma of this thread
// have completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// umma_commit arriving on the mbarrier at the same offset in every CTA of the
// cluster named by cta_mask.
__device__ __forceinline__ void umma_commit_multicast(uint64_t* bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(cta_mask)
        : "memory");
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 accumulator, dense.
//   bits 4-5 D format (1 = f32), 7-9 A format (1 = bf16), 10-12 B format,
//   15 A major (1 = MN), 16 B major, 17-22 N >> 3, 24-28 M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
           (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand.
//   bits 0-13 start address >> 4, 16-29 leading byte offset >> 4,
//   32-45 stride byte offset >> 4, 46-47 version (1 on sm_100),
//   49-51 base offset (0: atoms 1024-byte aligned), 61-63 layout (2 = SW128).
// K-major: rows of 128 B, 8-row atoms SBO apart (LBO unused).
// MN-major: 64-element (128 B) runs along M/N, LBO between runs, 8 K-rows per
// atom, SBO between 8-row K groups.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    d |= static_cast<uint64_t>(2u) << 61;
    return d;
}

// 32 lanes x 32 consecutive fp32 columns of TMEM into 32 registers per thread.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

// 32 lanes x 16 consecutive fp32 columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ bool elect_lane0() { return (threadIdx.x & 31u) == 0u; }

}  // namespace qlora
