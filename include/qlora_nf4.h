/*
 * qlora_nf4.h - C ABI of libqlora_nf4.so, the frozen-NF4 QLoRA linear layer
 * on one NVIDIA B200 (sm_100a).
 *
 * What is computed (sources: the pages on QLoRA):
 *   - "ta-paperlens QLoRA explainer" (QLoRA - 650億パラメータのモデルをGPU 1枚で
 *     微調整する), sections 量子化を1段落で (blockwise absmax over 64 weights,
 *     nearest of 16 levels), NF4 (normal-quantile levels, exact zero, ends +-1),
 *     二重量子化 (absmax constants centred by their mean, stored as 8-bit floats
 *     in groups of 256 with one fp32 constant per group), 勾配は実際どこへ行くのか
 *     (stored NF4, computed BF16; the gradient flows through deq(W) but W gets
 *     none; only A and B are trained);
 *   - "QLoRA" glossary (ultralytics), the NF4 level construction and the
 *     nearest-level argmin;
 *   - "waylandz LLM book ch.26", 26.2.4: y = W x + (alpha/r) B (A x); 26.2.2:
 *     the adapter merged once for inference, W + (alpha/r) B A.
 *
 * Conventions
 *   W is N x K row-major fp32 (bf16 for the *_bf16 quantisers; N = out
 *   features, K = in features), K % 64 == 0.
 *   X is M x K, Y is M x N, A is r x K, B is N x r, dY is M x N, all row-major.
 *   bf16 tensors are passed as uint16_t bit patterns (IEEE bfloat16).
 *   s = alpha / r.
 *   Every pointer argument is a DEVICE pointer unless it says "host".
 *   The caller allocates and frees every buffer (the library never allocates
 *   device memory); `stream` is a cudaStream_t (NULL = legacy default stream).
 *   Calls are asynchronous and stream-ordered. A return value of QLORA_OK means
 *   the arguments were valid and every kernel was launched; errors found by
 *   the device itself (a pipeline wait that ran out) are recorded in the
 *   workspace's status word, read back with qlora_device_status().
 *   Device buffers must be 16-byte aligned.
 *
 * Quantised weight format (qlora_nf4_weight), for nb = N*K/64 blocks and
 * ng = ceil(nb/256) groups:
 *   codes   uint8[N*K/2]  flat row-major element 2j in the HIGH nibble of byte j,
 *                         element 2j+1 in the low nibble; code = index of the
 *                         nearest NF4 level (0 = -1, 7 = 0, 15 = +1)
 *   qabsmax uint8[nb]     OCP FP8 E4M3 code of (absmax_b - mean) / s2_g
 *   s2      float[ng]     second-level constant of group g (blocks 256g..256g+255)
 *   mean    float[1]      mean of all first-level absmax constants
 *   Dequantised weight: c'_b = fmaf(E4M3(qabsmax_b), s2_g, mean) (one fp32
 *   rounding), w_hat = bf16_rn(fp32_rn(level[code] * c'_b)).
 *
 * Storage without double quantisation (absmax set in qlora_nf4_weight): the
 * same codes, and one fp32 constant per block, absmax float[nb] = the block's
 * max|w| itself, 4 + 32/64 = 4.5 bits per weight [explainer 二重量子化, the
 * count before the constants are quantised]. w_hat = bf16_rn(fp32_rn(
 * level[code] * absmax_b)).
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int qlora_status;

#define QLORA_OK                        0
#define QLORA_ERR_INVALID_ARG          -1  /* NULL pointer, alpha not finite, bad op   */
#define QLORA_ERR_BAD_SHAPE            -2  /* K % 64 != 0, N*K == 0, N % 8 != 0, M < 0 */
#define QLORA_ERR_MISALIGNED           -3  /* a device pointer not 16-byte aligned     */
#define QLORA_ERR_UNSUPPORTED_RANK     -4  /* r not in {8, 16, 32, 64}                 */
#define QLORA_ERR_WORKSPACE_TOO_SMALL  -5  /* ws_bytes < qlora_workspace_bytes(...)    */
#define QLORA_ERR_CUDA                 -6  /* a CUDA call or launch failed; see
                                              qlora_last_error()                        */
#define QLORA_ERR_DEVICE_TIMEOUT       -7  /* device status: a pipeline wait ran out   */
#define QLORA_ERR_UNSUPPORTED_DEVICE   -8  /* current device is not sm_100             */
#define QLORA_ERR_EXCEEDS_STATIC_SCRATCH -9 /* N*K above the no-allocation limit        */

/* Read-only view of a quantised weight. All pointers are device pointers
 * owned by the caller; the library never writes through them. With absmax
 * NULL (zero-initialised) the weight uses double quantisation and qabsmax,
 * s2 and mean are required; with absmax set it is stored without, and
 * qabsmax, s2 and mean are ignored (they may be NULL). */
typedef struct {
    const uint8_t* codes;
    const uint8_t* qabsmax;
    const float*   s2;
    const float*   mean;
    int64_t        N;
    int64_t        K;
    const float*   absmax;
} qlora_nf4_weight;

/* Sizes in bytes of the four buffers of an N x K quantised weight. Host only;
 * any out-pointer may be NULL. Returns their sum, or -1 for a bad shape.
 * 8 * sum / (N*K) = 4 + 8/64 + 32/(64*256) + 32/(N*K) bits per weight, the
 * 4.127 of the explainer's 二重量子化 section. */
int64_t qlora_nf4_bytes(int64_t N, int64_t K, size_t* codes, size_t* qabsmax,
                        size_t* s2, size_t* mean);

/* Workspace (device scratch, caller-allocated) needed by one call. */
#define QLORA_OP_QUANTIZE 0
#define QLORA_OP_FWD      1
#define QLORA_OP_BWD      2
/* Returns the byte count, or 0 for an invalid op/shape. Host only. */
size_t qlora_workspace_bytes(int op, int64_t M, int64_t N, int64_t K, int r);

/* Quantise W (fp32 [N, K], device) to NF4 with double quantisation.
 * [explainer 量子化を1段落で + NF4 + 二重量子化; glossary NF4 snippet]
 * Per 64-block: absmax c (fp32), v = w / c (IEEE fp32 division), code = number
 * of decision thresholds below v (exactly the nearest level, ties to the lower
 * index; a block with c == 0 codes every element 7). Then mean = fp32 of the
 * fp64 pairwise-tree sum of all c divided by nb; per group of 256 blocks
 * d = c - mean, s2 = max|d| / 448, qabsmax = E4M3_rn_satfinite(d / s2)
 * (0x00 when s2 == 0).
 * Outputs codes/qabsmax/s2/mean are device buffers sized by qlora_nf4_bytes;
 * ws needs qlora_workspace_bytes(QLORA_OP_QUANTIZE, 0, N, K, 0) bytes.
 * Deterministic: the same W always gives the same bits. */
qlora_status qlora_quantize_nf4(const float* W, int64_t N, int64_t K,
                                uint8_t* codes, uint8_t* qabsmax, float* s2, float* mean,
                                void* ws, size_t ws_bytes, void* stream);

/* qlora_quantize_nf4 for a weight stored in bf16 (bf16 [N, K], device): the
 * ordinary 16-bit form of pretrained weights [explainer, opening: a 65B
 * model is 130 GB of BF16 weights], and the form a 16-bit merge of the
 * adapters produces before it is quantised again [explainer 落とし穴].
 * Every bf16 value is exactly an fp32 value, so the result is bit for bit
 * that of qlora_quantize_nf4 on the fp32 upcast of W; the encoder reads half
 * the bytes. Arguments, workspace and errors as for qlora_quantize_nf4. */
qlora_status qlora_quantize_nf4_bf16(const uint16_t* W, int64_t N, int64_t K,
                                     uint8_t* codes, uint8_t* qabsmax, float* s2, float* mean,
                                     void* ws, size_t ws_bytes, void* stream);

/* The same quantisation as qlora_quantize_nf4, for callers that cannot
 * allocate device memory at the point of the call: inference-runtime plugin
 * interfaces that hand over only input and output buffers and no workspace,
 * and latency-critical code that must not call cudaMalloc because it can
 * block or synchronise the device in the middle of a step. The pages about
 * QLoRA have no counterpart to this call; it exists only for such callers.
 *   - It takes no workspace and allocates nothing. Its scratch (the fp32
 *     per-block absmax, the fp64 partial sums of the mean and a ticket)
 *     lives in one static device array of 4 MiB + 768 B that every GPU
 *     which loads the library keeps until the process exits.
 *   - Limit: N*K <= 67,108,864 weights (at most 1,048,576 blocks of 64, e.g.
 *     8192 x 8192). Larger weights return QLORA_ERR_EXCEEDS_STATIC_SCRATCH
 *     and launch nothing; use qlora_quantize_nf4 with a workspace instead.
 *   - Every call looks up the array's address in the current context
 *     (cudaGetSymbolAddress); the first call on a device, and the first after
 *     a cudaDeviceReset, also loads the library's module there, so make it
 *     before any stream capture on the device.
 *   - All calls share the one array: calls that overlap on the GPU (for
 *     example on two streams at once) race and corrupt each other's results.
 *     Calls in one stream are ordered and safe; nothing in the array has to
 *     start at zero, every byte read is written earlier in the same call
 *     (the ticket by the encoder).
 *   - Outputs, argument checks and determinism are those of
 *     qlora_quantize_nf4. */
qlora_status qlora_quantize_nf4_noalloc(const float* W, int64_t N, int64_t K,
                                        uint8_t* codes, uint8_t* qabsmax, float* s2, float* mean,
                                        void* stream);

/* Quantise without double quantisation [explainer 二重量子化, first
 * paragraph: one fp32 constant per block of 64, 4.5 bits per weight].
 * Codes exactly as qlora_quantize_nf4 (same rule, same bits); absmax
 * (float[N*K/64], device) receives each block's max|w|. W is fp32 [N, K]
 * (qlora_quantize_nf4_nodq) or bf16 [N, K] (qlora_quantize_nf4_bf16_nodq,
 * the bits of its fp32 upcast). No workspace; one kernel launch. Use the
 * result through a qlora_nf4_weight with absmax set. */
qlora_status qlora_quantize_nf4_nodq(const float* W, int64_t N, int64_t K,
                                     uint8_t* codes, float* absmax, void* stream);
qlora_status qlora_quantize_nf4_bf16_nodq(const uint16_t* W, int64_t N, int64_t K,
                                          uint8_t* codes, float* absmax, void* stream);

/* Dequantise to bf16 [N, K] (device W_out), bit-exact with the format's
 * definition above, for either storage. [explainer 量子化を1段落で:
 * x_hat = c * level[code]] */
qlora_status qlora_dequantize_nf4(const qlora_nf4_weight* w, uint16_t* W_out, void* stream);

/* Fold an adapter into a 16-bit copy of the weight for inference [waylandz
 * 26.2.2, inference: merge once, W_merged = W + (alpha/r) B A; explainer
 * 落とし穴: the merge goes to the 16-bit weight, not to the 4-bit one]:
 *   W_out = bf16_rn( fmaf(s, sum_j B[n, j] A[j, k], w_hat[n, k]) ),  s = alpha/r,
 * w_hat the dequantised weight above (either storage), the rank-r sum of
 * exact bf16 products accumulated in fp32 (order unspecified): an entry is
 * off the exact merge by at most one bf16 step plus that fp32 error.
 * A: bf16 [r, K]; B: bf16 [N, r]; W_out: bf16 [N, K] (device, caller-owned);
 * r in {8, 16, 32, 64}. No workspace: a device wait that ran out is recorded
 * in the status word read by qlora_device_status(NULL, ...); other errors as
 * for qlora_linear_fwd. To
 * store the merged weight in 4 bits again, quantise W_out with
 * qlora_quantize_nf4_bf16 (the update may be lost, as the explainer warns). */
qlora_status qlora_merge_lora(const qlora_nf4_weight* w, const uint16_t* A, const uint16_t* B,
                              int r, float alpha, uint16_t* W_out, void* stream);

/* Forward of the QLoRA linear layer [waylandz 26.2.4; explainer 勾配は...]:
 *   sT = bf16( s * X A^T )                    (M x r, written to sT_save if not NULL)
 *   Y  = bf16( X deq(W)^T + sT B^T )           (M x N)
 * The NF4 weight is dequantised tile by tile inside the matmul (no bf16 copy
 * of W is ever written to memory). X: bf16 [M, K]; A: bf16 [r, K];
 * B: bf16 [N, r]; r in {8, 16, 32, 64}; M >= 0 (M == 0 is a no-op).
 * ws needs qlora_workspace_bytes(QLORA_OP_FWD, M, N, K, r) bytes. */
qlora_status qlora_linear_fwd(const uint16_t* X, int64_t M, const qlora_nf4_weight* w,
                              const uint16_t* A, const uint16_t* B, int r, float alpha,
                              uint16_t* Y, uint16_t* sT_save,
                              void* ws, size_t ws_bytes, void* stream);

/* Backward of the layer, gradients of <dY, Y> [explainer 勾配は実際どこへ行くのか:
 * the input gradient needs deq(W)^T; W itself gets no gradient]:
 *   sU = bf16( s * dY B )                      (M x r)
 *   dX = bf16( dY deq(W) + sU A )               (M x K)
 *   dA = fp32( sU^T X )      = s (dY B)^T X     (r x K, overwritten)
 *   dB = fp32( dY^T sT )     = s dY^T (X A^T)   (N x r, overwritten)
 * sT is the forward's sT_save (bf16 [M, r]) or NULL to recompute it.
 * ws needs qlora_workspace_bytes(QLORA_OP_BWD, M, N, K, r) bytes. */
qlora_status qlora_linear_bwd(const uint16_t* dY, const uint16_t* X, int64_t M,
                              const qlora_nf4_weight* w, const uint16_t* A, const uint16_t* B,
                              int r, float alpha, const uint16_t* sT,
                              uint16_t* dX, float* dA, float* dB,
                              void* ws, size_t ws_bytes, void* stream);

/* Several adapters over one frozen base in one call ["waylandz LLM book
 * ch.26", 26.7.3: one base model hosts many adapters and switches between
 * them at run time; "agentlenshq" summary, 利用ケース: one 4-bit base serves
 * several adapters]. Token row m uses adapter k = ids[m]:
 *   Y[m] = X[m] deq(W)^T + (alpha/r) (X[m] A_k^T) B_k^T.
 * P adapters of one rank r in {8, 16, 32, 64}, P r <= 256; all share alpha.
 *   A:   bf16 [P r, K], adapter k in rows [k r, (k + 1) r) (the A_k stacked)
 *   B:   bf16 [N, P r], adapter k in columns [k r, (k + 1) r) (the B_k side by side)
 *   ids: int32 [M] (device, 4-byte aligned); a row whose id is outside
 *        [0, P) uses no adapter (the frozen base layer only).
 * The rank-r inputs are those of a layer of rank P r whose columns other
 * than the row's own adapter are zero: sT_save (bf16 [M, P r], may be NULL)
 * holds s X A_k^T in the row's own columns and zeros elsewhere. The
 * backward returns every adapter's gradients at once, each from the rows
 * that use it (an adapter no row uses gets exactly zero):
 *   dA: fp32 [P r, K] (dA_k in rows [k r, (k + 1) r)), dB: fp32 [N, P r].
 * sT: the forward's sT_save, or NULL to recompute it. The workspace size
 * comes from qlora_workspace_bytes_multi (same op codes, P adapters of rank
 * r). Errors, asynchrony and ownership as for qlora_linear_fwd/bwd; ids is
 * read on the device only. */
size_t qlora_workspace_bytes_multi(int op, int64_t M, int64_t N, int64_t K, int r, int P);
qlora_status qlora_linear_fwd_multi(const uint16_t* X, int64_t M, const qlora_nf4_weight* w,
                                    const uint16_t* A, const uint16_t* B, int r, int P,
                                    const int32_t* ids, float alpha, uint16_t* Y, uint16_t* sT_save,
                                    void* ws, size_t ws_bytes, void* stream);
qlora_status qlora_linear_bwd_multi(const uint16_t* dY, const uint16_t* X, int64_t M,
                                    const qlora_nf4_weight* w, const uint16_t* A, const uint16_t* B,
                                    int r, int P, const int32_t* ids, float alpha, const uint16_t* sT,
                                    uint16_t* dX, float* dA, float* dB,
                                    void* ws, size_t ws_bytes, void* stream);

/* Projections that share one input, each with its own frozen NF4 weight and
 * adapter, in one call: q, k, v of attention or gate and up of the MLP
 * ["ta-paperlens QLoRA explainer", コードで見る: target_modules names every
 * linear layer; 落とし穴: adapters on attention alone leave a gap].
 * w[0..P-1] (1 <= P <= 4): weights N_i x K, all with the same K and the same
 * storage (all with or all without double quantisation), each quantised on
 * its own (its own mean and s2), and with their codes back to back in one
 * buffer: w[i+1].codes == w[i].codes + N_i K / 2 (quantise each into its
 * slice of one allocation). N = sum N_i.
 *   A:  bf16 [P r, K], projection i's A_i in rows [i r, (i + 1) r)
 *   B:  bf16 [N, r], the B_i [N_i, r] stacked (projection i in rows
 *       [n_i, n_i + N_i), n_i = N_0 + ... + N_{i-1})
 *   Y:  bf16 [M, N] = [Y_0 | Y_1 | ...], Y_i = X deq(W_i)^T + (alpha/r) (X A_i^T) B_i^T
 *   sT_save: bf16 [M, P r] = [s X A_0^T | s X A_1^T | ...] (may be NULL)
 * Backward, with dY bf16 [M, N] = [dY_0 | dY_1 | ...]:
 *   dX = sum_i (dY_i deq(W_i) + (alpha/r) (dY_i B_i) A_i)   bf16 [M, K]
 *   dA: fp32 [P r, K] (dA_i in rows [i r, (i + 1) r))
 *   dB: fp32 [N, r]   (dB_i in rows [n_i, n_i + N_i))
 * r in {8, 16, 32, 64}. The workspace size comes from
 * qlora_workspace_bytes_group (N: host array of the P row counts). Errors,
 * asynchrony and ownership as for qlora_linear_fwd/bwd. */
size_t qlora_workspace_bytes_group(int op, int64_t M, const int64_t* N, int P, int64_t K, int r);
qlora_status qlora_linear_fwd_group(const uint16_t* X, int64_t M, const qlora_nf4_weight* w, int P,
                                    const uint16_t* A, const uint16_t* B, int r, float alpha,
                                    uint16_t* Y, uint16_t* sT_save,
                                    void* ws, size_t ws_bytes, void* stream);
qlora_status qlora_linear_bwd_group(const uint16_t* dY, const uint16_t* X, int64_t M,
                                    const qlora_nf4_weight* w, int P, const uint16_t* A,
                                    const uint16_t* B, int r, float alpha, const uint16_t* sT,
                                    uint16_t* dX, float* dA, float* dB,
                                    void* ws, size_t ws_bytes, void* stream);

/* Host copies of the library's own NF4 tables: levels[16] (fp32, ascending)
 * and thresholds[15] (the fp32 decision points between neighbouring levels).
 * Computed on the host at load time, independently of any test code. */
qlora_status qlora_nf4_tables(float* levels_host, float* thresholds_host);

/* Read the device status word at the head of a fwd/bwd workspace (0 = ok,
 * otherwise a QLORA_ERR_DEVICE_* code). With ws = NULL it reads, and clears,
 * the library's own status word of the calls that take no workspace
 * (qlora_merge_lora) on the current device. Synchronises `stream`. */
qlora_status qlora_device_status(const void* ws, int* status_host, void* stream);

/* Human-readable name of a status code, and the text of the last CUDA error
 * seen by this thread (empty if none). Host only; static strings. */
const char* qlora_status_string(qlora_status s);
const char* qlora_last_error(void);

/* Test and tuning hooks (not needed for normal use).
 *   QLORA_OPT_SMALL_M_MAX   token count up to which the forward uses the
 *                           small-batch weight-streaming kernel (default 16,
 *                           maximum 64; 0 forces the tiled GEMM for every M);
 *                           above it the tiled GEMM, which splits its tiles
 *                           over K when they are fewer than the SMs
 *   QLORA_OPT_FAIL_LAUNCHES the next `value` kernel launches report
 *                           QLORA_ERR_CUDA without launching (host-side fault
 *                           injection; nothing reaches the GPU)
 *   QLORA_OPT_WAIT_TIMEOUT_US per-wait limit of the pipelined kernels' barrier
 *                           waits in microseconds (default 1000000)
 *   QLORA_OPT_STALL_PRODUCER 1 = the next forward's tiled GEMM loads nothing,
 *                           so its consumers' waits run out and the device
 *                           status reports QLORA_ERR_DEVICE_TIMEOUT */
#define QLORA_OPT_SMALL_M_MAX     1
#define QLORA_OPT_FAIL_LAUNCHES   2
#define QLORA_OPT_WAIT_TIMEOUT_US 3
#define QLORA_OPT_STALL_PRODUCER  4
#define QLORA_OPT_LAUNCH_COUNT    5  /* read: kernels launched by this library so
                                        far in this process; set: reset to value */
#define QLORA_OPT_SKINNY_MAX_SPLITS 6 /* tuning: cap on the reduction splits of
                                        the rank-r matmuls, which are the CTAs
                                        of one cluster: 1, 2, 4 or 8 (0 = no
                                        cap; other values round down to one of
                                        these; workspaces do not depend on it) */
#define QLORA_OPT_FUSED_PAIRS     8  /* 1 (default): with whole output tiles the
                                        fused matmuls run in CTA pairs sharing
                                        each dequantised weight tile; 0: one
                                        CTA per tile, each decoding its own */
#define QLORA_OPT_FUSED_TAIL      9  /* 1: when the last wave of CTA pairs
                                        would be short, its tiles run on the
                                        one-CTA kernel split over every SM
                                        (stream-K, fp32 partial tiles added in
                                        a fixed order); 0 (default): whole
                                        waves of pairs only */
qlora_status qlora_set_option(int option, int64_t value);
int64_t qlora_get_option(int option);

/* Profiling hook: record the CUDA events ev_start / ev_stop (cudaEvent_t,
 * owned by the caller) on the launch stream immediately before and after the
 * next launch of the named kernel; the request is consumed by that launch.
 * Inside stream capture the records are external event records, so the
 * captured graph times every replay. A profiled call launches that kernel in
 * plain stream order (an event between two launches breaks a programmatic
 * dependent launch), so it may run a little slower than an unprofiled one. */
#define QLORA_KERNEL_FUSED_FWD 1   /* the forward's weight kernel: the
                                      dequant-fused matmul, or the small-batch
                                      kernel when M <= QLORA_OPT_SMALL_M_MAX  */
#define QLORA_KERNEL_FUSED_DX  2   /* the transposed-dequant dX matmul       */
qlora_status qlora_profile_next_launch(int kernel, void* ev_start, void* ev_stop);

/* Test hook: E4M3 round-to-nearest-even with saturation, exactly as the
 * double quantisation stores constants (the sm_100 cvt instruction), on n
 * device floats. */
qlora_status qlora_e4m3_encode(const float* x, uint8_t* q, int64_t n, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_NF4_H */
