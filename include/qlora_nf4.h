/*
 * qlora_nf4.h -- C ABI of the B200 (sm_100a) QLoRA NF4 linear-layer library.
 *
 * The library implements the data-parallel hot path of QLoRA (Dettmers et al.
 * 2023) as described on the pages "QLoRAの理論と実装" (disassemble-channel.com)
 * and the Qiita article on why QLoRA survives 4-bit:
 *
 *   1. blockwise NF4 quantization of a frozen fp32 weight with double
 *      quantization of its absmax constants (§5-1 and §5-2 of the first page);
 *   2. the frozen-NF4 linear layer with its LoRA adapter, computed in bf16
 *      (the "storage 4-bit / compute BF16" split), forward and backward
 *      ("QLoRAの計算フロー", "逆伝播と勾配の流れ").
 *
 * Conventions shared by every entry point
 * ----------------------------------------
 * - Shapes: the weight W is N x K (n_out x k_in), row-major, the pages' d x k.
 *   Activations X are M x K (tokens x in), outputs Y are M x N.  LoRA A is
 *   r x K, B is N x r, the adapter scale is s = alpha / r.
 * - bf16 tensors are passed as uint16_t bit patterns; fp32 as float.
 * - Every pointer argument is a DEVICE pointer (CUDA global memory on the
 *   current device), except where a comment says "host".  The caller owns
 *   every buffer; the library allocates no device memory.  Scratch comes from
 *   the caller's `workspace` (size from qlora_workspace_bytes).
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   Every call is asynchronous on that stream: it validates its arguments on
 *   the host, enqueues kernels and returns.
 * - The quantized weight is three flat buffers (double quantization):
 *     codes  uint8_t[N*K/2]      NF4 codes, row-major, element 2j in the low
 *                                nibble of byte j;
 *     q8     uint8_t[N*K/64]     8-bit absmax constant of each 64-block;
 *     s2     float[ceil(N*K/16384)]  fp32 second-level constant of each group
 *                                of 256 consecutive blocks.  Its sign bit
 *                                gives the group's 8-bit format: clear =
 *                                linear (c1 = q8 * s2), set = FP8-E4M3
 *                                (c1 = E4M3(q8) * |s2|);
 *   or, with single quantization (the second stage off, 4.5 bit/param), two:
 *     codes  as above;  q8 = NULL;
 *     s2     float[N*K/64]       the fp32 absmax constant of each 64-block.
 *   Every call that takes (codes, q8, s2) reads q8 == NULL as single
 *   quantization.  Fixed by the method: block 64, group 256.
 * - Preconditions checked on the host (QLORA_ERR_* on violation, nothing
 *   enqueued): non-NULL required pointers, every pointer 16-byte aligned,
 *   K % 64 == 0, N % 64 == 0 (N, K >= 64 for the layer), M >= 0,
 *   1 <= r <= 256 with r % 8 == 0, alpha finite.  NaN or Inf inside W is a
 *   caller error; the result is unspecified.
 * - Empty inputs.  M == 0 (an empty batch, e.g. a data-parallel rank that
 *   received no tokens) is valid: the forward enqueues nothing, the backward
 *   sets dA and dB to zero (sums over no tokens) and nothing else, and the
 *   pointers to M-row buffers (X, Y, U, dY, dX) may be NULL.  A weight with
 *   no element (n_out == 0 or k_in == 0) makes the quantizers, the
 *   dequantizer and the merge no-ops whose pointers may be NULL.  The layer
 *   itself needs N, K >= 64.
 * - Launch order.  Every kernel is launched with programmatic stream
 *   serialisation, and the first kernel of a call waits for the previous work
 *   on the stream to complete before it reads anything.  Stream order holds as
 *   usual: a call reads its inputs after all earlier work on the stream and
 *   its outputs are complete for all later work.  One exception is a later
 *   kernel that the caller launches with programmatic stream serialisation of
 *   its own.  It may start before the call's last kernel ends, and it must
 *   wait for its grid dependency (cudaGridDependencySynchronize) before it
 *   touches the call's outputs.  Inside a call, kernels overlap where their
 *   data allow: the fused kernels start on the adapter products' free SMs, and
 *   the backward's gradient kernel runs on a second, library-owned stream of
 *   the device, joined back before the call's last kernel completes.
 * - Return value: QLORA_OK (0) or a negative QLORA_ERR_* code.  Errors raised
 *   on the device after a call returned (a bounded wait inside a kernel that
 *   gave up) are latched in a device flag and reported by qlora_device_status.
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QLORA_OK 0
#define QLORA_ERR_INVALID_ARG (-1)     /* NULL pointer, r or alpha out of range    */
#define QLORA_ERR_UNSUPPORTED_SHAPE (-2) /* K or N not a multiple of 64, misalignment */
#define QLORA_ERR_CUDA (-3)            /* a CUDA runtime call or launch failed      */
#define QLORA_ERR_DEVICE_TIMEOUT (-4)  /* a kernel's bounded wait expired           */
#define QLORA_ERR_WORKSPACE (-5)       /* workspace NULL or smaller than required   */
#define QLORA_ERR_NO_DEVICE (-6)       /* no sm_100 device is current               */
#define QLORA_ERR_UNAVAILABLE (-7)     /* the call needs the checked build           */

#define QLORA_OUT_BF16 0
#define QLORA_OUT_FP32 1

/* Human-readable name of a return code (static string, never NULL). */
const char* qlora_strerror(int code);

/*
 * The 16 NF4 levels, ascending, as fp32 (host pointer `out`, 16 floats).
 * Built once on the host from the quantile definition of "QLoRAの理論と実装",
 * listing create_nf4_codebook (levels Phi^-1(i/18), i=1..8, then 0, then
 * Phi^-1(j/16), j=9..15, divided by |Phi^-1(1/18)|).  Returns QLORA_OK.
 */
int qlora_nf4_codebook(float* out);

/*
 * Blockwise NF4 quantization with double quantization.
 * "QLoRAの理論と実装" §5-1 (steps 1-2: absmax per 64 elements, w/absmax,
 * nearest of the 16 levels stored in 4 bits) and §5-2 (the fp32 absmax
 * constants re-quantized to 8 bits in groups of 256 with one fp32
 * second-level constant); the Qiita page's W ~ (c2 * c1_quant) * W_quant.
 *
 *   W      fp32[N*K] device, row-major, read only.
 *   codes  uint8_t[N*K/2]   written.
 *   q8     uint8_t[N*K/64]  written.
 *   s2     float[ceil(N*K/16384)] written.
 * Per block: absmax = max|w|; n = fp32(w/absmax) (0 if absmax == 0); code =
 * exact nearest level, lowest index on a tie.  Per group of 256 blocks:
 * s2 = fp32(max absmax / 255); q = min(255, round-half-even(fp32(absmax/s2))),
 * q = 0 when s2 == 0.  One kernel launch.
 */
int qlora_quantize_nf4_dq(const float* W, int64_t n_out, int64_t k_in,
                          uint8_t* codes, uint8_t* q8, float* s2, void* stream);

/*
 * The same with the FP8 reading of the second stage ("QLoRAの理論と実装" §5-2:
 * "8bit量子化（FP8相当）"): per group of 256 blocks s = fp32(c2 / 448), so the
 * group maximum maps to E4M3's largest finite value, and
 * q = E4M3(fp32(absmax / s)), rounded to nearest even and saturated at 448
 * (q = 0 when s == 0).  s2 receives -s: the sign bit marks the FP8 format,
 * and every call that reads (codes, q8, s2) decodes c1 = fp32(E4M3(q) * s).
 * Same buffers and sizes as qlora_quantize_nf4_dq; codes are identical.
 * One kernel launch.
 */
int qlora_quantize_nf4_dq_fp8(const float* W, int64_t n_out, int64_t k_in,
                              uint8_t* codes, uint8_t* q8, float* s2, void* stream);

/*
 * Blockwise NF4 quantization without the second stage (single quantization):
 * "QLoRAの理論と実装" §5-1 steps 1-2 alone; §5-2's memory arithmetic prices it
 * at 4 + 32/64 = 4.5 bit/param, and the page's bitsandbytes listing selects it
 * with bnb_4bit_use_double_quant=False.
 *
 *   W       fp32[N*K] device, row-major, read only.
 *   codes   uint8_t[N*K/2] written (identical to qlora_quantize_nf4_dq's).
 *   absmax  float[N*K/64]  written: max|w| of each 64-block, exact.
 * Pass (codes, NULL, absmax) to the dequantization and linear-layer calls.
 * One kernel launch.
 */
int qlora_quantize_nf4(const float* W, int64_t n_out, int64_t k_in,
                       uint8_t* codes, float* absmax, void* stream);

/*
 * Dequantization to a dense N x K matrix ("QLoRAの理論と実装" §5-1 step 3 with
 * the two-level constant):  w = fp32(level[code] * c1) with c1 = fp32(q8 * s2)
 * (or fp32(E4M3(q8) * |s2|) for an FP8 group), or with q8 == NULL
 * w = fp32(level[code] * absmax) (s2 = absmax), written as
 * fp32 (out_dtype QLORA_OUT_FP32) or rounded to nearest-even bf16
 * (QLORA_OUT_BF16).  `out` is device memory of N*K elements.  This is for
 * tests and export; the linear layer never materialises it.
 */
int qlora_dequant(const uint8_t* codes, const uint8_t* q8, const float* s2,
                  int64_t n_out, int64_t k_in, void* out, int out_dtype,
                  void* stream);

/*
 * Adapter merge for distribution ("QLoRAとは？4bit量子化＋LoRAの仕組み・VRAM
 * 目安・実装手順と採用判断を解説", section on merging a trained adapter):
 * merging onto the 4-bit base rounds the adapter's small differences onto the
 * 4-bit grid, so the adapter is folded into the unquantized base in bf16 and
 * the merged 16-bit weight is quantized again.  Per element:
 *   merged = bf16( fp64(bf16(W)) + fp64(s) * sum_{j=0..r-1} B[n,j] A[j,k] ),
 * the sum in fp64 in that order (each product and addition rounded once,
 * no fused multiply-add), one rounding to bf16 at the end; s = fp32(alpha/r).
 *
 *   W    fp32[N*K] device, the original (unquantized) weight, read only.
 *   A    bf16[r*K], B bf16[N*r] device (the trained adapter), read only.
 *   out  N*K elements: bf16 bits (QLORA_OUT_BF16), or the same bf16 values as
 *        fp32 (QLORA_OUT_FP32), which qlora_quantize_nf4_dq / qlora_quantize_nf4
 *        take directly to re-quantize.
 * 1 <= r <= 256, alpha finite, K % 64 == 0, N <= 1048560, every pointer 16-byte
 * aligned.  One kernel launch.  There is no counterpart that merges into the NF4
 * weight: that is the lossy path the page warns against.
 */
int qlora_merge_adapter(const float* W, int64_t n_out, int64_t k_in, const uint16_t* A, const uint16_t* B, int r,
                        float alpha, void* out, int out_dtype, void* stream);

/* Bytes of workspace qlora_linear_fwd / qlora_linear_bwd need for these sizes
 * (0 on invalid sizes).  The workspace is device memory, 256-byte aligned,
 * owned by the caller; its contents need not be initialised and are not
 * preserved between calls. */
size_t qlora_workspace_bytes(int64_t M, int64_t n_out, int64_t k_in, int r);

/*
 * Forward of the frozen-NF4 linear layer with LoRA, "QLoRAの計算フロー"
 * steps 1-4 and "LoRAの復習" (h = W0 x + (alpha/r) B A x), row-major:
 *
 *   U = X A^T                        (M x r, fp32 accumulate)
 *   Y = X dequant(W)^T + s U B^T     (M x N, fp32 accumulate, bf16 out)
 *
 * dequant(W) is rebuilt tile by tile in shared memory and consumed there by
 * the tensor cores; no dense copy of W is written.
 *   X  bf16[M*K], A bf16[r*K], B bf16[N*r]  read.
 *   Y  bf16[M*N]  written.
 *   U_save bf16[M*r] written with U (for the backward pass) unless NULL.
 * Launches by batch size: M <= 4, two (U, which also prefetches the packed
 * weight into L2, then a kernel that turns each code byte into a pair of fp16
 * NF4 levels through a shared-memory table and applies c1 to each 64-column
 * block's fp32 dot product, so it multiplies by the fp32 dequantized value
 * level * c1 (to the level's fp16 rounding) rather than its bf16 rounding: a
 * difference of about 2^-9 of each weight, well within the layer's tolerance;
 * shapes whose table-kernel shared memory would exceed 224 KiB take the next
 * path instead); M <= 32, one (few-token tensor-memory kernel); larger M, U and
 * then the fused GEMM.
 */
int qlora_linear_fwd(const uint8_t* codes, const uint8_t* q8, const float* s2,
                     int64_t n_out, int64_t k_in,
                     const uint16_t* X, int64_t M,
                     const uint16_t* A, const uint16_t* B, int r, float alpha,
                     uint16_t* Y, uint16_t* U_save,
                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * Forward without any allocation (the pages have no counterpart; this is an
 * integration aid).  Same computation, arguments and results as
 * qlora_linear_fwd, but the scratch comes from a fixed device array inside the
 * library instead of a caller workspace.  It is for callers that cannot call
 * cudaMalloc or hand over a workspace: a host whose device memory is entirely
 * owned by another allocator, or a latency-bound caller that cannot afford
 * cudaMalloc's implicit device synchronisation.
 *
 * - Limit: the fixed scratch is 4 MiB per device, held by every GPU that loads
 *   the library until the process exits.  A call with
 *   qlora_workspace_bytes(M, N, K, r) > 4 MiB (M * r above about 524,288)
 *   returns QLORA_ERR_WORKSPACE and enqueues nothing.
 * - Allocates nothing: no cudaMalloc, cudaFree or allocating library routine,
 *   as long as launch timing (qlora_timing_enable) is off, which is the default.
 * - Set-up: the first call on a device looks up the scratch's device address
 *   (cudaGetSymbolAddress, with that device current) and caches it.  Make that
 *   first call before any stream capture.  The cached address belongs to the
 *   device's primary context: after cudaDeviceReset it is stale, so do not
 *   call this entry point again in that process.
 * - Sharing: every call uses the same scratch, which keeps the last call's
 *   contents.  Every element this path reads is written by the same call first,
 *   so nothing needs clearing.  Calls that overlap on the GPU (different
 *   streams, or different host threads) race on the scratch: serialise them.
 */
int qlora_linear_fwd_noalloc(const uint8_t* codes, const uint8_t* q8, const float* s2,
                             int64_t n_out, int64_t k_in,
                             const uint16_t* X, int64_t M,
                             const uint16_t* A, const uint16_t* B, int r, float alpha,
                             uint16_t* Y, uint16_t* U_save, void* stream);

/*
 * Backward, "逆伝播と勾配の流れ" (W frozen, gradients reach A and B only):
 *
 *   V  = dY B                                  (M x r)
 *   dB = s dY^T U        (dL/dB = (alpha/r) dL/dY (A X)^T)     fp32 N x r
 *   dA = s V^T X         (dL/dA = (alpha/r) B^T dL/dY X^T)     fp32 r x K
 *   dX = dY dequant(W) + s V A   (chain rule through both paths) bf16 M x K
 *
 *   dY bf16[M*N] read; U_saved bf16[M*r] from the forward, or NULL to
 *   recompute U = X A^T here.  dX may be NULL (not computed).  dA and dB are
 *   overwritten (not accumulated).  The reductions over M are deterministic:
 *   the same inputs give bit-identical dA and dB on every call.
 *
 *   With dX requested, the kernel for dA and dB runs on a second stream that
 *   the library keeps per device, forked from `stream` by an event and joined
 *   back before the call returns, so the caller sees plain stream order.  A
 *   stream capture on `stream` takes that branch into its graph.  While the
 *   second stream belongs to a capture of another stream, calls outside that
 *   capture keep the kernel on their own stream.  Calls from several host
 *   threads take turns on the second stream under a lock.
 */
int qlora_linear_bwd(const uint8_t* codes, const uint8_t* q8, const float* s2,
                     int64_t n_out, int64_t k_in,
                     const uint16_t* X, int64_t M,
                     const uint16_t* A, const uint16_t* B, int r, float alpha,
                     const uint16_t* dY, const uint16_t* U_saved,
                     uint16_t* dX, float* dA, float* dB,
                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * LoRA dropout on the adapter input ("QLoRAの理論と実装", PEFT listing:
 * LoraConfig(..., lora_dropout=0.05)).  The adapter sees x * keep / (1 - p);
 * the frozen NF4 path sees x:
 *   Y  = X dequant(W)^T + s (Xd A^T) B^T,  U = Xd A^T,  Xd = X * keep / (1 - p)
 *   dX = dY dequant(W) + s ((dY B) A) * keep / (1 - p)
 *   dA = s (dY B)^T Xd,  dB = s dY^T U
 * keep(e) for element e = m*K + k of X: the 16-bit half (e & 1), low half
 * first, of word ((e >> 1) & 3) of Philox4x32-10 (Salmon et al., SC'11) at
 * counter (lo32(e>>3), hi32(e>>3), lo32(offset), hi32(offset)) with key
 * (lo32(seed), hi32(seed)) is >= floor(p * 2^16), so the drop probability is
 * within 2^-16 of p; the scale is fp32(1 / (1 - p)); both are taken from the
 * fp32 p.  p must be in
 * [0, 1) (else QLORA_ERR_INVALID_ARG); p == 0 is exactly the plain call.
 * Pass the same (p, seed, offset) to the forward and the backward of a step.
 * The workspace must hold qlora_workspace_bytes_dropout(M, N, K, r) bytes
 * (the plain size plus a bf16 M x K masked copy of X and the keep bits).
 *
 * Kept dropout state (optional; both pointers or neither, 16-byte aligned):
 *   Xd_save   bf16 [M x K]: the forward writes X * keep (dropped elements +0,
 *             the 1/(1 - p) not applied), the adapter's input;
 *   keep_save uint32 [M*K/32]: bit (e mod 32) of word e/32 is the keep
 *             decision of element e = m*K + k.
 * Given the same buffers as Xd_saved / keep_saved, the backward reads them
 * instead of generating the mask again (what an autograd framework saves for
 * dropout's backward), which takes one pass over X out of the backward; the
 * results are bit-identical either way.  NULL, NULL: the backward generates
 * the mask from (seed, offset) as the forward did.  Ignored when p == 0.
 *
 * Arguments otherwise as qlora_linear_fwd / qlora_linear_bwd.  Launches: mask,
 * U, the fused GEMM (forward); [mask], [U], V, dY dequant(W), the masked
 * adapter term of dX, dA/dB (backward; the mask pass only without kept state,
 * U only when U_saved is NULL).  M <= 32 takes the tiled path (the few-token
 * kernel forms U from the unmasked tile).
 */
size_t qlora_workspace_bytes_dropout(int64_t M, int64_t n_out, int64_t k_in, int r);

int qlora_linear_fwd_dropout(const uint8_t* codes, const uint8_t* q8, const float* s2,
                             int64_t n_out, int64_t k_in,
                             const uint16_t* X, int64_t M,
                             const uint16_t* A, const uint16_t* B, int r, float alpha,
                             float p, uint64_t seed, uint64_t offset,
                             uint16_t* Y, uint16_t* U_save,
                             uint16_t* Xd_save, uint32_t* keep_save,
                             void* workspace, size_t workspace_bytes, void* stream);

int qlora_linear_bwd_dropout(const uint8_t* codes, const uint8_t* q8, const float* s2,
                             int64_t n_out, int64_t k_in,
                             const uint16_t* X, int64_t M,
                             const uint16_t* A, const uint16_t* B, int r, float alpha,
                             float p, uint64_t seed, uint64_t offset,
                             const uint16_t* dY, const uint16_t* U_saved,
                             const uint16_t* Xd_saved, const uint32_t* keep_saved,
                             uint16_t* dX, float* dA, float* dB,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * The masked adapter input of the dropout calls: out = X * keep (bf16 M x K,
 * dropped elements +0; the 1/(1 - p) is not applied).  For tests and export;
 * the dropout calls form it in their workspace.  One kernel launch.
 */
int qlora_dropout_apply(const uint16_t* X, int64_t M, int64_t k_in, float p, uint64_t seed,
                        uint64_t offset, uint16_t* out, void* stream);

/*
 * Diagnostic for the failure path.  Enqueues one warp that waits, bounded, on
 * an mbarrier nothing arrives at: the wait gives up after the library's limit
 * (2 s of %globaltimer), latches the device error flag exactly as an expired
 * wait in any kernel does, and the kernel exits normally (no trap, fault or
 * hang; the context stays usable).  qlora_device_status then returns
 * QLORA_ERR_DEVICE_TIMEOUT once.  waited_ns: device uint64 receiving the
 * wait's duration in ns, or NULL.  The pages have no counterpart.
 */
int qlora_selftest_device_timeout(unsigned long long* waited_ns, void* stream);

/*
 * Synchronises `stream`, then returns and clears the device error flag of the
 * current device: QLORA_OK, QLORA_ERR_DEVICE_TIMEOUT if a kernel's bounded
 * wait expired since the last call, or QLORA_ERR_CUDA if the stream reports a
 * CUDA error.
 */
int qlora_device_status(void* stream);

/*
 * Launch timing (measurement support; no counterpart on the pages).
 * While enabled, the library records a CUDA event pair on the launching
 * stream around every kernel it enqueues.  qlora_timing_collect synchronises
 * those events, adds each launch's elapsed milliseconds to ms[kind] and
 * counts[kind] (host arrays of QLORA_KERNEL_COUNT entries, accumulated into,
 * not overwritten) and forgets them.  Kinds are the QLORA_KERNEL_* values.
 * Enabling clears any uncollected records.  Not thread-safe with respect to
 * concurrent calls from several host threads while enabled.
 */
#define QLORA_KERNEL_QUANTIZE 0    /* NF4 + double quant                     */
#define QLORA_KERNEL_DEQUANT 1     /* dense dequantization                   */
#define QLORA_KERNEL_LORA_GEMM 2   /* U = X A^T or V = dY B (split partials)  */
#define QLORA_KERNEL_LORA_REDUCE 3 /* reduction of U / V partials            */
#define QLORA_KERNEL_FWD 4         /* fused dequant GEMM: Y                   */
#define QLORA_KERNEL_DX 5          /* fused transposed-dequant GEMM: dX       */
#define QLORA_KERNEL_GRAD_GEMM 6   /* dA^T = X^T V, dB = dY^T U (partials)    */
#define QLORA_KERNEL_GRAD_REDUCE 7 /* reduction of dA / dB partials          */
#define QLORA_KERNEL_FWD_DECODE 8  /* small-M forward (M <= 32)              */
#define QLORA_KERNEL_MERGE 9       /* adapter merge into the 16-bit base      */
#define QLORA_KERNEL_DROPOUT 10    /* dropout mask / masked adapter dX        */
#define QLORA_KERNEL_COUNT 11
int qlora_timing_enable(int on);
/* Number of kernels the library has enqueued since it was loaded (all
 * devices, all streams), counted whether or not timing is enabled. */
int64_t qlora_launch_count(void);
int qlora_timing_collect(double* ms, int64_t* counts, int n_kinds);

/*
 * Checked build: libqlora_nf4_debug.so, the same library compiled with
 * QLORA_DEBUG (build.py --debug).  Its kernels check, before each access, the
 * coordinates and shared-memory address of every TMA copy (x a multiple of 16
 * bytes, no store at a negative coordinate, 16-byte aligned shared memory), the
 * offsets of every cluster exchange (inside the receiving region) and the
 * alignment of the quantizer's bulk copies.  A failed check is counted, the
 * first one's code, value and CTA are kept, and the access is skipped (the
 * kernel then ends through its bounded waits, with QLORA_ERR_DEVICE_TIMEOUT).
 * It stands in for a memory checker on GPUs where none can run; results are
 * bit-identical to the ordinary build's.  No counterpart on the pages.
 *
 *   out[0] failed checks since the last call, out[1] the first one's code
 *   (1 TMA x misaligned, 2 TMA store at a negative coordinate, 3 shared-memory
 *   address misaligned, 4 cluster-exchange offset out of range, 5 bulk copy
 *   misaligned), out[2] its value, out[3] its CTA (linear index).  out: host
 *   int64[4].  Reads and clears the record of the current device; synchronises
 *   with the device.  The ordinary build returns QLORA_ERR_UNAVAILABLE.
 */
int qlora_debug_record(int64_t* out);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_NF4_H */
