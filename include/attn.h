/*
 * attn.h -- C ABI of libattn.so: the fused, exact scaled-dot-product attention
 * forward for NVIDIA B200 (sm_100a).
 *
 * Operation (aiinarabic.com "flash-attention", Equation (1), with the optional
 * additive bias and sigmoid gate of the gated Evoformer variant named in the
 * gist.science FLASHLIGHT summary):
 *
 *     S   = scale * Q K^T (+ bias),   S_ij = -inf for j > i + (Nk - N) when causal
 *     O   = softmax_rows(S) V   (then O <- O * sigmoid(G) when a gate is given)
 *     lse = per-row natural-log logsumexp of S, i.e. m + ln(l) for the row
 *           maximum m and the sum l of exp(S - m); the gate does not enter it.
 *
 * It is computed block by block with an online softmax (running max and
 * running sum, the sum rescaled by e^(m_old - m_new) when the max grows; the
 * gist.science FLASHLIGHT summary, Methodology item 3), so the N x N score
 * matrix never reaches global memory (aiinarabic.com "flash-attention", the
 * kernel-fusion and tiling sections).  lse is the per-row normaliser that a
 * backward pass needs to recompute the softmax (the same page, recomputation).
 *
 * Threading and ownership: the caller owns every buffer.  The library keeps no
 * per-call allocations; it caches nothing but an internal device status word.
 * All calls are asynchronous on `stream` and never synchronise it (except
 * attn_last_device_status, which says so).  Outputs are valid once `stream`
 * reaches the call.
 */
#ifndef ATTN_B200_ATTN_H_
#define ATTN_B200_ATTN_H_

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID_ARG = 1,   /* null pointer, shape/stride mismatch, misalignment, non-finite scale */
    ATTN_ERR_UNSUPPORTED = 2,   /* a valid request this kernel does not implement (fp32, head dim, ...) */
    ATTN_ERR_CUDA = 3,          /* a CUDA runtime/driver call or the launch failed */
    ATTN_ERR_TIMEOUT = 4,       /* a bounded device-side wait gave up (status word, see below) */
    ATTN_ERR_CHECK = 5          /* debug builds only: a device-side index or range check failed */
} attn_status_t;

typedef enum {
    ATTN_F16 = 0,
    ATTN_BF16 = 1,
    ATTN_F32 = 2,               /* accepted by the type only so that it can be rejected (UNSUPPORTED) */
    ATTN_E4M3 = 3               /* 8-bit float e4m3, finite variant (max 448): attn_fwd_fp8 inputs only */
} attn_dtype_t;

/*
 * A strided view of a device tensor.  shape and stride are in ELEMENTS, outer
 * to inner; only the first `ndim` entries are read.  Q, O and the gate are 4-D
 * [B, H, N, d], K and V [B, H, Nk, d]; the innermost stride must be 1 and every other stride
 * times the element size must be a multiple of 16 bytes, and `data` must be
 * 16-byte aligned (tensor-memory-accelerator copies need both).
 */
typedef struct {
    void* data;
    attn_dtype_t dtype;
    int32_t ndim;
    int64_t shape[4];
    int64_t stride[4];
} attn_tensor_t;

/*
 * attn_fwd -- O = softmax(scale * Q K^T [+ bias]) V [* sigmoid(G)] and lse.
 *
 *   q       [B, H, N, d]  fp16 or bf16, device memory: N query rows.
 *   k, v    [B, H, Nk, d] same dtype, B, H and d as q; Nk >= 1 key rows (Nk may
 *           differ from N: a prefill chunk or a decode step against a KV cache).
 *   bias    nullable.  Additive score bias of q's dtype, either [H, N, Nk]
 *           (shared over B, the Evoformer pair bias) or [B, H, N, Nk]; the
 *           innermost stride must be 1 and rows 16-byte aligned.
 *   gate    nullable.  [B, H, N, d] of q's dtype; O is multiplied elementwise
 *           by 1/(1+exp(-gate)) after normalisation.
 *   causal  nonzero: key j is visible to query i iff j <= i + (Nk - N), i.e. the
 *           queries are the last N positions of the Nk-long sequence (bottom-right
 *           alignment; j <= i when N == Nk).  With N > Nk the first N - Nk rows see
 *           no key and get O = 0, lse = -inf.
 *   scale   multiplies Q K^T; must be finite (0 is legal).  Callers normally
 *           pass 1/sqrt(d).
 *   out     [B, H, N, d] of q's dtype, written (fp32 accumulator rounded to
 *           nearest even).  Must not alias q, k, v, bias or gate.
 *   lse     nullable.  B*H*N contiguous fp32, row (b, h, i) at (b*H + h)*N + i,
 *           natural log.  A row with every score -inf gets O = 0, lse = -inf.
 *   stream  CUDA stream of the launch (0 = legacy default stream).
 *
 * Supported: d in {32, 64, 128}; N, Nk >= 1 (any sizes, ragged tails are
 * masked); B*H >= 1.  N == 0 or B*H == 0 returns ATTN_OK without launching;
 * Nk == 0 with N > 0 is ATTN_ERR_INVALID_ARG.
 * Errors are detected on the host before any launch and return a status with
 * no side effect: ATTN_ERR_INVALID_ARG for nulls, rank/shape/stride mismatch,
 * misalignment, aliasing of out with an input, or a non-finite scale;
 * ATTN_ERR_UNSUPPORTED for fp32, mixed dtypes, or d outside {32, 64, 128};
 * ATTN_ERR_CUDA if the launch fails.
 */
attn_status_t attn_fwd(const attn_tensor_t* q, const attn_tensor_t* k, const attn_tensor_t* v,
                       const attn_tensor_t* bias, const attn_tensor_t* gate,
                       int causal, float scale,
                       attn_tensor_t* out, float* lse,
                       cudaStream_t stream);

/*
 * Optional score modifications (attention variants the pages list), applied
 * after scale and bias, in this order, to the score s of query i and key j:
 *   alibi_slopes  nullable; device fp32 [H]: s -= slope_h * |i + (Nk - N) - j|
 *   softcap       > 0: s <- softcap * tanh(s / softcap); 0 turns it off
 *   window_left   >= 0: keys j < i + (Nk - N) - window_left are masked (a left
 *                 sliding window; with causal masking a band of window_left + 1
 *                 keys); negative turns it off
 * With a window, the key tiles wholly left of the window of a 256-row unit's
 * first row are skipped; the tiles the window's edge cuts are masked.
 */
typedef struct {
    const float* alibi_slopes;
    float softcap;
    int32_t window_left;
} attn_mods_t;

/*
 * attn_fwd_ex -- attn_fwd with score modifications (`mods` nullable: none).
 * Errors as attn_fwd, plus ATTN_ERR_INVALID_ARG for a negative or non-finite
 * softcap or a misaligned alibi_slopes, and ATTN_ERR_UNSUPPORTED for a
 * modification together with a bias or a gate.  attn_fwd(...) is
 * attn_fwd_ex(..., NULL, ...).
 */
attn_status_t attn_fwd_ex(const attn_tensor_t* q, const attn_tensor_t* k, const attn_tensor_t* v,
                          const attn_tensor_t* bias, const attn_tensor_t* gate, int causal, float scale,
                          const attn_mods_t* mods, attn_tensor_t* out, float* lse, cudaStream_t stream);

/*
 * attn_fwd_varlen -- a batch of sequences of different lengths, packed along
 * the token axis (each sequence is its own attention problem; no token attends
 * across a sequence boundary).
 *
 *   q, out     [Tq, H, d] device views; sequence b owns rows
 *              cu_seqlens_q[b] .. cu_seqlens_q[b+1]
 *   k, v       [Tk, H, d]; sequence b owns rows cu_seqlens_k[b] .. cu_seqlens_k[b+1]
 *   cu_seqlens_q, cu_seqlens_k
 *              HOST int32 arrays of batch + 1 non-decreasing offsets, starting
 *              at 0 and ending at Tq (resp. Tk)
 *   causal     per sequence, aligned at the bottom right as in attn_fwd
 *   lse        nullable; [H, Tq] fp32, row (h, t) at h * Tq + t
 *
 * Layout rules as attn_fwd (unit inner stride, other strides multiples of 16
 * bytes, 16-byte aligned data).  A sequence with no query rows is skipped; one
 * with query rows but no key rows is ATTN_ERR_INVALID_ARG.  The packed out
 * must not overlap q, k or v anywhere (not only within one sequence), and lse's
 * H*Tq floats must not overlap any of the four: ATTN_ERR_INVALID_ARG.  Every
 * sequence is checked before the first launch.  The fused kernel runs once per
 * 64 non-empty sequences (one launch for batches of up to 64): the sequences'
 * sizes and offsets travel in the kernel's parameters, heaviest sequences first,
 * and every CTA of the persistent grid takes units of any sequence.  Tiles are
 * read through one tensor map over the packed tensors, so a tile that runs past
 * its sequence's end reads the next sequence's rows: such keys get weight
 * exactly 0 and such query rows are never stored, but a non-finite value in a
 * neighbouring sequence's V is multiplied by that zero (as it would be within
 * one sequence).
 */
attn_status_t attn_fwd_varlen(const attn_tensor_t* q, const attn_tensor_t* k, const attn_tensor_t* v,
                              const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int32_t batch, int causal,
                              float scale, attn_tensor_t* out, float* lse, cudaStream_t stream);

/*
 * attn_fwd_host -- the same operation end to end from HOST memory.
 *
 *   q, k, v, bias?, gate?   views of the inputs in host memory (layout rules of
 *                           attn_fwd, except that they need not be device memory)
 *   out, lse?               host destinations of O and lse (lse: B*H*N fp32)
 *   q_dev ... out_dev, lse_dev
 *                           caller-owned DEVICE staging buffers: each view has the
 *                           dtype, shape and strides of its host counterpart; bias_dev
 *                           / gate_dev / lse_dev are NULL exactly when bias / gate /
 *                           lse are.
 *
 * Enqueued on `stream`, in order: one cudaMemcpyAsync per input (the span from
 * its first to one past its last element) host -> device, attn_fwd on the
 * staging views, then O and lse device -> host.  Returns once all of it is
 * enqueued; the host results are valid once `stream` reaches the end of the
 * call.  Host buffers should be page-locked (cudaHostAlloc, cudaHostRegister)
 * so that the copies are asynchronous: calls on separate streams with separate
 * staging buffers then run one problem's copies under another's kernel.  The
 * library allocates nothing.  Errors: every check of attn_fwd applies to the
 * staging views, a host view whose dtype, shape or strides differ from its
 * staging view (or a NULL that does not match) is ATTN_ERR_INVALID_ARG, all
 * before any copy is enqueued; ATTN_ERR_CUDA if a copy or the launch fails
 * (earlier copies of the call may then already be enqueued).
 */
attn_status_t attn_fwd_host(const attn_tensor_t* q, const attn_tensor_t* k, const attn_tensor_t* v,
                            const attn_tensor_t* bias, const attn_tensor_t* gate, int causal, float scale,
                            attn_tensor_t* out, float* lse,
                            const attn_tensor_t* q_dev, const attn_tensor_t* k_dev, const attn_tensor_t* v_dev,
                            const attn_tensor_t* bias_dev, const attn_tensor_t* gate_dev,
                            attn_tensor_t* out_dev, float* lse_dev, cudaStream_t stream);

/*
 * attn_fwd_host_ex -- attn_fwd_host with score modifications (`mods` nullable:
 * none), applied as attn_fwd_ex applies them.  mods->alibi_slopes, when given,
 * points to DEVICE memory (H fp32), like the staging buffers; it is read by the
 * kernel, not copied.  The checks of attn_fwd_ex's mods run with the others,
 * before any copy is enqueued.  attn_fwd_host(...) is attn_fwd_host_ex with
 * mods = NULL.
 */
attn_status_t attn_fwd_host_ex(const attn_tensor_t* q, const attn_tensor_t* k, const attn_tensor_t* v,
                               const attn_tensor_t* bias, const attn_tensor_t* gate, int causal, float scale,
                               const attn_mods_t* mods, attn_tensor_t* out, float* lse,
                               const attn_tensor_t* q_dev, const attn_tensor_t* k_dev, const attn_tensor_t* v_dev,
                               const attn_tensor_t* bias_dev, const attn_tensor_t* gate_dev,
                               attn_tensor_t* out_dev, float* lse_dev, cudaStream_t stream);

/*
 * attn_bwd -- gradients of attn_fwd (without bias or gate) for an upstream dO:
 *
 *     P  = exp(scale Q K^T - lse)  (masked as in the forward)
 *     dV = P^T dO,  dS = P * (dO V^T - D),  D_i = sum_c dO_ic O_ic
 *     dQ = scale dS K,  dK = scale dS^T Q
 *
 * (the derivatives of the forward's definition; S and P are recomputed tile by
 * tile from Q, K and the forward's lse, as the recomputation section of
 * aiinarabic.com "flash-attention" describes, and never stored).
 *
 *   q, k, v, causal, scale   exactly as given to attn_fwd
 *   out, lse                 attn_fwd's O [B, H, N, d] and lse (B*H*N fp32, required)
 *   dout                     upstream gradient, O's shape and dtype
 *   dq                       [B, H, N, d], written; dk, dv [B, H, Nk, d], written
 *                            (fp32 accumulation, rounded to nearest-even into
 *                            the dtype); none may overlap an input or another.
 *
 * Layout rules and errors as attn_fwd; additionally ATTN_ERR_INVALID_ARG for a
 * missing lse, dout, dq, dk or dv, a shape mismatch or an overlap (lse's
 * B*H*N floats included: they must not overlap dq, dk or dv), and
 * ATTN_ERR_UNSUPPORTED for B*H > 65535.  Asynchronous on `stream`, three kernel
 * launches on the tensor cores: D_i (written as an fp32 into the first bytes of
 * dq's row i, which the last launch then overwrites with dQ), dK/dV (one CTA per
 * 128 keys), dQ (one CTA per 128 queries); no atomics, allocates nothing.
 */
attn_status_t attn_bwd(const attn_tensor_t* q, const attn_tensor_t* k, const attn_tensor_t* v,
                       const attn_tensor_t* out, const float* lse, const attn_tensor_t* dout, int causal,
                       float scale, attn_tensor_t* dq, attn_tensor_t* dk, attn_tensor_t* dv,
                       cudaStream_t stream);

/* A static, NUL-terminated description of a status code (never NULL). */
const char* attn_status_string(attn_status_t status);

/*
 * attn_last_device_status -- reads and clears the device status word of the
 * current device in one atomic exchange enqueued on `stream` (after the kernels
 * already enqueued there), then synchronises `stream`.  Kernels bound every
 * wait on an mbarrier; a wait that gives up records ATTN_ERR_TIMEOUT there
 * (and the kernel returns without hanging).  The word is DEVICE-WIDE: every
 * launch of the library on that device, on any stream, shares it.  A timeout
 * of a kernel still running on another stream may therefore be reported by
 * this call, or by a later one, instead of the caller whose launch it was;
 * callers that run the library on several streams and need per-call status
 * must serialise their reads.  Returns ATTN_OK, ATTN_ERR_TIMEOUT, ATTN_ERR_CHECK
 * (a debug build's device-side index or range check failed; see
 * attn_build_flags), or ATTN_ERR_CUDA if the exchange, the read or the
 * synchronisation failed.
 */
attn_status_t attn_last_device_status(cudaStream_t stream);

/*
 * attn_set_wait_limit -- sets the clock-cycle budget of every bounded device
 * wait for later launches, process-wide (default 2^32 cycles, about two
 * seconds at 1.9 GHz).  Values below 1024 are raised to 1024.  A wait whose
 * phase completes returns as soon as it does; the budget only bounds waits
 * that would otherwise never end (see attn_debug_inject_stall).  Not
 * thread-safe with concurrent attn_fwd calls.
 */
void attn_set_wait_limit(uint64_t cycles);

/*
 * attn_debug_inject_stall -- test hook for failure detection without a GPU
 * fault.  While enabled, every later launch on any device makes its MMA warp
 * first wait on a barrier that nothing arrives on; the bounded wait gives up
 * after the wait limit (attn_set_wait_limit), records ATTN_ERR_TIMEOUT in the
 * status word, and every role of the kernel stops, drains its in-flight copies
 * and MMAs and returns (outputs are then undefined).  Not thread-safe with
 * concurrent attn_fwd calls.  enable = 0 turns it off.
 */
void attn_debug_inject_stall(int enable);

/*
 * attn_fwd_fp8 -- the forward on 8-bit (e4m3) inputs with per-tensor scales: the
 * low-precision variant of hamidun.com's FlashAttention-3 article (the FP8
 * section: about twice the 16-bit throughput, error close to plain FP8
 * attention).  The page fixes no format or scaling rule; the readings taken:
 *
 *   element x of q, k or v_t stands for decode_e4m3(x) * that tensor's scale;
 *   O and lse are those of attn_fwd's exact operation on those values; the
 *   kernel's one added rounding is P's: each p (relative to the running row
 *   maximum, at most 2^8) is rounded to e4m3 (nearest even, saturating) before
 *   P V runs on the 8-bit tensor core, while the row sum l adds the unrounded p.
 *   Per output element the result then differs from the exact one by at most
 *   sum_j max(2^-4 p_ij, 2^-10) |v_jc| / l_i (p against the row maximum), plus
 *   out's own rounding.
 *
 *   q        [B, H, N, d]  e4m3 codes (ATTN_E4M3), device memory; d in {64, 128}.
 *   k        [B, H, Nk, d] e4m3.
 *   v_t      V TRANSPOSED: [B, H, d, Nk] e4m3 (both tensor-core operands of P V are
 *            then read along the key axis).
 *   q_scale, k_scale, v_scale   finite, > 0.
 *   causal, scale               as attn_fwd (scale multiplies the decoded, scaled
 *                               Q K^T; q_scale * k_scale * scale is folded into one
 *                               factor, v_scale into the epilogue).
 *   out      [B, H, N, d] fp16 or bf16 (the output type).
 *   lse      nullable; [B, H, N] fp32 as attn_fwd.
 *
 * Layout: inner stride 1; every other stride a multiple of 16 elements (bytes for
 * the e4m3 tensors); 16-byte aligned data.  No bias, gate or score modification.
 * ATTN_ERR_UNSUPPORTED for non-e4m3 inputs, another d or an out dtype other than
 * fp16/bf16; ATTN_ERR_INVALID_ARG for nulls, shape mismatches, a non-finite or
 * non-positive scale, misalignment, or out overlapping an input.  Asynchronous on
 * `stream`; allocates nothing.
 */
attn_status_t attn_fwd_fp8(const attn_tensor_t* q, const attn_tensor_t* k, const attn_tensor_t* v_t, float q_scale,
                           float k_scale, float v_scale, int causal, float scale, attn_tensor_t* out, float* lse,
                           cudaStream_t stream);

/*
 * attn_debug_exp2 -- test hook: evaluates, on the device, one of the base-2
 * exponentials the forward kernel's softmax uses, so that each can be checked
 * against the exact value and against CUDA's exp2f.  Not part of the
 * attention computation (the pages define no such call).
 *
 *   x, y    device float arrays of n elements (4-byte aligned); y[i] = 2^x[i].
 *           Elements are taken in pairs (2t, 2t + 1), as the softmax does.
 *   mode    ATTN_EXP2_FMA_PIPE: the kernel's FMA-pipe 2^x (range reduction with a
 *           round-down add, a cubic for 2^f on [0, 1), the integer part added to
 *           the exponent field).  Stated bound: relative error <= 7.5e-5 for
 *           x in (-126, 8]; x <= -126 gives a value <= 2^-126 (flushed later).
 *           ATTN_EXP2_MUFU: ex2.approx.ftz.f32 on the special-function unit.
 *           ATTN_EXP2_CUDA_EXP2F: CUDA's exp2f (the comparison reference).
 *
 * Returns ATTN_ERR_INVALID_ARG for n < 0, an unknown mode, or (n > 0) a null or
 * misaligned pointer; ATTN_ERR_CUDA if the launch fails.  Asynchronous on
 * `stream`; allocates nothing.
 */
enum { ATTN_EXP2_FMA_PIPE = 0, ATTN_EXP2_MUFU = 1, ATTN_EXP2_CUDA_EXP2F = 2 };
attn_status_t attn_debug_exp2(const float* x, float* y, int64_t n, int mode, cudaStream_t stream);

/*
 * attn_build_flags -- how this library was built.  ATTN_BUILD_DEBUG_CHECKS: the
 * debug build (libattn_debug.so, compiled with -DATTN_DEBUG=1).  Its kernels check
 * the indices and ranges they derive (the work-unit decode, tile coordinates and
 * their 16-byte alignment, the tensor-memory allocation, output rows) and record a
 * failure in the device status word (ATTN_ERR_CHECK from attn_last_device_status)
 * instead of faulting; results are otherwise the release build's.
 */
enum { ATTN_BUILD_DEBUG_CHECKS = 1 };
int attn_build_flags(void);

/* The library version as "major.minor.patch" (static string). */
const char* attn_version(void);


/*
 * attn_bwd_ex -- attn_bwd for a forward run with score modifications (`mods` as given to
 * attn_fwd_ex; nullable: none).  The softcap's derivative 1 - tanh(s / c)^2 enters dS; the ALiBi
 * shift and the window mask only change P.  Errors as attn_bwd, plus those of attn_fwd_ex's mods.
 */
attn_status_t attn_bwd_ex(const attn_tensor_t* q, const attn_tensor_t* k, const attn_tensor_t* v,
                          const attn_tensor_t* out, const float* lse, const attn_tensor_t* dout, int causal,
                          float scale, const attn_mods_t* mods, attn_tensor_t* dq, attn_tensor_t* dk,
                          attn_tensor_t* dv, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_ATTN_H_ */
