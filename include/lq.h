/*
 * lq.h -- C ABI of the LiftQuant lift-then-project layer on NVIDIA B200 (sm_100a).
 *
 * The layer (LiftQuant: Continuous Bit-Width LLM via Dimensional Lifting and
 * Projection, ICML 2026; paper note "Key designs" 1, 3 and 4) computes
 *
 *     o = diag(s) . W_q . (blockdiag(M^T) . T^{-1} . a)
 *
 * with W_q in {+-1}^{out x K} stored as packed sign bits, M in R^{d x D} the
 * global projection, T^{-1} the per-layer whitening inverse and
 * K = (in/d)*D rounded up to a multiple of 32, so the weight bit-width is D/d.
 *
 * Conventions shared by every call
 *  - All tensor pointers are caller-owned DEVICE memory (lq_lift_gemv's `a`
 *    and `o` may also be mapped page-locked host memory), 16-byte aligned,
 *    densely packed row-major; the compute calls check this with
 *    cudaPointerGetAttributes and refuse host memory with LQ_ERR_INVALID_ARG.
 *    The library frees nothing and keeps no pointer.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream). Calls are
 *    stream-ordered and asynchronous: they return after enqueueing work.
 *  - Argument checks are synchronous and happen before any launch; a call
 *    that fails them launches nothing and returns LQ_ERR_INVALID_ARG.
 *  - No output may share a byte with an input or another output of the same
 *    call (in-place calls are refused): the checks compare the byte ranges
 *    that the pointers and the sizes in the arguments imply (for a workspace,
 *    the bytes the shape needs). Inputs may overlap one another.
 *  - A failed launch returns LQ_ERR_CUDA. Errors detected on the device
 *    (a bounded wait that ran out; in the debug build, an index outside its
 *    buffer) are latched on the device and read by lq_get_device_status().
 *  - Debug build: liblq_debug.so, the same entry points compiled with
 *    -DLQ_DEBUG. Its kernels test the element index of each computed global
 *    load and store of the pack, lift, Kronecker lift, prefill GEMM and
 *    encoder kernels against the extent of its buffer (from the call's
 *    arguments) before the access; a failed test skips the access and latches
 *    LQ_ERR_BOUNDS. Nothing traps. TMA copies are bounded by their tensor maps
 *    in both builds. The release library compiles the tests away.
 *  - Packed signs: 32 per uint32, least significant bit first along the
 *    lifted axis, bit 1 = +1, row-major [out][K/32].
 *  - Fault injection for error-path tests (host side only): with the
 *    environment variable LQ_FAULT=launch every compute call returns
 *    LQ_ERR_CUDA after its argument checks, without launching; with
 *    LQ_FAULT=timeout lq_get_device_status returns LQ_ERR_TIMEOUT without
 *    touching the device.
 *  - bf16 values are passed as their uint16 bit patterns.
 */
#ifndef LQ_H
#define LQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LQ_API __attribute__((visibility("default")))
#else
#define LQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LQ_OK = 0,
    LQ_ERR_INVALID_ARG = 1,  /* bad pointer, size, alignment or dtype; nothing launched */
    LQ_ERR_UNSUPPORTED = 2,  /* valid but not supported on this device (needs sm_100) */
    LQ_ERR_CUDA = 3,         /* a CUDA runtime call or kernel launch failed */
    LQ_ERR_TIMEOUT = 4,      /* a device-side bounded wait expired (from lq_get_device_status) */
    LQ_ERR_TOO_LARGE = 5,    /* the shape needs more scratch than lq_gemv_noalloc's fixed array holds */
    LQ_ERR_BOUNDS = 6        /* debug build: a kernel skipped an access outside its buffer (from lq_get_device_status) */
} lq_status;

typedef enum { LQ_F32 = 0, LQ_BF16 = 1 } lq_dtype;

/* Human-readable name of a status code; never NULL. */
LQ_API const char* lq_status_str(int status);

/* Lifted width K = (in/d)*D rounded up to a multiple of 32 (storage of D sign
 * bits per d weights, "Key designs" 1). Returns -1 if d does not divide in or
 * an argument is not positive or the result overflows int. Host only. */
LQ_API int lq_lifted_dim(int in, int d, int D);

/* Pack +-1 signs into words (the 1-bit W_q of "Key designs" 4).
 *   signs_pm1 : int8 [out][K], each +1 or -1 (any value > 0 packs as 1)
 *   out >= 1, K >= 32 and K % 32 == 0
 *   packed    : uint32 [out][K/32] (written)
 * Bit-exact. */
LQ_API int lq_pack_signs(const int8_t* signs_pm1, int out, int K, uint32_t* packed, void* stream);

/* Inverse of lq_pack_signs: words -> int8 +-1 [out][K]. Bit-exact. */
LQ_API int lq_unpack_signs(const uint32_t* packed, int out, int K, int8_t* signs_pm1, void* stream);

/* Encoder, the offline step that produces W_q ("Key designs" 2): each block w
 * of d consecutive weights of a row gets the sign pattern y in {+-1}^D whose
 * codeword M y is (approximately) nearest, found as the page describes -- a
 * pseudo-inverse start plus a search over an auxiliary vector that cuts the
 * 2^D patterns to 2^{D-d}:
 *   candidate 0:     y = sign(M^+ w), M^+ = M^T (M M^T)^{-1};
 *   candidate 1 + p: the first D-d coordinates are the pattern p (bit a set
 *                    <=> +1), the last d are sign(M_B^{-1} (w - M_A z)) with
 *                    M_A, M_B the first D-d and last d columns of M;
 *   sign(0) = +1; the smallest ||w - M y||^2 wins, the earliest on ties.
 *   w      : fp32 [rows][in] (the weights to encode, already scaled/whitened)
 *   M      : fp32 [d][D]; 1 <= d <= 24, d <= D <= 63, D - d <= 24, in % d == 0
 *   packed : uint32 [rows][K/32] (written, the layout lq_gemv reads: block b of
 *            a row occupies bits [b*D, (b+1)*D) of the lifted axis; padding 0)
 *   K      : must equal lq_lifted_dim(in, d, D)
 *   err    : fp32 [rows][in/d] squared errors ||w_blk - M y||^2, or NULL
 * The search runs in float64 (its result is an integer code). If M M^T or M_B
 * is singular every pattern is written as 0 and every err as NaN. Cost grows as
 * 2^{D-d} per block. Requires an sm_100 device (else LQ_ERR_UNSUPPORTED). */
LQ_API int lq_encode(const float* w, int rows, int in, const float* M, int d, int D,
                     uint32_t* packed, int K, float* err, void* stream);

/* Activation lift u = blockdiag(M^T) . T^{-1} . a  (the small matmul T* a
 * computed once before the 1-bit matmul, "Key designs" 4; T on the activation
 * side, "Key designs" 3).
 *   a      : [batch][in], a_dtype LQ_F32 or LQ_BF16
 *   tinv   : fp32 [in/tblk][tblk][tblk], block-diagonal T^{-1}, block b maps
 *            channels [b*tblk, (b+1)*tblk); NULL means T = identity (tblk ignored)
 *            1 <= tblk <= 256, in % tblk == 0
 *   M      : fp32 [d][D]; in % d == 0, 1 <= d <= 64, 1 <= D <= 256, d*D <= 4096
 *   u      : [batch][K] written in u_dtype: LQ_F32 (decode) or LQ_BF16 (prefill,
 *            round to nearest even); u[c][b*D + j] = sum_i M[i][j] a'[c][b*d + i]
 *            with a' = T^{-1} a; entries at (in/d)*D .. K-1 are written as 0
 *   K      : must equal lq_lifted_dim(in, d, D); batch >= 1
 * Accumulation is fp32. For bf16 activations with 128-wide whitening blocks and
 * at least 64 tokens the whitening runs on the tensor cores with T^{-1} split
 * into three bf16 parts (24 significant bits, fp32 accumulation): the same
 * accuracy class as the fp32 kernels. Bounded waits inside that kernel report
 * LQ_ERR_TIMEOUT through lq_get_device_status. The decode kernel is launched as
 * a programmatic dependent of the preceding kernel on the stream: it may read
 * tinv and M before that kernel completes (so that this overlaps it), and waits
 * for it before reading a. Do not let the preceding kernel write tinv or M.
 * Every pointer must be device memory. Requires an sm_100 device (else
 * LQ_ERR_UNSUPPORTED). */
LQ_API int lq_lift_activations(const void* a, int a_dtype, int batch, int in,
                        const float* tinv, int tblk,
                        const float* M, int d, int D,
                        void* u, int u_dtype, int K, void* stream);

/* Activation lift with the Kronecker-factored whitening of "Key designs" 3:
 * T = diag(s1) (P1 kron P2) diag(s2) with s2 constant over each d-block, so
 *   a' = T^{-1} a = diag(r2) (Q1 kron Q2) diag(r1) a,  r = 1/s, Q = P^{-1},
 * and then u as in lq_lift_activations (s2 is thereby folded into the lift).
 * The caller hands over the factors of T^{-1}; nothing is inverted here.
 *   a      : [batch][in], a_dtype LQ_F32 or LQ_BF16; in = n1 * n2 <= 16384
 *   r1     : fp32 [in] (1/s1), or NULL for ones
 *   q1     : fp32 [n1][n1] (P1^{-1}), 1 <= n1 <= 256
 *   q2     : fp32 [n2][n2] (P2^{-1}), 1 <= n2 <= 128
 *   r2     : fp32 [in/d] (1/s2 of each d-block), or NULL for ones
 *   M, d, D, u, u_dtype, K : as lq_lift_activations (in % d == 0)
 * Kronecker entry ((i1, i2), (j1, j2)) is q1[i1][j1] * q2[i2][j2] with channel
 * i = i1 * n2 + i2, so for one token, X = a reshaped row-major to n1 x n2,
 * (Q1 kron Q2) x = Q1 X Q2^T: in * (n1 + n2) multiply-adds per token.
 * Two implementations, chosen by shape:
 *  - Prefill on the tensor cores: bf16 a and u, batch >= 64, 8 <= n1 <= 64,
 *    16 <= n2 <= 128 a multiple of 16, d <= 16 dividing n2, D >= 2 d a
 *    multiple of 4. Z = (r1 o X) Q2^T over all tokens, then Q1 Z per token,
 *    with the fp32 factors and Z split into three bf16 parts (24 significant
 *    bits, fp32 accumulation: the accuracy class of fp32 arithmetic), then
 *    the lift on the CUDA cores. Z of token t is kept in row t of u until the
 *    lift of t overwrites it, so u must not alias a. Bounded waits inside
 *    report LQ_ERR_TIMEOUT through lq_get_device_status.
 *  - Otherwise (decode batches, fp32 a or u, other factor sizes): fp32
 *    throughout, computed as (Q1 X) Q2^T with each CTA owning a slice of rows
 *    of the result, no scratch memory and no exchange between CTAs; shapes
 *    whose shared-memory plan does not fit (e.g. a large odd n1) return
 *    LQ_ERR_INVALID_ARG.
 * Launched as a programmatic dependent of the preceding kernel; it reads a
 * only after that kernel completes. Requires an sm_100 device (else
 * LQ_ERR_UNSUPPORTED). */
LQ_API int lq_lift_activations_kron(const void* a, int a_dtype, int batch, int in,
                                    const float* r1, const float* q1, int n1, const float* q2, int n2,
                                    const float* r2, const float* M, int d, int D,
                                    void* u, int u_dtype, int K, void* stream);

/* Workspace bytes lq_gemv and lq_lift_gemv need for (out, K, batch); 0 if the
 * arguments are invalid or no launch plan fits the shape. Host only; the size
 * depends on the device's SM count only through the plan, so query it on the
 * device that will run the call. */
LQ_API size_t lq_gemv_workspace_size(int out, int K, int batch);

/* Decode 1-bit GEMV, batch 1..16 (the +-1 by float matmul of "Key designs" 4):
 *   o[c][r] = s[r] * sum_k sigma[r][k] * u[c][k],  sigma = +1 if bit set else -1
 *   packed : uint32 [out][K/32]; s : fp32 [out]; u : fp32 [batch][K]
 *   o      : fp32 [batch][out] (written)
 *   out >= 1, K >= 32, K % 32 == 0, 1 <= batch <= 16
 *   workspace : caller-owned device scratch of at least
 *               lq_gemv_workspace_size(out, K, batch) bytes, 256-byte aligned;
 *               its contents need no initialization and are overwritten.
 * Arithmetic: one or two columns (three below 40 MB of packed weights) run on
 * mma.sync, which converts each
 * column of u (over the K range of each launch) to 32-bit fixed point with one
 * power-of-two scale -- an element's error is at most 2^-31 of the largest |u|
 * of its column and range -- and contracts the signs in exact integer
 * arithmetic; the result is within ~1e-7 relative (Frobenius) of the exact
 * value, and equal to it when u holds small integers. More columns run on
 * tcgen05 block-scaled 4-bit MMAs, which read every weight once for all
 * columns: u is converted once per call into the workspace, each 32-element
 * block with its own power-of-two scale to 21 bits (7 base-8 digits, error at
 * most 2^-21 of the block's largest |u|), accumulated in fp32 (~1e-6 relative).
 * Non-finite activations propagate as in an exact IEEE sum: a column holding
 * a NaN gives NaN; a column holding +-Inf gives, per row, +-Inf or NaN by the
 * signs of its Inf terms.
 * Deterministic. Calls that share a workspace must be
 * ordered (the same stream): overlapping calls race on it. Every pointer must
 * be device memory. Launch order: the call's first kernel is a programmatic
 * dependent of the preceding kernel on the stream. With four or more columns
 * (and three from 40 MB of packed weights) that first kernel is the quantizer
 * of u, which waits for the preceding kernel before it reads anything, so no
 * read of the call can overlap it. With one to three columns on the mma.sync
 * kernel, packed and s may be read before the preceding kernel completes, when
 * that kernel lets its dependents start early (this library's lift kernels
 * do); u is read only after it completes. So the preceding kernel must not
 * write packed or s. Requires an sm_100 device (else LQ_ERR_UNSUPPORTED). */
LQ_API int lq_gemv(const uint32_t* packed, const float* s, int out, int K,
            const float* u, int batch, float* o, void* workspace, size_t workspace_bytes, void* stream);

/* Decode step in one call: lq_lift_activations followed by lq_gemv (the small
 * matmul T* a, then the 1-bit x float matmul and diag(s) -- "Key designs" 4),
 * with the arguments of both calls:
 *   a, a_dtype, batch, in, tinv, tblk, M, d, D, K : as lq_lift_activations
 *   packed, s, out, workspace, workspace_bytes     : as lq_gemv
 *   u : fp32 [batch][K] (written: the lifted activations)
 *   o : fp32 [batch][out] (written); 1 <= batch <= 16
 * Results are exactly those of the two calls; the kernels are chained as
 * programmatic dependents, so each one's setup overlaps the one before.
 * Zero-copy decode: `a` and `o` (only these two) may instead be page-locked
 * host memory that the device addresses at the same pointer (with unified
 * addressing, any cudaHostAlloc / cudaMallocHost buffer). The lift then loads
 * the activations, and the GEMV stores the outputs, across the host link
 * itself, so a step from host buffers needs no separate copies; the results
 * are identical. The call checks every pointer with cudaPointerGetAttributes
 * and returns LQ_ERR_INVALID_ARG for pageable or unmapped host memory (and for
 * host memory anywhere but `a` and `o`). The host must not touch `a` or `o`
 * until the stream has passed the call. Requires an sm_100 device (else
 * LQ_ERR_UNSUPPORTED). */
LQ_API int lq_lift_gemv(const void* a, int a_dtype, int batch, int in, const float* tinv, int tblk,
                        const float* M, int d, int D, const uint32_t* packed, const float* s, int out, int K,
                        float* u, float* o, void* workspace, size_t workspace_bytes, void* stream);

/* Decode GEMV that allocates nothing: lq_gemv with the same arguments and the
 * same results, minus the workspace. (The paper has no counterpart; this is a
 * service of the library.) Some callers cannot call cudaMalloc or own scratch
 * buffers: code that runs while a stream is being captured into a CUDA graph
 * (allocation there is not allowed or would be baked into the graph), serving
 * loops whose memory pool is fixed up front and may not grow (cudaMalloc can
 * also synchronize the device, stalling every stream), and plug-ins or hooks
 * that only receive tensors from their host framework. For them the scratch
 * lives in a fixed device array of LQ_GEMV_NOALLOC_SCRATCH_BYTES inside the
 * library, which every GPU that loads the library keeps until the process
 * exits.
 *   Sizes: shapes whose lq_gemv_workspace_size exceeds that array return
 *   LQ_ERR_TOO_LARGE before any launch (every configured decode layer fits at
 *   batches up to eight; the widest batches of large layers need lq_gemv).
 *   Sharing: every call on a device uses the same array, and the array keeps
 *   the previous call's contents (each call rewrites all it reads, so nothing
 *   needs clearing). Calls that can overlap on the GPU -- on different streams
 *   without ordering, or from several host threads -- race on it: issue them in
 *   one stream order.
 *   Set-up: the first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before capturing any stream.
 *   Allocation: none (no cudaMalloc, cudaFree or allocating library routine).
 * Requires an sm_100 device (else LQ_ERR_UNSUPPORTED). */
#define LQ_GEMV_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)
LQ_API int lq_gemv_noalloc(const uint32_t* packed, const float* s, int out, int K,
                           const float* u, int batch, float* o, void* stream);

/* Prefill 1-bit GEMM on the tensor cores (tcgen05, bf16 operands, fp32 accumulate):
 *   o[t][r] = s[r] * sum_k sigma[r][k] * u[t][k]
 *   packed : uint32 [out][K/32]; s : fp32 [out]; u_bf16 : bf16 bits [tokens][K]
 *   o      : fp32 [tokens][out] (written)
 *   out >= 1, K >= 32, K % 32 == 0, tokens >= 1
 * +-1 is exact in bf16 and products are exact, so the only rounding is fp32
 * accumulation. Requires an sm_100 device (else LQ_ERR_UNSUPPORTED). */
LQ_API int lq_gemm(const uint32_t* packed, const float* s, int out, int K,
            const uint16_t* u_bf16, int tokens, float* o, void* stream);

/* Self-test of the failure reporting: launches one thread that waits, through
 * the bounded-wait helper the GEMV and GEMM use, on an mbarrier that nothing
 * ever completes. After limit_us microseconds (1 .. 1000000) the wait gives up,
 * latches LQ_ERR_TIMEOUT in the device status word and the kernel returns; the
 * next lq_get_device_status reports it. Nothing faults or hangs. Requires an
 * sm_100 device (else LQ_ERR_UNSUPPORTED). */
LQ_API int lq_selftest_wait_timeout(unsigned limit_us, void* stream);

/* Self-test of the debug build's bounds reporting: launches one thread that
 * tests index 1 against an extent of 1, through the same check the kernels
 * use, with no memory access behind it. The check fails and latches
 * LQ_ERR_BOUNDS, which the next lq_get_device_status reports. Returns LQ_OK
 * after enqueueing it in the debug build, LQ_ERR_UNSUPPORTED in the release
 * build (whose kernels carry no checks) and on devices other than sm_100. */
LQ_API int lq_selftest_bounds(void* stream);

/* 1 in the debug build (liblq_debug.so), 0 in the release build. */
LQ_API int lq_is_debug_build(void);

/* Synchronizes `stream`, then reads and clears, in one atomic exchange on the
 * device, the status word of the stream's device: LQ_OK, or LQ_ERR_TIMEOUT if a
 * kernel there gave up a bounded wait since the last call. A timeout latched
 * meanwhile by a kernel on another stream is either returned or kept for the
 * next call. The debug build also reads and clears the bounds flags of the
 * device and returns LQ_ERR_BOUNDS, ahead of LQ_ERR_TIMEOUT, if any check
 * failed since the last call. Returns LQ_ERR_CUDA if a CUDA call fails. */
LQ_API int lq_get_device_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LQ_H */
