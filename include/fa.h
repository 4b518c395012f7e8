/*
 * fa.h -- C ABI of the B200 (sm_100a) exact attention forward library.
 *
 * The operation is the one the pages state as the attention problem and then
 * compute tile by tile:
 *
 *     S = scale * Q K^T,   P = softmax(S),   O = P V
 *
 * (Chapter 15 -- FlashAttention, "Standard vs Flash Attention": S = Q @ K^T,
 * P = softmax(S), O = P @ V; the FlashAttention column computes the same O
 * from tiles with an online softmax, writing O once.)  The library computes
 * it without ever writing the N x N score matrix to memory, using the online
 * softmax (running row max m, running row sum l, rescale of the accumulator
 * when the max grows; FlashAttention, Playable, EP 04) and writes O and the
 * per-row log-sum-exp exactly once (FlashAttention: Tiled & Fused, diagram:
 * "Output O written once", with the "online-softmax stats").
 *
 * Not on the pages, and fixed here: the softmax scale multiplies Q K^T before
 * the softmax; the optional causal mask keeps keys j <= i for query row i;
 * lse_i = ln(sum_j exp(scale * q_i . k_j)) over the allowed keys (natural
 * log, fp32).
 *
 * Every function is callable from C.  Pointers named "device" must point to
 * memory of the current CUDA device; nothing here allocates or frees the
 * caller's buffers.
 */
#ifndef FA_B200_FA_H
#define FA_B200_FA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FA_VERSION_MAJOR 1
#define FA_VERSION_MINOR 0
#define FA_VERSION_PATCH 0

/* Element type of q, k, v and o. */
typedef enum {
    FA_DTYPE_F32 = 0,  /* fp32 in, fp32 out; CUDA-core FFMA kernel */
    FA_DTYPE_BF16 = 1  /* bf16 in, bf16 out, fp32 accumulation; tensor-core kernel */
} fa_dtype_t;

/* Status codes returned by every entry point. */
typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARGUMENT = 1, /* bad pointer, size, alignment, aliasing, dtype or scale */
    FA_ERR_UNSUPPORTED = 2,      /* well-formed but not implemented (head dim other than 64/128) */
    FA_ERR_CUDA = 3,             /* a CUDA runtime/driver call failed; see fa_last_error() */
    FA_ERR_DEVICE_TIMEOUT = 4    /* a kernel gave up on a bounded wait (reported by fa_check_device_status) */
} fa_status_t;

/*
 * fa_fwd -- exact attention forward.
 *
 *   q, k, v  device, contiguous row-major [B][H][N][d] of `dtype` (each head's
 *            N x d matrices Q, K, V as on the "Standard vs Flash Attention"
 *            panel).  16-byte aligned.
 *   o        device, [B][H][N][d] of `dtype`, written once per row.  16-byte
 *            aligned; must not overlap q, k, v or lse.
 *   lse      device, [B][H][N] fp32, natural-log log-sum-exp of each row's
 *            scaled, masked scores.  4-byte aligned; must not overlap the others.
 *   B, H, N  batch, heads, sequence length; each >= 1.  Any N is accepted (no
 *            multiple-of-tile requirement).
 *   d        head dimension: 64 or 128 (others: FA_ERR_UNSUPPORTED).
 *   scale    any finite float; multiplies Q K^T before the softmax (use
 *            1/sqrt(d) for the usual attention).
 *   causal   0: every key is visible; non-zero: query row i sees keys j <= i.
 *   dtype    FA_DTYPE_BF16 or FA_DTYPE_F32.
 *   stream   a cudaStream_t (NULL = the legacy default stream).
 *
 * Asynchronous: the work is enqueued on `stream` and the call returns; the
 * buffers must stay valid until the stream reaches it.  Argument errors are
 * reported synchronously before any CUDA call is made, and then nothing is
 * enqueued.  A device-side timeout (a bounded wait that expired) is not seen
 * here; call fa_check_device_status after the stream has run.
 * Thread safety: concurrent calls from several host threads are allowed.
 *
 * Kernels and launch (no effect on the result): bf16 problems run a kernel
 * with one 128-row query tile per CTA or one with two, whichever finishes
 * sooner for the shape (fa_fwd_kernel_choice); both give the same bits.  The bf16 kernels are launched with
 * programmatic stream serialization: their CTAs may start setting up while
 * the previous kernel on `stream` is still running, and wait for it to
 * complete before they read or write any memory, so stream order holds.
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
           int64_t B, int64_t H, int64_t N, int64_t d,
           float scale, int causal, int dtype, void* stream);

/*
 * fa_fwd_noalloc -- fa_fwd for callers that must not allocate device memory.
 * The pages have no counterpart: this is a deployment variant of the same
 * call, not part of the method.
 *
 * fa_fwd allocates a small device workspace (status word and work-queue
 * counters) with cudaMalloc on its first call on each device.  Callers that
 * cannot allow a library to allocate -- a serving process that has already
 * reserved all GPU memory for its own pool, code running inside an
 * allocator's hooks, strict per-library memory budgets -- use this entry
 * point instead: same arguments, layouts, results and errors as fa_fwd, but
 * the scratch lives in a fixed 256-byte device array that the library
 * carries (every GPU that loads the library holds it until the process
 * exits), and no allocating routine is called.
 *
 *   - The first call on a device, with that device current, looks up the
 *     array's device address (cudaGetSymbolAddress); make that first call
 *     before any stream capture.
 *   - Each call clears the array's work-queue words on `stream` before its
 *     kernel runs.  All calls share the one array: calls whose kernels can
 *     overlap on the GPU (different streams, several host threads) race on it
 *     and give wrong results; issue them in order on one stream.
 *   - The kernels use 24 of the array's 256 bytes (a compile-time check keeps
 *     them inside it); no argument makes a call need more.
 *   - A device-side timeout of a call made here (a bounded wait that ran out;
 *     that call's o and lse are invalid) sets the array's status word, which
 *     later calls leave set: fa_noalloc_check_status (below) reports it as
 *     FA_ERR_DEVICE_TIMEOUT and clears it.  fa_check_device_status reads
 *     fa_fwd's own status word, not this one.
 *   - fp32 inputs run the fp32 kernel, which needs no scratch.
 *   - bf16 problems whose 128-row tiles all fit on the GPU at once
 *     (B * H * ceil(N / 128) <= SM count) run the one-tile kernel, the rest
 *     the two-tile kernel (fa_fwd's schedule-based choice keeps a host-side
 *     cache, which this entry point does not).
 */
int fa_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                   int64_t B, int64_t H, int64_t N, int64_t d,
                   float scale, int causal, int dtype, void* stream);

/*
 * fa_noalloc_check_status -- the status of the fa_fwd_noalloc calls made on
 * the current device since the last check.  No counterpart in the pages (it
 * belongs to the no-allocation variant above).  Synchronises `stream` (a
 * cudaStream_t), reads the no-alloc array's status word with a plain
 * device-to-host copy (nothing is allocated) and, if a kernel gave up on a
 * bounded wait, clears the word and returns FA_ERR_DEVICE_TIMEOUT (the outputs
 * of the call that timed out are invalid; the context stays usable).
 * Returns FA_OK when no timeout was recorded, FA_ERR_CUDA if a CUDA call
 * failed.  Like the calls it checks, it must not overlap another no-alloc
 * call on the GPU.
 */
int fa_noalloc_check_status(void* stream);

/*
 * fa_fwd_fp8 -- the attention forward with 8-bit float inputs.
 *
 * The pages name low precision (FP8) as the step the third FlashAttention
 * generation took on Hopper (Chapter 15 -- FlashAttention, "FlashAttention
 * Evolution", FA-3) and fix nothing more.  Computed here, per head:
 *
 *     O = softmax(scale * (descale_q Q8)(descale_k K8)^T [causal]) (descale_v V8)
 *
 * with Q8, K8, V8 in OCP E4M3 (1 sign, 4 exponent, 3 mantissa bits, bias 7,
 * largest finite 448; torch.float8_e4m3fn), Q K^T and P V on the tensor core
 * with fp32 accumulation, P rounded to E4M3 (nearest) as the operand of P V,
 * the running max and sum in fp32.  Q8 K8^T is exact in fp32 up to the
 * accumulation order; the rounding of P is the one approximation, and each
 * element of O lies within |descale_v| (2^-4 sum_j p_j |v8_j| + 2^-10
 * sum_j |v8_j| / l) (+ the bf16 rounding of O) of the exact result, p_j the
 * exact softmax weights and l = exp(lse - max_j s_j).
 *
 *   q, k, v  device, contiguous [B][H][N][d] one-byte E4M3.  16-byte aligned.
 *   o        device, [B][H][N][d] bf16, written once per row.  16-byte aligned.
 *   lse      device, [B][H][N] fp32 natural-log log-sum-exp of the scaled
 *            scores (scale * descale_q * descale_k * q8 . k8).  4-byte aligned.
 *   B, H, N  each >= 1; any N.
 *   d        128 (others: FA_ERR_UNSUPPORTED).
 *   scale, descale_q, descale_k, descale_v  finite floats; the product
 *            scale * descale_q * descale_k must stay finite in fp32.
 *   causal   as for fa_fwd.
 *
 * No output may overlap an input or the other output.  Asynchronous on
 * `stream`; argument errors are reported before any CUDA call; device-side
 * timeouts are reported by fa_check_device_status.
 */
int fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse,
               int64_t B, int64_t H, int64_t N, int64_t d, float scale,
               float descale_q, float descale_k, float descale_v, int causal, void* stream);

/*
 * fa_fwd_fp8_host -- fa_fwd_fp8 on buffers in host memory: the same
 * operation, arguments, layouts, results and errors as fa_fwd_fp8, with q, k,
 * v, o and lse allowed to be host pointers, and the same chunked pipeline of
 * copy-in, kernel and copy-out (and the same staging buffers and ordering on
 * `stream`) as fa_fwd_host.  No alignment is required.
 */
int fa_fwd_fp8_host(const void* q, const void* k, const void* v, void* o, float* lse,
                    int64_t B, int64_t H, int64_t N, int64_t d, float scale,
                    float descale_q, float descale_k, float descale_v, int causal, void* stream);

/*
 * fa_fwd_host -- fa_fwd on buffers in host memory: the same operation,
 * arguments, layouts, results and errors, but q, k, v, o and lse may be host
 * pointers (page-locked memory, e.g. from cudaHostAlloc, for the copies to
 * run asynchronously; pageable memory works but its copies are synchronous).
 * Device pointers are accepted too (copies are direction-inferred).  No
 * alignment is required.  The pages have no counterpart: this is the path a
 * caller with host-resident data uses, and the one end-to-end timings go
 * through.
 *
 * The heads are processed in chunks (about eight per call) that flow through
 * three device staging buffers and three internal streams: while one chunk
 * is copied in, the kernel runs on the previous one and the one before is
 * copied out.  The staging buffers are allocated on first use on each device
 * and grown when a call needs more; they are kept until process exit.  Work
 * starts after everything already enqueued on `stream` and `stream` waits for
 * the last copy-out, so synchronising `stream` (or fa_check_device_status)
 * makes o and lse valid on the host; the host buffers must stay valid until
 * then.  Concurrent calls on one device are serialised while they enqueue and
 * then run in order on the device.
 */
int fa_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse,
                int64_t B, int64_t H, int64_t N, int64_t d,
                float scale, int causal, int dtype, void* stream);

/*
 * fa_decode -- attention of Nq new queries over a key/value cache of Nk
 * positions: the generation step ("FlashAttention: Tiled & Fused", card "KV
 * Cache: Why Generation Speeds Up": past K and V are cached and each new
 * token computes only its own).  The same operation as fa_fwd, with queries
 * and keys of different lengths:
 *
 *   q        device, [B][H][Nq][d] of `dtype`: the new tokens' queries.
 *   k, v     device, [B][H][Nk][d] of `dtype`: the cache, the new tokens'
 *            own keys and values included as its last Nq rows.
 *   o        device, [B][H][Nq][d] of `dtype`; lse device, [B][H][Nq] fp32
 *            (natural log), each written once.
 *   causal   0: every query uses all Nk keys; non-zero: query i sits at
 *            position Nk - Nq + i and uses keys j <= Nk - Nq + i (needs
 *            Nq <= Nk).  With Nq = 1 both are the same.
 *   scale, dtype, stream: as for fa_fwd; d is 64 or 128.
 *   workspace, workspace_bytes: device scratch of at least
 *            fa_decode_workspace_bytes(B, H, Nq, Nk, d) bytes, 256-byte
 *            aligned, no initialisation needed (the call clears the part it
 *            uses as counters on `stream` first).  May be NULL when that size
 *            is 0.  Calls that may run at the same time need separate
 *            workspaces.
 *
 * The key range of each head is split into chunks that separate CTAs process
 * (partial results merged by their log-sum-exp, as the online softmax
 * merges tiles), so a single long head still uses the whole GPU.  bf16 runs
 * on the warp-level tensor-core MMA in groups of 16 queries (P rounded to
 * bf16 before P V, as in fa_fwd); fp32 on CUDA cores.  Errors and asynchrony
 * as for fa_fwd.  Alignment: q, k, v, o 16 bytes, lse 4 bytes.
 */
int fa_decode(const void* q, const void* k, const void* v, void* o, float* lse,
              int64_t B, int64_t H, int64_t Nq, int64_t Nk, int64_t d,
              float scale, int causal, int dtype,
              void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_decode_workspace_bytes -- the workspace fa_decode needs for these sizes,
 * for either dtype (the two dtypes group queries differently; the larger
 * need is returned).  0 when one CTA per head and query group suffices, or
 * for invalid sizes.  Depends only on the arguments, not on the device.
 */
size_t fa_decode_workspace_bytes(int64_t B, int64_t H, int64_t Nq, int64_t Nk, int64_t d);

/*
 * fa_bwd -- gradients of fa_fwd: given the forward's q, k, v, o and lse and
 * the gradient dout of a loss with respect to o, writes dq, dk, dv (the
 * gradient of the exact function; the pages give the forward only and name
 * training as what the method enables -- "FlashAttention: Tiled & Fused",
 * "Enabling longer contexts in training and inference"):
 *
 *   P = exp(scale * q k^T - lse) [causal],  D = rowsum(dout * o)
 *   dv = P^T dout,  dS = P * (dout v^T - D),  dq = scale dS k,  dk = scale dS^T q
 *
 *   q, k, v, o, dout  device, [B][H][N][d] bf16 (o and lse exactly as fa_fwd
 *                     wrote them); lse device [B][H][N] fp32.
 *   dq, dk, dv        device, [B][H][N][d] bf16, written once.
 *   workspace         device scratch of fa_bwd_workspace_bytes(B, H, N, d)
 *                     bytes, 16-byte aligned: per row (padded to whole
 *                     128-row blocks) D and -lse*log2(e), and an fp32
 *                     accumulator for dq ([B*H][N rounded up to 128][d]);
 *                     its contents on entry do not matter.
 *   scale, causal     as for fa_fwd; dtype must be FA_DTYPE_BF16
 *                     (FA_ERR_UNSUPPORTED otherwise); d is 64 or 128.
 * No score matrix reaches memory: P is recomputed tile by tile from lse, and
 * each of the five products runs once per tile pair.  dq is accumulated over
 * key blocks by fp32 reduce-adds whose order varies from run to run, so dq
 * is reproducible to fp32 rounding, not bit for bit (dk, dv are).
 * Asynchronous on `stream` (three kernel launches); argument errors are
 * reported before any CUDA call.  Alignment 16 bytes (lse 4).  Outputs and
 * workspace must not overlap the inputs or each other.
 */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dout, void* dq, void* dk, void* dv,
           int64_t B, int64_t H, int64_t N, int64_t d, float scale, int causal, int dtype,
           void* workspace, size_t workspace_bytes, void* stream);

/* fa_bwd_workspace_bytes -- the workspace fa_bwd needs (0 for invalid sizes,
 * including d other than 64 or 128). */
size_t fa_bwd_workspace_bytes(int64_t B, int64_t H, int64_t N, int64_t d);

/*
 * fa_merge -- combine attention results computed over disjoint key sets into
 * the result over their union, per query row:
 *     lse = ln sum_i exp(lse_i),   o = sum_i exp(lse_i - lse) o_i
 * (the online softmax's rescale -- "FlashAttention, Playable", EP 04 --
 * applied to whole partial results; the combining step of a
 * sequence-parallel forward, where each rank attends to every key chunk).
 *   o_parts    device, [parts][rows][d] of `dtype` (each part as fa_fwd or
 *              fa_decode wrote it); lse_parts device, [parts][rows] fp32.  A
 *              part with lse = -inf for a row (no usable key) adds nothing.
 *   o, lse     device, [rows][d] of `dtype` and [rows] fp32; rows with no
 *              usable key in any part get o = 0 and lse = -inf.
 *   d 64 or 128; dtype FA_DTYPE_BF16 or FA_DTYPE_F32.  Alignment 16 bytes
 *   (lse arrays 4); outputs must not overlap inputs.  Asynchronous on stream.
 */
int fa_merge(const void* o_parts, const float* lse_parts, int64_t parts, int64_t rows, int64_t d,
             void* o, float* lse, int dtype, void* stream);

/*
 * fa_check_device_status -- synchronise `stream`, then read and clear the
 * library's device status word for the current device.  Returns FA_OK,
 * FA_ERR_DEVICE_TIMEOUT when a kernel launched by this library gave up on a
 * bounded wait since the last check (its outputs are then invalid), or
 * FA_ERR_CUDA.
 */
int fa_check_device_status(void* stream);

/*
 * fa_clock_record -- a measurement aid, not part of the attention result:
 * how fast the SM clock ran while the persistent forward kernels (fa_fwd on
 * bf16, fa_fwd_fp8; not fa_fwd_noalloc) ran on the current device.  Each CTA
 * of those kernels adds, when it ends, the SM cycles it ran (clock64), the
 * global-timer nanoseconds it ran and 1 to three device counters.  This call
 * synchronises `stream`, then writes the counters to out[0] (cycles),
 * out[1] (nanoseconds) and out[2] (CTAs), and clears them when `reset` is
 * non-zero.  out[0] / out[1] is the clock in GHz averaged over the kernels'
 * running time; out[0] / out[2] the cycles of an average CTA, i.e. of a
 * launch when every CTA runs to the end.  Launches on other streams that are
 * still running may or may not be counted yet.
 *   out   host, int64_t[3], written by the call.
 * Returns FA_OK, FA_ERR_INVALID_ARGUMENT (out NULL) or FA_ERR_CUDA.
 */
int fa_clock_record(void* stream, int reset, int64_t* out);

/* The forward kernels fa_fwd can launch (see fa_fwd_kernel_choice). */
typedef enum {
    FA_KERNEL_F32 = 0,            /* fp32, CUDA cores */
    FA_KERNEL_BF16_TWO_TILE = 1,  /* bf16, two 128-row query tiles per CTA (256-row units) */
    FA_KERNEL_BF16_ONE_TILE = 2   /* bf16, one 128-row query tile per CTA */
} fa_kernel_t;

/*
 * fa_fwd_kernel_choice -- which kernel fa_fwd (and fa_fwd_host per chunk of
 * heads) launches for a problem, written to *kernel as an fa_kernel_t.  Not
 * part of the method; the choice never changes the result (the two bf16
 * kernels give the same bits), only the time.  For bf16 the library
 * simulates how the work units of each kernel would be spread over the SMs
 * (both take units from a queue in the same order, each CTA the next one
 * when it is free; a unit costs its KV blocks times a measured cycle count
 * per block) and takes the shorter schedule: the one-tile kernel when every
 * 128-row tile gets its own SM, the two-tile kernel from 8 tiles per SM on.
 *   sm_count  SMs to plan for; < 1 means the current device's (then a CUDA
 *             call is made, and FA_ERR_CUDA is possible).
 * The test hook fa_test_force_forward_kernel overrides the choice in fa_fwd
 * but not here.  Returns FA_OK, FA_ERR_INVALID_ARGUMENT, FA_ERR_UNSUPPORTED
 * (d other than 64 or 128) or FA_ERR_CUDA.
 */
int fa_fwd_kernel_choice(int64_t B, int64_t H, int64_t N, int64_t d, int causal, int dtype,
                         int sm_count, int* kernel);

/* fa_status_string -- static, never-NULL description of a status code. */
const char* fa_status_string(int status);

/*
 * fa_last_error -- description of the last failure seen by the calling host
 * thread (which argument was rejected, or the CUDA error text).  The pointer
 * stays valid until the thread's next call into the library.
 */
const char* fa_last_error(void);

/* fa_version -- MAJOR * 10000 + MINOR * 100 + PATCH of the loaded library. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_FA_H */
