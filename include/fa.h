/*
 * fa.h -- C ABI of the B200 (sm_100a) exact-attention library (libfa_b200.so).
 *
 * What the library computes is standard scaled-dot-product attention,
 *   S = scale * Q K^T  (+ causal mask),  P = softmax(S),  O = P V,
 *   L = m + ln(l)      (per-row logsumexp of the scaled, masked scores),
 * as defined on the "FlashAttention" concept note ("Definition", "How it
 * works") and in the online-softmax section of "FlashAttention v1/v2/v3/v4:
 * the librarian who never clears the desk" (eq. 1 and eq. 2).  The forward
 * never writes the N x N score matrix to memory; the backward rebuilds P
 * from L ("How it works", recomputation).
 *
 * Conventions shared by every entry point
 *  - Tensors are [B, H, N, d] row-major and contiguous (d fastest), one
 *    device allocation each, base address 16-byte aligned.  bf16 means
 *    __nv_bfloat16; e4m3 means the OCP e4m3fn byte (max 448, no infinity).
 *  - LSE tensors are [B, H, N] fp32, natural log, of scale * Q K^T.
 *  - All pointers are DEVICE pointers owned by the caller.  Nothing is
 *    allocated, freed or retained by the library.
 *  - ``stream`` is a cudaStream_t (NULL = the legacy default stream).  All
 *    calls are asynchronous on that stream.
 *  - Argument errors are returned synchronously, before any launch, and
 *    leave the outputs untouched.  Supported: d in {64, 128, 256} for the
 *    bf16 forward and backward, d = 128 for FP8; 0 <= N <=
 *    2^20; 0 <= B * H <= 2^20; scale finite and >= 0.  B * H * N == 0 is a
 *    valid empty problem: FA_OK, nothing launched.
 *  - Causal reading: with equal query and key lengths, key j is visible to
 *    query i iff j <= i.
 *  - A pipeline wait inside a kernel that exceeds ~2 s gives up: the kernel
 *    ends early and records FA_ERR_PIPELINE_TIMEOUT in a device status word
 *    that fa_get_status() reads after the caller has synchronised.
 *  - The library keeps no state besides that status word, the scratch array
 *    of fa_bwd_noalloc and per-process caches of kernel attributes; calls on
 *    different streams may overlap (except fa_bwd_noalloc calls, see there).
 */
#ifndef FA_B200_H_
#define FA_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fa_status {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,      /* null pointer, negative size, bad scale     */
  FA_ERR_UNSUPPORTED = 2,      /* unsupported d, size limit, not sm_100      */
  FA_ERR_MISALIGNED = 3,       /* a tensor base not 16-byte aligned          */
  FA_ERR_WORKSPACE = 4,        /* workspace null or smaller than required    */
  FA_ERR_LAUNCH = 5,           /* CUDA reported an error at launch           */
  FA_ERR_PIPELINE_TIMEOUT = 6, /* a bounded in-kernel wait ran out           */
  FA_ERR_NO_DEVICE = 7,        /* no CUDA device / driver entry point        */
  FA_ERR_SCRATCH_LIMIT = 8     /* fa_bwd_noalloc: problem exceeds its scratch */
} fa_status;

/*
 * Forward: O = softmax(scale * Q K^T [causal]) V and L = logsumexp per row.
 *  q, k, v : bf16 [B, H, N, d] inputs.
 *  o       : bf16 [B, H, N, d] output (O rounded to nearest even).
 *  lse     : fp32 [B, H, N] output, natural log.
 * One fused kernel: for each 128-row query tile it streams 128-row K/V tiles
 * through shared memory, keeps the score tile and the running (m, l, o) on
 * chip and divides by l once at the end ("How it works"; the lineage page,
 * "FA2 (2023)", deferred normalisation).  Causal runs skip fully masked
 * tiles.
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int N, int d, float scale, int causal, void* stream);

/*
 * Bytes of scratch fa_bwd needs for this shape (fp32 dQ accumulator
 * [B, H, N, d] plus fp32 D [B, H, N], rounded up to 256 bytes each).
 * Returns 0 for an unsupported d or a negative size.
 */
size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * Backward of the forward above for the loss sum(O * dO).
 *  q, k, v, o, dout : bf16 [B, H, N, d]; o and lse from fa_fwd on the same
 *                     inputs.
 *  lse              : fp32 [B, H, N].
 *  dq, dk, dv       : bf16 [B, H, N, d] outputs.
 *  workspace        : device scratch of at least fa_bwd_workspace_size()
 *                     bytes, 256-byte aligned; its contents on entry do not
 *                     matter.
 * P is recomputed as exp(S - L) tile by tile, never stored ("How it works",
 * recomputation; lineage page "FA1 (2022)", idea 3).  The gradient itself is
 * the textbook one: dV = P^T dO, dP = dO V^T, D = rowsum(dO o O),
 * dS = P o (dP - D), dQ = scale dS K, dK = scale dS^T Q.
 * At d = 256 there is one backward for both entry points: dK, dV per (key
 * block, head-dim half) and dQ per query block, in a fixed order; its
 * workspace is the D array only (fa_bwd_workspace_size reports that).
 */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                 const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                 float scale, int causal, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Bytes of scratch fa_bwd_deterministic needs (fp32 D [B, H, N], rounded up
 * to 256 bytes).  Returns 0 for an unsupported d or a negative size.
 */
size_t fa_bwd_deterministic_workspace_size(int B, int H, int N, int d);

/*
 * Deterministic backward: same arguments, layouts and results as fa_bwd,
 * with a workspace of at least fa_bwd_deterministic_workspace_size() bytes
 * (256-byte aligned).  dQ, dK and dV are bitwise identical from run to run
 * on the same device.  fa_bwd adds each key block's share of dQ into an fp32
 * buffer from many thread blocks, in an order that varies; here one kernel
 * produces dK and dV (one thread block per key block, as in fa_bwd) and a
 * second owns each 128-row query block, recomputes S and dP for it
 * (the same recomputation from L, "How it works") and sums dS K over the
 * key blocks in ascending order.  The extra recomputation costs two more
 * tile products per (query block, key block) pair; no dQ reductions go to
 * memory.  The pages fix only that the backward recomputes P from L; how
 * dQ is accumulated is this library's design, and this is its reproducible
 * form.
 */
fa_status fa_bwd_deterministic(const void* q, const void* k, const void* v, const void* o,
                               const void* dout, const float* lse, void* dq, void* dk, void* dv,
                               int B, int H, int N, int d, float scale, int causal,
                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * Allocation-free backward.  No counterpart in the papers: it exists for
 * callers that cannot allocate device memory themselves (code inside a host
 * framework that owns all device memory through its own pool, or a
 * latency-critical path where cudaMalloc's device synchronisation is not
 * acceptable).  Same arguments and results as fa_bwd, without the
 * workspace: the scratch is a device array built into the library, of
 * FA_BWD_NOALLOC_SCRATCH_BYTES (32 MiB), held on every GPU that loads the
 * library until the process exits.  Nothing is allocated or freed.
 *  - Problems whose fa_bwd_workspace_size() exceeds that size are rejected
 *    with FA_ERR_SCRATCH_LIMIT before any launch (at d = 128 that is
 *    B * H * N above 65,027 rows; at d = 64, above 129,055; at d = 256,
 *    whose backward needs only D, above 8,388,608).
 *  - The first call on a device looks up the array's device address on that
 *    device (cudaGetSymbolAddress); make that first call before any stream
 *    capture.  The address is remembered per device together with the
 *    CUDA context it was looked up in; after a device reset (a new primary
 *    context) the next call looks it up again.
 *  - All calls share the one array, which keeps the previous call's
 *    contents (the part that must start at zero is cleared on every call).
 *    Calls that can overlap on the GPU race on it: serialise them.
 */
#define FA_BWD_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                         int H, int N, int d, float scale, int causal, void* stream);

/*
 * FP8 block quantisation of one tensor ("the librarian" page, "FA3 -- the
 * Hopper moment", pillar 3; lineage page, "FA3 (2024)", idea 3).
 *  x      : bf16 [B, H, N, d] input.
 *  x8     : e4m3 [B, H, N, d] output codes.
 *  scales : fp32 [B, H, ceil(N / 128)] output, one per 128-row block:
 *           scale = amax / 448 (1 for an all-zero block).
 *  signs  : NULL for no rotation, else d fp32 device values in {+1, -1}:
 *           each row is first multiplied by diag(signs) H_d / sqrt(d) (H_d
 *           the Sylvester Hadamard matrix), which leaves Q K^T unchanged when
 *           applied to both Q and K with the same signs.  V is quantised
 *           with signs = NULL.
 * code = round_to_nearest_even_satfinite(fp32(x) / scale), with
 * scale = max(amax / 448, 2^-126) for a block with a nonzero entry (the
 * floor keeps the scale a normal fp32 number, so its reciprocal is finite).
 * Contract note: the random signs are an argument, not drawn from a seed
 * inside the library.  The pages ask for a random-sign Hadamard rotation but
 * name no generator; taking the signs as data lets the caller choose the
 * generator and lets a checker apply exactly the same rotation, and it keeps
 * the library free of hidden random state.  (A (rotate, seed) form is this
 * call with signs drawn by the caller from that seed.)
 */
fa_status fa_quant_fp8(const void* x, void* x8, float* scales, int B, int H, int N, int d,
                       const float* signs, void* stream);

/*
 * FP8 forward: attention on block-quantised inputs.
 *  q8, k8, v8 : e4m3 [B, H, N, d] from fa_quant_fp8.
 *  sq, sk, sv : their fp32 block scales [B, H, ceil(N / 128)].
 *  o, lse     : as in fa_fwd (bf16 O, fp32 natural-log L).
 * Both products run on the E4M3 tensor cores; the scores are dequantised
 * with sq * sk per tile pair, P is rounded to E4M3 (scaled by a power of
 * two) and V's scale is applied to the accumulator per key tile.
 */
fa_status fa_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* sq,
                     const float* sk, const float* sv, void* o, float* lse, int B, int H, int N,
                     int d, float scale, int causal, void* stream);

/*
 * Extended entry points: grouped K/V heads, a causal sliding window, ALiBi.
 *
 * Grouped K/V heads (GQA; MQA when H_kv = 1).  The librarian page lists
 * GQA/MQA as natively supported ("Cases where FlashAttention does not
 * help"); the pages give no formula, so the reading here is the usual one:
 * query head h of batch b attends with K/V head h / G of the same batch,
 * G = H / H_kv.
 *  k, v (k8, v8)   : [B, H_kv, N, d]; q, o, dout, dq : [B, H, N, d].
 *  sk, sv           : [B, H_kv, ceil(N / 128)] block scales (FP8).
 *  dk, dv           : [B, H_kv, N, d]: the sum over the group's G query
 *                     heads of each head's gradient.
 *  H_kv             : 1 <= H_kv, H a multiple of H_kv, else
 *                     FA_ERR_INVALID_ARG.
 *
 * Sliding window (the same page's list names it among the masks FA ships;
 * again no formula).  Reading: with causal = 1 and window_left = w >= 0, key
 * j is visible to query i iff i - w <= j <= i (w + 1 keys at most; w = 0
 * keeps the diagonal only).  window_left = -1 means no window.  A window
 * without causal, or window_left < -1, is FA_ERR_INVALID_ARG.  Key blocks
 * wholly outside every row's window are skipped, not masked.
 *
 * ALiBi (the same list names it; no formula).  Reading: the scaled score of
 * query i and key j gets -slope_h * |i - j| added before the softmax (natural
 * log units, one slope per query head h).  alibi_slopes: NULL for none, else
 * a device array of H fp32 slopes (finite, >= 0; 4-byte aligned, else
 * FA_ERR_MISALIGNED), read by the kernels.  The returned L includes the bias.
 *
 * H_kv = H with window_left = -1 and alibi_slopes = NULL is exactly fa_fwd /
 * fa_bwd / fa_bwd_deterministic / fa_fwd_fp8.  fa_bwd_ex takes a workspace of
 * fa_bwd_ex_workspace_size(B, H, H_kv, N, d, deterministic) bytes (256-byte
 * aligned).  In the backward a thread block per (K/V head, key block)
 * visits the query blocks of the group's query heads in turn, so dK and dV
 * are summed on chip in a fixed order.  When B * H_kv * ceil(N / 128) is too
 * small to fill the GPU (few K/V heads), the group is shared out over S
 * thread blocks (S the smallest divisor of G giving about three per SM);
 * each writes fp32 partial dK, dV to the workspace and a reduction kernel
 * adds them in split order, so the results stay reproducible.
 */
size_t fa_bwd_ex_workspace_size(int B, int H, int H_kv, int N, int d, int deterministic);
fa_status fa_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                    int H_kv, int N, int d, float scale, int causal, int window_left,
                    const float* alibi_slopes, void* stream);
fa_status fa_bwd_ex(const void* q, const void* k, const void* v, const void* o, const void* dout,
                    const float* lse, void* dq, void* dk, void* dv, int B, int H, int H_kv, int N,
                    int d, float scale, int causal, int window_left, const float* alibi_slopes,
                    int deterministic, void* workspace, size_t workspace_bytes, void* stream);
fa_status fa_fwd_fp8_ex(const void* q8, const void* k8, const void* v8, const float* sq,
                        const float* sk, const float* sv, void* o, float* lse, int B, int H,
                        int H_kv, int N, int d, float scale, int causal, int window_left,
                        const float* alibi_slopes, void* stream);

/*
 * Measurement controls (not part of the attention contract).  The softmax's
 * exp2 can run on the SFU (ex2.approx) or, for a share of the elements, as a
 * polynomial on the FMA pipe (the librarian page, "FA4 -- Blackwell's
 * asymmetry", idea 1).  Which share is fastest was chosen by measurement per
 * kernel and head dim; these knobs let a caller (the benchmark, the tests)
 * re-run that measurement.  Settings are process-wide, apply to calls made
 * after them, and are not meant to be changed while other threads launch.
 *  FA_TUNE_FWD_POLY_PAIRS   forward bf16, of every 8 score pairs: 0, 2 or 4
 *  FA_TUNE_FWD_POLY_DEGREE  forward polynomial degree: 3 or 4
 *  FA_TUNE_BWD_POLY_GROUPS  backward P phase, of every 4 column groups: 0, 1 or 2
 *  FA_TUNE_DQ_POLY_PAIRS    deterministic dQ kernel at d = 64: 0, 2 or 4
 *  FA_TUNE_FP8_POLY_PAIRS   FP8 forward, of every 8 score pairs: 0, 2 or 4
 *                           (same polynomial degree as the bf16 forward)
 *  FA_TUNE_BWD_PAIR         deterministic backward at d = 128: dK, dV from
 *                           CTA pairs sharing each product (1) or from single
 *                           CTAs (0); same results either way
 *  FA_TUNE_FWD_PERSISTENT   two-tile forward (d <= 128, bf16 and FP8): a
 *                           persistent grid of one CTA per SM walking the work
 *                           items (1) or one CTA per work item (0); by default
 *                           chosen per call (persistent except for the FP8
 *                           non-causal forward), which fa_get_tuning reports as -1; calls
 *                           with ALiBi or a polynomial exp2 share use one CTA
 *                           per item
 *  FA_TUNE_FWD_CAUSAL_GROUP causal two-tile forward: work items longest first
 *                           within groups of heads whose K and V fit in L2
 *                           together (1), or over all heads (0); by default
 *                           grouped on the persistent grid and global with one
 *                           CTA per work item, which fa_get_tuning reports as -1
 *  FA_TUNE_FWD_Q1           bf16 forward, d <= 128: one 128-row query tile per
 *                           work item with two score buffers (1), or two query
 *                           tiles per CTA (0; FA_TUNE_FWD_PERSISTENT picks which);
 *                           by default chosen per call (the one-tile kernel when
 *                           the problem has fewer pairs of query tiles than the
 *                           device has SMs), which fa_get_tuning reports as -1
 *  FA_TUNE_BWD_CAUSAL_GROUP causal backward (main and dQ kernels): CTAs ordered
 *                           longest first within groups of heads whose working
 *                           set fits in L2 (1), or head by head (0)
 * value -1 restores the built-in default.  Any other value, or an unknown
 * knob, is FA_ERR_INVALID_ARG.  fa_get_tuning returns the value a call with
 * head dim d would use now.
 */
typedef enum fa_tune_knob {
  FA_TUNE_FWD_POLY_PAIRS = 1,
  FA_TUNE_FWD_POLY_DEGREE = 2,
  FA_TUNE_BWD_POLY_GROUPS = 3,
  FA_TUNE_DQ_POLY_PAIRS = 4,
  FA_TUNE_FP8_POLY_PAIRS = 5,
  FA_TUNE_BWD_PAIR = 6,
  FA_TUNE_FWD_PERSISTENT = 8,
  FA_TUNE_FWD_CAUSAL_GROUP = 9,
  FA_TUNE_FWD_Q1 = 10,
  FA_TUNE_BWD_CAUSAL_GROUP = 11,
  FA_TUNE_COUNT = 12
} fa_tune_knob;
fa_status fa_set_tuning(int knob, int value);
int fa_get_tuning(int knob, int d);

/*
 * Device status word of the current device: FA_OK, or the first in-kernel
 * failure (FA_ERR_PIPELINE_TIMEOUT, with the failing wait's site in bits
 * 8..15) since the last fa_clear_status().  Synchronises with the device
 * (cudaMemcpyFromSymbol); call it after synchronising your stream.
 */
unsigned int fa_get_status(void);
void fa_clear_status(void);

/*
 * Self-test of the failure path (not part of the attention computation):
 * launches one CTA whose pipeline wait can never complete.  After the bounded
 * wait (~2 s) it records FA_ERR_PIPELINE_TIMEOUT (site 0x7F) in the status
 * word and returns; nothing is faulted or trapped and the context stays
 * usable.  Synchronise, then read fa_get_status() and fa_clear_status().
 */
fa_status fa_selftest_wait_timeout(void* stream);

/*
 * Self-test of the softmax's exp2 (not part of the attention computation):
 * y[i] = 2^x[i] for n (even) fp32 device values, evaluated in pairs exactly
 * as the attention kernels evaluate it.  degree 0 is the SFU instruction;
 * 3, 4 or 5 the FMA-pipe polynomial of that degree (Cody-Waite reduction and
 * a minimax polynomial on [-1/2, 1/2]; inputs below -126 are clamped).  x and
 * y are 8-byte aligned.  Lets a test measure the approximation's relative
 * error against fp64 on a dense grid.
 */
fa_status fa_selftest_exp2(const float* x, float* y, long long n, int degree, void* stream);

/* Static, human-readable name of a status code. */
const char* fa_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H_ */
