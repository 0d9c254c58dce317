/*
 * exattn — exact scaled-dot-product attention for NVIDIA B200 (sm_100a).
 *
 * What it computes.  For every batch b and head h:
 *
 *     S = scale * Q K^T,   P = softmax(S) row by row,   O = P V,
 *
 * the definition in "11.11 Flash Attention" (algomaster.io), section
 * "Standard Attention: Step by Step" (Attention(Q,K,V) = softmax(Q K^T /
 * sqrt(d_k)) V).  It is computed tile by tile with an online softmax (same
 * page, sections "Flash Attention: The Key Insight" and "The Tiling
 * Algorithm"), so the N x N matrices S and P never reach device memory.
 * The forward also writes the per-row logsumexp
 *
 *     LSE_i = ln sum_j exp(S_ij),
 *
 * the per-row maximum m and running sum l of "Walk through the
 * FlashAttention algorithm ..." (zenaique.com), answer to "How does the
 * backward pass avoid storing the n x n attention matrix?", folded into one
 * number.  The backward recomputes P from Q, K and LSE tile by tile ("11.11
 * Flash Attention", section "The Recomputation Trade-off") and returns dQ, dK
 * and dV, the chain rule of the definition above:
 *
 *     dV = P^T dO,  dP = dO V^T,  D_i = sum_k dO_ik O_ik,
 *     dS = P o (dP - D 1^T),  dQ = scale dS K,  dK = scale dS^T Q.
 *
 * Conventions shared by every entry point
 * ----------------------------------------
 *  - Tensors q, k, v, o, dO, dq, dk, dv are bf16 (passed as raw 16-bit
 *    patterns; the _fp16 entry points take fp16 instead), contiguous, row-major [B, H, N, d]: the (batch, heads,
 *    seq_len, head_dim) order of the pages' PyTorch examples.  lse is fp32
 *    [B, H, N].  All of them are DEVICE pointers on the current CUDA device.
 *  - d must be 64 or 128; the forward entry points (attn_fwd, attn_fwd_fp16,
 *    attn_fwd_kvsplit) also take 256 (PyTorch SDPA's limit quoted in "11.11
 *    Flash Attention", section "Using Flash Attention"); attn_fwd_fp8 takes
 *    128 only.  N >= 1 is arbitrary (no multiple-of-tile rule).
 *    B, H or N equal to 0 is an empty problem: the call returns
 *    ATTN_OK and touches nothing (pointers may then be NULL).
 *  - causal != 0 applies the square top-left mask: query i sees key j iff
 *    j <= i.  (The pages do not discuss masking; this is the usual reading.)
 *  - scale is the softmax scale (1/sqrt(d) in the pages' formula); it must be
 *    finite and > 0.
 *  - Every pointer must be 16-byte aligned.  Outputs must not overlap inputs.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream).  They never synchronise and never allocate device
 *    memory: the caller owns every buffer, including the backward workspace.
 *  - Return value: an attn_status code.  Argument errors are detected on the
 *    host before anything is launched.  A kernel that gives up waiting on an
 *    internal barrier (a bounded wait of about one second; it should never
 *    happen) records ATTN_ERR_TIMEOUT in a device status word that
 *    attn_get_device_status() reports.
 */
#ifndef EXATTN_H_
#define EXATTN_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* attn_stream_t;

typedef enum attn_status {
  ATTN_OK = 0,
  ATTN_ERR_INVALID = 1,            /* bad argument: null/misaligned pointer, negative size,
                                      d not supported by the call, scale not finite or <= 0,
                                      workspace too small, size overflow (B*H times N
                                      rounded up to 128 must stay below 2^31) */
  ATTN_ERR_UNSUPPORTED_DEVICE = 2, /* current device is not sm_100 (B200) */
  ATTN_ERR_LAUNCH = 3,             /* a CUDA call failed (launch, attribute, tensor map) */
  ATTN_ERR_TIMEOUT = 4             /* a device-side wait ran out (see above) */
} attn_status;

/*
 * Forward pass.
 *   q, k, v : in,  bf16 [B,H,N,d]
 *   o       : out, bf16 [B,H,N,d]   O = softmax(scale Q K^T [+ mask]) V
 *   lse     : out, fp32 [B,H,N]     natural-log logsumexp of each scaled score row
 * Work: 4*d flops per unmasked (query, key) pair.
 */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
             float scale, int causal, attn_stream_t stream);

/*
 * Size in bytes of the device workspace attn_bwd() needs: an fp32 dQ
 * accumulator [B,H,Np,d] plus fp32 D and pre-scaled LSE rows [B,H,Np], where
 * Np is N rounded up to a multiple of 128.  Returns 0 for an empty or invalid
 * problem.
 */
size_t attn_bwd_workspace_bytes(int B, int H, int N, int d);

/*
 * Backward pass: the three stages below, in order, on `stream`.
 *   q, k, v, o, dO : in,  bf16 [B,H,N,d] (o from attn_fwd on the same inputs)
 *   lse            : in,  fp32 [B,H,N]   (from attn_fwd)
 *   dq, dk, dv     : out, bf16 [B,H,N,d]
 *   workspace      : scratch, device, >= attn_bwd_workspace_bytes(B,H,N,d)
 *                    bytes, 256-byte aligned; contents on entry are ignored.
 * Work: 10*d flops per unmasked pair (five matmuls, one of them the
 * recomputation of Q K^T).
 */
int attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
             void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale, int causal, void* workspace,
             size_t workspace_bytes, attn_stream_t stream);

/*
 * The backward's stages, callable one by one (attn_bwd calls exactly these).
 *
 * Stage 1: D_i = sum_k dO_ik O_ik (fp32) and the LSE rows pre-multiplied by
 * log2(e) into the workspace (padded rows get D = 0 and LSE = +inf, which
 * makes their probabilities exactly 0), and zero the fp32 dQ accumulator.
 */
int attn_bwd_preprocess(const void* o, const void* dO, const float* lse, int B, int H, int N, int d,
                        void* workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * Stage 2: for each key tile, recompute S^T and P^T tile by tile and
 * accumulate dV = P^T dO and dK = scale dS^T Q (written as bf16 to dk, dv),
 * and add each tile's dS K into the fp32 dQ accumulator of the workspace.
 * Needs stage 1's workspace contents.
 */
int attn_bwd_dkdv(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv, int B, int H,
                  int N, int d, float scale, int causal, void* workspace, size_t workspace_bytes,
                  attn_stream_t stream);

/* Stage 3: dq = bf16(scale * dQ accumulator). */
int attn_bwd_dq_convert(void* dq, int B, int H, int N, int d, float scale, const void* workspace,
                        size_t workspace_bytes, attn_stream_t stream);

/*
 * Forward on FP8 (e4m3) inputs, the low-precision mode the pages give the
 * third version of the method ("11.11 Flash Attention", section "Flash
 * Attention 3", FP8 support; the v1/v2/v3 comparison table of "Walk through
 * the FlashAttention algorithm ...").
 *   q, k, v : in,  e4m3 [B,H,N,d] (one byte per element), d = 128 only;
 *             the real values are q * q_descale, k * k_descale, v * v_descale
 *             (per-tensor factors, finite and > 0)
 *   o       : out, bf16 [B,H,N,d]
 *   lse     : out, fp32 [B,H,N], as attn_fwd, of the scaled real scores
 * S = (scale q_descale k_descale) Q K^T is computed by e4m3 tensor-core
 * products with fp32 accumulation.  The probabilities are scaled into e4m3's
 * normal range and rounded to e4m3 for the P V product (relative error at
 * most 2^-4 each); the softmax sums and the LSE use them unrounded, in fp32.
 * Same conventions and status codes as attn_fwd (d != 128 is
 * ATTN_ERR_INVALID).
 */
int attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                 float scale, int causal, float q_descale, float k_descale, float v_descale, attn_stream_t stream);

/*
 * Forward with the keys of each query row split into ranges: decode (a few
 * new queries against a long key/value history) and long rows that leave the
 * machine under-filled.
 *
 *   q, o  : bf16 [B,H,Nq,d] (in / out)     k, v : bf16 [B,H,Nk,d] (in)
 *           (fp16 through attn_fwd_kvsplit_fp16, below)
 *   lse   : fp32 [B,H,Nq] (out), natural-log logsumexp of each scaled score row
 *   causal: the Nq queries are the LAST Nq positions of the Nk-token
 *           sequence: query i sees key j iff j <= Nk - Nq + i (for Nq = Nk
 *           the square mask of attn_fwd).  Requires Nq <= Nk.
 *   splits: key ranges per query row; 0 lets the library choose (it simulates
 *           the launch on the device's SM count), n > 0 asks for n (capped at
 *           64 and at the number of 128-key tiles).  The ranges hold equal
 *           numbers of tiles, ceil(tiles / n) each, so fewer than n may be
 *           used (attn_fwd_kvsplit_count reports how many).
 *   workspace: device, 256-byte aligned, >= attn_fwd_kvsplit_workspace_bytes()
 *           with the same arguments (0 bytes, and NULL allowed, when a single
 *           range is used); contents on entry are ignored.
 *
 * Each range is reduced tile by tile exactly as in attn_fwd, giving a partial
 * output normalised by its own sum and its own logsumexp; a second kernel
 * merges them, O = sum_s exp(LSE_s - LSE) O_s with LSE = log sum_s exp(LSE_s).
 * This is the online-softmax algebra of "11.11 Flash Attention" (section
 * "Flash Attention: The Key Insight") applied across ranges instead of
 * tiles.  The serving use it exists for is named on the pages ("Walk through
 * the FlashAttention algorithm ...", paragraph on products: vLLM, TensorRT-LLM).
 * Nq = 0, B = 0 or H = 0 is an empty problem; Nk = 0 (no keys) is invalid.
 * Same status codes as attn_fwd.
 */
int attn_fwd_kvsplit(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq,
                     int Nk, int d, float scale, int causal, int splits, void* workspace, size_t workspace_bytes,
                     attn_stream_t stream);

/* Workspace bytes attn_fwd_kvsplit() needs for these arguments (0 if one
 * range is used, or if the sizes are invalid or empty). */
size_t attn_fwd_kvsplit_workspace_bytes(int B, int H, int Nq, int Nk, int d, int causal, int splits);

/* The number of key ranges attn_fwd_kvsplit() uses for these arguments (0 if
 * the sizes are invalid or empty). */
int attn_fwd_kvsplit_count(int B, int H, int Nq, int Nk, int d, int causal, int splits);

/*
 * fp16 inputs.  The same operations on IEEE half-precision tensors: q, k, v,
 * o, dO, dq, dk, dv are fp16 (raw 16-bit patterns) instead of bf16; every
 * other argument, the layout and the rules are those of attn_fwd and
 * attn_bwd above (the same workspace size).  The probabilities P and the
 * score gradients dS that feed the tensor cores are rounded to fp16, the
 * accumulators stay fp32.  The pages list FP16 beside BF16 for every version
 * of the method ("Walk through the FlashAttention algorithm ...", the
 * v1/v2/v3 comparison table, precision row).  No range check is made: as
 * with any fp16 computation, scores or gradients beyond the fp16 range
 * (65504) overflow.
 */
int attn_fwd_fp16(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                  float scale, int causal, attn_stream_t stream);

int attn_bwd_fp16(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                  void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale, int causal,
                  void* workspace, size_t workspace_bytes, attn_stream_t stream);

/* attn_fwd_kvsplit() on fp16 q, k, v and o; attn_fwd_kvsplit_workspace_bytes()
 * and attn_fwd_kvsplit_count() apply unchanged (they do not depend on which
 * 16-bit type is used). */
int attn_fwd_kvsplit_fp16(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq,
                          int Nk, int d, float scale, int causal, int splits, void* workspace,
                          size_t workspace_bytes, attn_stream_t stream);

/*
 * Backward without any device allocation: attn_bwd() run on scratch memory
 * that the library itself holds.  (The pages have no counterpart to this
 * entry point; it exists for how callers manage memory, not for the method.)
 *
 * Meant for callers that cannot call cudaMalloc: code that must run within a
 * device-memory budget fixed at start-up, plugins inside a host program that
 * owns the device allocator, and code where an allocation, which can
 * synchronise the whole device, is not allowed.  Such a caller still passes
 * every input and output (same meaning, layout and rules as attn_bwd()); the
 * workspace comes from one file-scope device array of
 * EXATTN_NOALLOC_SCRATCH_BYTES (64 MiB) that every GPU which loads the
 * library holds until the process exits.
 *
 *  - Problems whose attn_bwd_workspace_bytes(B,H,N,d) exceeds
 *    EXATTN_NOALLOC_SCRATCH_BYTES are rejected with ATTN_ERR_INVALID before
 *    anything runs: for d = 128 when B*H*ceil(N/128) > 1008, for d = 64
 *    when B*H*ceil(N/128) > 1985.
 *  - Every call looks up the array's device address in the current device's
 *    context (a host-side lookup, no device work), so a context that was
 *    re-created, e.g. after cudaDeviceReset, is followed.  The first call on
 *    a device may load the library's kernels into the context: make it
 *    before any stream capture.
 *  - Every call on a device shares the one array.  Each call re-initialises
 *    the parts it reads, so leftover contents never leak into results, but
 *    calls that overlap on the GPU (other streams, other host threads) race
 *    on it: serialise them.
 */
#define EXATTN_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

int attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                     const void* dO, void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale,
                     int causal, attn_stream_t stream);

/*
 * One forward and backward pass over tensors that live in HOST memory: the
 * copies to and from the device are part of the call.  (The pages have no
 * counterpart: it strings attn_fwd and attn_bwd above together with the
 * transfers, for callers whose data is not resident on the GPU.)
 *
 *   q, k, v, dO     host, [B, H, N, d] bf16, read
 *   o, dq, dk, dv   host, [B, H, N, d] bf16, written (as attn_fwd / attn_bwd)
 *   lse             host, [B, H, N] fp32, written
 *   dev_buf         device memory of at least
 *                   attn_fwd_bwd_host_buffer_bytes(B, H, N, d, heads_per_chunk)
 *                   bytes, 256-byte aligned, owned by the caller and not used
 *                   by anything else until the call's work on `stream` ends
 *   heads_per_chunk (batch, head) pairs per pipeline chunk; 0 = B*H/8
 *                   rounded up
 *
 * The (batch, head) pairs are independent, so the call splits them into
 * chunks of heads_per_chunk consecutive pairs and pipelines the chunks over
 * three buffer sets in dev_buf: while chunk c runs its kernels on `stream`,
 * the inputs of chunk c+1 are copied in and the results of chunk c-1 copied
 * out, on two internal streams of this library.  Like the calls above it only
 * enqueues work: all of it completes before anything enqueued on `stream`
 * after the call, and the host buffers must stay valid until then.  For the
 * copies to overlap, the host buffers must be page-locked (cudaHostAlloc or
 * cudaHostRegister); pageable buffers give the same results, slower.
 *
 * Returns ATTN_OK (also for empty problems), ATTN_ERR_INVALID (a bad size,
 * scale or pointer, or dev_buf too small or misaligned), or ATTN_ERR_LAUNCH.
 */
int attn_fwd_bwd_host(const void* q, const void* k, const void* v, const void* dO, void* o, float* lse, void* dq,
                      void* dk, void* dv, int B, int H, int N, int d, float scale, int causal, void* dev_buf,
                      size_t dev_buf_bytes, int heads_per_chunk, attn_stream_t stream);

/* Device bytes attn_fwd_bwd_host() needs; 0 if the sizes are invalid or empty. */
size_t attn_fwd_bwd_host_buffer_bytes(int B, int H, int N, int d, int heads_per_chunk);

/*
 * Synchronises `stream`, then returns and clears the device status word of
 * the current device: ATTN_OK, or ATTN_ERR_TIMEOUT if any kernel of this
 * library gave up waiting since the last call (ATTN_ERR_LAUNCH if the
 * synchronisation itself failed).
 */
int attn_get_device_status(attn_stream_t stream);

/*
 * Failure detection.  Every wait of a kernel on one of its internal barriers
 * is limited in time (1 s by default).  When a limit runs out the kernel
 * records ATTN_ERR_TIMEOUT for attn_get_device_status(), all of its roles
 * leave their loops, copies and matrix multiplies already in flight are
 * allowed to finish, and the kernel returns: it never hangs the GPU, and the
 * CUDA context stays usable.  This sets the limit used by launches made after
 * the call, process-wide; 0 restores the default.  A limit of a few
 * nanoseconds makes ordinary waits run out, which is how the failure path is
 * tested.  (The pages have no counterpart; this is an operational control.)
 */
void attn_set_wait_timeout_ns(unsigned long long ns);

/*
 * Fault injection for testing the path above.  While `on` is nonzero, the
 * forward and main backward kernels launched afterwards skip their first K/V
 * tile load, so one of their roles waits on a barrier that nothing will ever
 * complete; the bounded wait then runs out and the call reports
 * ATTN_ERR_TIMEOUT (results are then undefined).  No fault, trap or hang is
 * involved.  Off by default; process-wide.
 */
void attn_debug_inject_stall(int on);

/* Static, human-readable name of a status code. */
const char* attn_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* EXATTN_H_ */
