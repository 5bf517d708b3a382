/*
 * attn.h -- C ABI of the B200 (sm_100a) attention library: the forward pass in bf16
 * (attn_fwd, attn_fwd_ws, attn_fwd_noalloc; attn_fwd_from_host on host buffers) and E4M3
 * (attn_fwd_fp8), its gradients (attn_bwd), and rotary position embedding of Q and K
 * (attn_rope_tables, attn_rope_qk, attn_fwd_rope; their backward attn_rope_qk_inverse, attn_bwd_rope).
 *
 * The operation is the tiled attention forward pass named by "HipKittens:
 * fast and furious AMD kernels" (section "Performance results": an attention
 * forward kernel over several head dims D and sequence lengths N, causal and
 * non-causal) and "Making AMD GPUs go brrr" (section "Real kernel example":
 * a hot loop built from a score matmul, exp2 and row sums).  The pages print
 * no formula; the library computes the plain definition
 *
 *     O[b,h]    = softmax(scale * Q[b,h] K[b,g(h)]^T  (+ causal mask)) V[b,g(h)]
 *     LSE[b,h,i] = ln sum_j exp(scale * q_i . k_j)      (over the allowed keys j)
 *
 * with g(h) = h / (Hq / Hkv) (contiguous groups of query heads share one KV
 * head) and, when causal, key j allowed for query i iff j <= i.
 *
 * Every entry point validates its arguments on the host before touching the
 * GPU and returns an attn_status_t code; ATTN_OK is 0.
 */
#ifndef ATTN_H_
#define ATTN_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1, /* null pointer, negative size, Hq % Hkv != 0, non-finite scale */
  ATTN_ERR_UNSUPPORTED = 2, /* a head dim D the entry point does not cover, or a size beyond the limits below */
  ATTN_ERR_MISALIGNED = 3,  /* a tensor pointer not 16-byte aligned, lse not 4-byte aligned, or a
                               workspace not 256-byte aligned (per entry point below) */
  ATTN_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed (launch, attribute, tensor map) */
  ATTN_ERR_TIMEOUT = 5      /* a kernel wait gave up (reported by attn_device_status) */
} attn_status_t;

/*
 * attn_fwd -- enqueue one attention forward pass on `stream`.
 *
 * Arguments (all pointers are DEVICE pointers; the caller allocates, owns and
 * frees every buffer; the library allocates nothing and keeps no pointer):
 *   q     bf16 [B, Hq,  N, D], contiguous, row-major (D fastest).   read
 *   k     bf16 [B, Hkv, N, D], contiguous.                          read
 *   v     bf16 [B, Hkv, N, D], contiguous.                          read
 *   o     bf16 [B, Hq,  N, D], contiguous.                          written (every element)
 *   lse   fp32 [B, Hq,  N],    contiguous; natural-log log-sum-exp of the
 *         scaled, masked scores of each query row.                  written (every element)
 *   B, Hq, Hkv, N   batch, query heads, key/value heads, sequence length.
 *         B >= 0, N >= 0, Hq >= 1, Hkv >= 1, Hq % Hkv == 0.  B == 0 or N == 0
 *         is an empty problem: ATTN_OK is returned and nothing is launched
 *         (pointers may then be null).  Limits: B*Hq <= 2^31-1, N <= 2^31-1 and
 *         B*Hq*ceil(N/256) <= 2^31-1 (work units of 256 query rows, indexed in 32 bits
 *         by the scheduler), and at D = 192, 256 B*Hq*ceil(N/128) <= 2^30 (query tiles of the
 *         wide-head kernel); beyond them ATTN_ERR_UNSUPPORTED.
 *   D     head dim of q, k, v and o: 32, 64, 96, 128, 192 or 256.  D <= 128 runs on the two-tile
 *         kernel (two 128-row Q tiles per CTA ping-pong on the tensor core); 192 and 256 run on a
 *         one-tile kernel that ping-pongs two score buffers instead (2 x (128 + D) tensor-memory
 *         columns would exceed 512).
 *   causal  0: every key is visible; non-zero: key j is visible to query i
 *         iff j <= i (queries and keys share positions 0..N-1).
 *   scale   finite float multiplying q.k before the softmax (1/sqrt(D) is
 *         the usual choice; 0 and negative values are accepted).
 *   stream  cudaStream_t (passed as void*) on which the kernel is enqueued;
 *         null means the legacy default stream.  The call is asynchronous:
 *         results are valid once the stream has reached this point.
 *
 * Errors: the host checks above are made before any CUDA call; on any error
 * return nothing is launched and o/lse are untouched.  ATTN_ERR_CUDA means a
 * CUDA call (tensor-map encode, attribute, launch) failed; the CUDA error
 * string is available from attn_last_cuda_error().  The kernel's waits are
 * bounded; if one gives up the kernel exits early and records the fact, which
 * attn_device_status() reports after the caller synchronises.
 *
 * Numerics: fp32 accumulation of Q K^T and P V on the tensor cores, base-2
 * online softmax in fp32, probabilities rounded to bf16 before P V, O rounded
 * to bf16 (nearest-even).  The result is bitwise deterministic for a given
 * input, device and build.
 *
 * Thread safety: calls are independent and may be made from several host
 * threads and streams at once.
 */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
             int B, int Hq, int Hkv, int N, int D, int causal, float scale,
             void* stream);

/*
 * attn_fwd_ws -- attn_fwd with a caller-provided device workspace.
 *
 * Same operation, arguments, errors and numerics as attn_fwd.  When the problem is
 * non-causal and its last wave of work units would leave at least half of the GPU
 * idle, each unit of that wave is split into two ranges of KV blocks that run on
 * separate SMs; the range that finishes first writes its unnormalised fp32 O rows and
 * (max, sum) to the workspace and the other merges them with its own (always in range
 * order: results are deterministic, and equal attn_fwd's up to fp32 rounding order).
 *   workspace        device pointer, 256-byte aligned, or NULL (then no split is made)
 *   workspace_bytes  its size; must be >= attn_fwd_workspace_bytes() for the problem
 *                    whenever a split is planned, else ATTN_ERR_INVALID_ARG
 * The workspace needs no initialisation and is left in a state any later call accepts
 * (a call from another loaded copy of this library included).
 * Calls that share a workspace must not run concurrently (same stream, or ordered).
 */
int attn_fwd_ws(const void* q, const void* k, const void* v, void* o, float* lse,
                int B, int Hq, int Hkv, int N, int D, int causal, float scale,
                void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_fwd_workspace_bytes -- workspace attn_fwd_ws needs for these sizes on the current
 * device (0 if it makes no split: causal problems, full last waves, D = 192 or 256).  At most
 * SMs/2 x 2 x 128 x (D + 2) x 4 bytes plus 16 bytes per split unit rounded up to 256
 * (about 9.9 MB on a 148-SM B200 at D=128).
 * Queries the current device's SM count; returns -1 on invalid sizes or a CUDA error.
 */
long long attn_fwd_workspace_bytes(int B, int Hq, int N, int D, int causal);

/*
 * attn_fwd_noalloc -- attn_fwd_ws for callers that cannot allocate device memory.
 *
 * (The pages have no counterpart: this is an interface convenience.)  Some callers may
 * not call cudaMalloc to provide attn_fwd_ws's workspace: code whose device memory is all
 * owned by another allocator (a framework's caching allocator, an embedded runtime that
 * forbids allocation after start-up), or latency-critical code that must not risk the
 * device-wide synchronisation an allocation can cause.  This entry point takes no
 * workspace argument and allocates nothing: the workspace is a 10 MiB
 * array inside the library, present once on every device that loads the library and kept
 * until the process exits.  Arguments, errors and numerics are those of attn_fwd; the
 * caller still owns q, k, v, o and lse.
 *   - Problems whose split needs more than the array (attn_fwd_workspace_bytes() larger
 *     than attn_fwd_noalloc_scratch_bytes(); not reachable at D <= 128 on a 148-SM B200)
 *     are rejected with ATTN_ERR_UNSUPPORTED and a message in attn_last_cuda_error().
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call before any
 *     stream capture.  A failed look-up returns ATTN_ERR_CUDA and is retried by the next
 *     call.  Nothing is cleared: the array starts at zero when the library loads, and the
 *     kernel tags its counter words with a per-launch epoch and zeroes them after use.
 *   - Every call shares the one array and leaves its contents behind; no later call
 *     needs them cleared.  Calls whose kernels overlap on the GPU (different streams
 *     without ordering) race on the array and must be avoided.
 */
int attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                     int B, int Hq, int Hkv, int N, int D, int causal, float scale,
                     void* stream);

/* Size in bytes of the array attn_fwd_noalloc uses as its workspace. */
size_t attn_fwd_noalloc_scratch_bytes(void);

/*
 * attn_fwd_from_host -- the attention forward of attn_fwd_ws on HOST buffers, end to end:
 * upload q, k, v, compute, download o and lse; returns once o_host and lse_host hold the
 * results.  (The pages have no counterpart: this is the library's end-to-end entry point for
 * data that lives in host memory.)
 *
 * Arguments:
 *   q_host, k_host, v_host   bf16 [B, Hq, N, D] / [B, Hkv, N, D] in HOST memory, contiguous. read
 *   o_host, lse_host         bf16 [B, Hq, N, D] and fp32 [B, Hq, N] in HOST memory.       written
 *                            Page-locked (pinned) host memory is needed for the copies to
 *                            overlap the kernels; pageable memory works, without overlap.
 *   q_dev, k_dev, v_dev, o_dev, lse_dev   DEVICE buffers of the same sizes (16-byte aligned;
 *                            lse_dev 4-byte), owned by the caller; the call copies into and out
 *                            of them and leaves the inputs and results there.
 *   workspace, workspace_bytes   optional split-tail workspace (256-byte aligned, or NULL with
 *                            0 bytes); a piece whose split needs more makes no split.
 *                            attn_fwd_from_host_workspace_bytes() gives the size every piece
 *                            can use.
 *   B, Hq, Hkv, N, D, causal, scale   as attn_fwd.
 *   pieces                   >= 1: the problem is cut into up to `pieces` (at most 64)
 *                            independent parts -- ranges of batch rows, or for B == 1 ranges
 *                            of whole KV-head groups -- so that each part's upload and
 *                            download overlap the neighbouring parts' kernels.
 *   stream                   the kernels run on `stream`; the copies on two non-blocking
 *                            streams the library creates once per device.  The uploads start
 *                            after the work enqueued on `stream` before the call.
 * The library allocates no device memory (streams and events only).  The call is synchronous:
 * it returns after the last download (or, on an error, after everything it enqueued).
 * Errors: as attn_fwd_ws; ATTN_ERR_INVALID_ARG also for a null host or device buffer or
 * pieces < 1; ATTN_ERR_CUDA if a copy, event or stream call fails (text in
 * attn_last_cuda_error()).  Results equal those of attn_fwd_ws on each piece.
 * Calls from several host threads share the copy streams (their copies then take turns) and
 * are otherwise independent, given distinct buffers and workspaces.
 */
int attn_fwd_from_host(const void* q_host, const void* k_host, const void* v_host, void* o_host,
                       float* lse_host, void* q_dev, void* k_dev, void* v_dev, void* o_dev,
                       float* lse_dev, void* workspace, size_t workspace_bytes,
                       int B, int Hq, int Hkv, int N, int D, int causal, float scale,
                       int pieces, void* stream);

/*
 * attn_fwd_from_host_workspace_bytes -- the largest split-tail workspace any piece of an
 * attn_fwd_from_host call with these sizes uses on the current device (0 if none splits);
 * -1 on invalid sizes or a CUDA error.
 */
long long attn_fwd_from_host_workspace_bytes(int B, int Hq, int Hkv, int N, int D, int causal,
                                             int pieces);

/*
 * attn_bwd -- enqueue the attention backward pass (gradients of the forward) on `stream`.
 *
 * The pages name an attention backward kernel beside the forward ("HipKittens: fast and
 * furious AMD kernels", section "Performance results") without a formula.  With P the
 * forward's probabilities (rebuilt from the saved LSE) and dO the gradient of a loss with
 * respect to O, the library computes the plain definition
 *
 *     delta_i = sum_d dO_id O_id,   dS = P o (dO V^T - delta)
 *     dQ[b,h]    = scale dS K[b,g(h)]
 *     dK[b,g]    = scale sum over the query heads h of group g of dS^T Q[b,h]
 *     dV[b,g]    = sum over the query heads h of group g of P^T dO[b,h]
 *
 * Arguments (DEVICE pointers; the caller allocates, owns and frees every buffer):
 *   q, k, v, o, lse   the forward's inputs and outputs, layouts as in attn_fwd     read
 *                     (o and lse as attn_fwd wrote them for the same q, k, v, causal, scale)
 *   dout  bf16 [B, Hq,  N, D], contiguous: dL/dO.                                  read
 *   dq    bf16 [B, Hq,  N, D], contiguous.                           written (every element)
 *   dk    bf16 [B, Hkv, N, D], contiguous.                           written (every element)
 *   dv    bf16 [B, Hkv, N, D], contiguous.                           written (every element)
 *   B, Hq, Hkv, N, D, causal, scale   as in attn_fwd, but D in {32, 64, 96, 128}; additionally
 *         B * Hq * ceil(N / 128) <= 2^30, else ATTN_ERR_UNSUPPORTED.
 *   workspace        device pointer, 256-byte aligned, of at least
 *                    attn_bwd_workspace_bytes(B, Hq, N) bytes (per-row delta and
 *                    LSE * log2(e)); needs no initialisation; calls sharing it must be
 *                    ordered (same stream).
 *   stream  cudaStream_t (void*), as in attn_fwd.  Three kernels are enqueued.
 *
 * Errors as in attn_fwd: host checks first (ATTN_ERR_INVALID_ARG also for a null or too
 * small workspace; ATTN_ERR_MISALIGNED for a tensor pointer not 16-byte aligned, lse not
 * 4-byte aligned or the workspace not 256-byte aligned); outputs untouched on error.
 *
 * Numerics: scores and dP = dO V^T accumulate in fp32 on the tensor cores; P and dS are
 * rounded to bf16 before the dV, dK and dQ matmuls, which accumulate in fp32 in tensor
 * memory; the gradients are rounded to bf16 (nearest-even).  Every output row is
 * produced by one CTA in a fixed order: results are bitwise deterministic.
 */
int attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
             const void* dout, void* dq, void* dk, void* dv,
             int B, int Hq, int Hkv, int N, int D, int causal, float scale,
             void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_bwd_workspace_bytes -- workspace attn_bwd needs: 2 x B x Hq x ceil(N/128) x 128 x 4
 * bytes, each half rounded up to 256.  Host-only, no CUDA call; 0 for an empty problem,
 * -1 on invalid sizes.
 */
long long attn_bwd_workspace_bytes(int B, int Hq, int N);

/*
 * attn_rope_qk -- rotary position embedding (RoPE) of Q and K, one pass over HBM.
 *
 * The pages list a rotary kernel among those built with the tile library ("HipKittens: fast
 * and furious AMD kernels", section "Performance results") without a formula.  Rotate-half
 * pairing: for the row of position p (its index 0..N-1 within the head) and d < D/2,
 *     x'_d       = x_d cos_t[p][d] - x_{d+D/2} sin_t[p][d]
 *     x'_{d+D/2} = x_{d+D/2} cos_t[p][d] + x_d sin_t[p][d]
 * (usually cos_t, sin_t = cos, sin of p * base^(-2d/D); the caller chooses the angles).
 *
 * Arguments (DEVICE pointers, caller-owned; all 16-byte aligned):
 *   q, k          bf16 [B, Hq, N, D] and [B, Hkv, N, D], contiguous.               read
 *   cos_t, sin_t  fp32 [N, D/2], contiguous.                                        read
 *   q_out, k_out  bf16, same shapes as q, k; written (every element).  May equal q, k
 *                 (in place).
 *   B, Hq, Hkv, N, D  as in attn_fwd (D in {32, 64, 96, 128}).
 *   stream        cudaStream_t (void*); asynchronous.
 * Errors: host checks as in attn_fwd, before any CUDA call (ATTN_ERR_MISALIGNED for any
 * pointer not 16-byte aligned); ATTN_ERR_UNSUPPORTED when B*(Hq+Hkv)*N*D/16 > 2^38.
 * Numerics: fp32 arithmetic on the bf16 inputs and fp32 tables, rounded to bf16 (nearest even).
 */
int attn_rope_qk(const void* q, const void* k, const float* cos_t, const float* sin_t,
                 void* q_out, void* k_out, int B, int Hq, int Hkv, int N, int D, void* stream);

/*
 * attn_rope_tables -- fill the usual RoPE angle tables on the device:
 *     cos_t[p][d] = cos(theta),  sin_t[p][d] = sin(theta),  theta = p * base^(-2d/D)
 * for positions p < N and d < D/2 (the frequencies of the rotary embedding the pages' rotary
 * kernel applies, "HipKittens: fast and furious AMD kernels", section "Performance results";
 * the pages print no schedule, so this is the common one with a caller-chosen base).
 *   cos_t, sin_t  DEVICE fp32 [N, D/2], contiguous, 16-byte aligned, caller-owned.  written
 *   N >= 0, D >= 2 even, base finite and > 0 (10000 is the usual value).
 *   stream        cudaStream_t (void*); asynchronous.
 * Numerics: theta, its cosine and sine in fp64, each rounded to fp32 (nearest).
 * Errors: ATTN_ERR_INVALID_ARG (sizes, base, null pointers with N > 0), ATTN_ERR_MISALIGNED,
 * ATTN_ERR_UNSUPPORTED for N * D/2 > 2^40, ATTN_ERR_CUDA on a launch failure.
 */
int attn_rope_tables(float* cos_t, float* sin_t, int N, int D, double base, void* stream);

/*
 * attn_fwd_rope -- attention forward of RoPE(Q), RoPE(K) and V in one call: attn_rope_qk into
 * the caller's workspace, then the forward kernel on the rotated tensors (both enqueued on
 * `stream`).  Arguments as attn_fwd plus the tables of attn_rope_qk and
 *   workspace        device pointer, 256-byte aligned, at least
 *                    attn_fwd_rope_workspace_bytes() bytes (fewer, but at least the two rotated
 *                    tensors, also works: the forward then makes no split); after the call it
 *                    holds RoPE(Q) at offset 0 and RoPE(K) at offset round_up(B*Hq*N*D*2, 256).
 * Errors as attn_fwd and attn_rope_qk (ATTN_ERR_INVALID_ARG for a null or too small
 * workspace).  The result equals attn_fwd_ws on the outputs of attn_rope_qk.
 */
int attn_fwd_rope(const void* q, const void* k, const void* v, const float* cos_t, const float* sin_t,
                  void* o, float* lse, int B, int Hq, int Hkv, int N, int D, int causal, float scale,
                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_fwd_rope_workspace_bytes -- workspace attn_fwd_rope uses for these sizes on the current
 * device: the rotated Q and K (each rounded up to 256 bytes) plus the non-causal split
 * workspace of attn_fwd_workspace_bytes().  -1 on invalid sizes or a CUDA error.
 */
long long attn_fwd_rope_workspace_bytes(int B, int Hq, int Hkv, int N, int D);

/*
 * attn_rope_qk_inverse -- the inverse of attn_rope_qk: rotates by -theta, i.e. for d < D/2
 *     x_d       = y_d cos(theta_pd) + y_{d+D/2} sin(theta_pd)
 *     x_{d+D/2} = y_{d+D/2} cos(theta_pd) - y_d sin(theta_pd).
 * The rotation is orthogonal, so this is also its transpose: given the gradients of a loss with
 * respect to RoPE(q) and RoPE(k) it returns the gradients with respect to q and k (the backward
 * of the rotary step).  Arguments, layouts, tables, in-place use and errors as attn_rope_qk
 * (dq_rot, dk_rot in; dq, dk out).
 */
int attn_rope_qk_inverse(const void* dq_rot, const void* dk_rot, const float* cos_t, const float* sin_t,
                         void* dq, void* dk, int B, int Hq, int Hkv, int N, int D, void* stream);

/*
 * attn_bwd_rope -- the backward of attn_fwd_rope: gradients of a loss L with respect to q, k
 * (before the rotation) and v, given dO = dL/dO for O = attention(RoPE(q), RoPE(k), v), with
 * the forward's O and LSE (as attn_fwd_rope wrote them).  Three steps on `stream`: attn_rope_qk
 * into the workspace, attn_bwd on the rotated tensors (writing dL/dRoPE(q), dL/dRoPE(k) into dq,
 * dk, and dv), then attn_rope_qk_inverse on dq, dk in place.  Arguments as attn_bwd plus the
 * tables of attn_rope_qk and
 *   workspace        device pointer, 256-byte aligned, at least attn_bwd_rope_workspace_bytes()
 *                    bytes; after the call it holds RoPE(q) at offset 0 and RoPE(k) at offset
 *                    round_up(B*Hq*N*D*2, 256), then the backward's per-row data.
 * D is 32, 64, 96 or 128 (the backward's head dims).  Every argument is checked before the
 * first launch; errors as attn_bwd and attn_rope_qk (ATTN_ERR_INVALID_ARG for a null or too
 * small workspace).
 */
int attn_bwd_rope(const void* q, const void* k, const void* v, const float* cos_t, const float* sin_t,
                  const void* o, const float* lse, const void* dout, void* dq, void* dk, void* dv,
                  int B, int Hq, int Hkv, int N, int D, int causal, float scale,
                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_bwd_rope_workspace_bytes -- workspace attn_bwd_rope needs: the rotated Q and K (each
 * rounded up to 256 bytes) plus attn_bwd_workspace_bytes().  -1 on invalid sizes (D must be
 * 32, 64, 96 or 128).
 */
long long attn_bwd_rope_workspace_bytes(int B, int Hq, int Hkv, int N, int D);

/*
 * attn_fwd_fp8 -- the attention forward on E4M3 (8-bit float) Q, K and V.
 *
 * The pages stress the low-precision tensor-core rates (FP8 GEMM in "HipKittens: fast and
 * furious AMD kernels", sections "State of the AMD ecosystem" and "Performance results") but
 * give no FP8 attention recipe.  The library computes the same definition as attn_fwd on the
 * dequantized inputs  Q = q_descale * q,  K = k_descale * k,  V = v_descale * v:
 *     O = softmax(scale * Q K^T (+ causal mask)) V,   LSE = ln sum_j exp(scale * Q_i . K_j)
 *   q, k, v      E4M3 (float8_e4m3fn: 1 sign, 4 exponent, 3 mantissa bits, max 448) bytes,
 *                [B, Hq, N, D] / [B, Hkv, N, D], contiguous, 16-byte aligned.       read
 *   o, lse       bf16 [B, Hq, N, D] and fp32 [B, Hq, N], as attn_fwd.              written
 *   q_descale, k_descale, v_descale   per-tensor factors (finite; q and k non-zero).
 *   D            32, 64, 96, 128, 192 or 256 (ATTN_ERR_UNSUPPORTED otherwise; 192 and 256 run
 *                on the wide-head kernel, one CTA per 128-row query tile, as attn_fwd does).
 *   workspace, workspace_bytes   optional split-tail workspace, as attn_fwd_ws (never used at
 *                D = 192 and 256).
 * Numerics: Q K^T on the E4M3 tensor cores (kind::f8f6f4) with fp32 accumulation; base-2 online
 * softmax in fp32; probabilities rounded to E4M3 (nearest even; p <= 2^8 by the lazy rescale,
 * inside E4M3's range) for P V, also E4M3 with fp32 accumulation; row sums of the fp32
 * probabilities; O rounded to bf16.  Deterministic.  Errors as attn_fwd_ws, plus
 * ATTN_ERR_INVALID_ARG for non-finite or zero descales.
 */
int attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int Hq, int Hkv, int N, int D, int causal, float scale,
                 float q_descale, float k_descale, float v_descale,
                 void* workspace, size_t workspace_bytes, void* stream);

/* Human-readable name of an attn_status_t value (static string, never null). */
const char* attn_status_string(int status);

/*
 * Text of the last CUDA error seen by an entry point on the calling host
 * thread ("" if none).  Static per-thread storage; valid until the next call
 * on that thread.
 */
const char* attn_last_cuda_error(void);

/*
 * attn_device_status -- synchronise `stream` (void* cudaStream_t) and report
 * whether any kernel of this library, on the current device, gave up on a
 * bounded wait since the previous call.  Returns ATTN_OK or ATTN_ERR_TIMEOUT
 * (and clears the record), or ATTN_ERR_CUDA if the synchronisation failed.
 * If `site` is non-null it receives the code of the first wait that gave up (0 if
 * none): 1-9 the forward kernel's roles (producer, MMA issuer, softmax, drain),
 * 10 the wait self-test, 11 the forward's split-tail merge, 12-19 the backward
 * kernels' roles.
 */
int attn_device_status(void* stream, int* site);

/*
 * attn_num_units -- number of work units (one unit = 256 query rows of one
 * query head) a call with these sizes schedules; the persistent grid is
 * min(units, SM count).  Host-only helper, no CUDA call.  Returns -1 on
 * invalid sizes.
 */
long long attn_num_units(int B, int Hq, int N);

/* Version string of the library build (static). */
const char* attn_version(void);

/* ---- self-test entry points (used by the library's tests; no part of the forward pass) ---- */

/*
 * attn_selftest_fast_div -- floor(n / d) computed on the host the way the forward kernel's
 * scheduler divides by its launch-constant divisors: the high 64 bits of n * m with the
 * precomputed reciprocal m = ceil(2^64 / d) (Granlund and Montgomery, "Division by
 * invariant integers using multiplication"; m = 0 stands for d = 1).  No CUDA call.
 * Returns 0 for d == 0.
 */
unsigned int attn_selftest_fast_div(unsigned int n, unsigned int d);

/*
 * attn_selftest_exp2_poly -- evaluate, on the device, the polynomial 2^x that the
 * softmax uses for part of its exponentials (round-to-nearest range reduction,
 * degree-3 minimax polynomial on [-1/2, 1/2], exponent-field scaling; inputs below
 * -125 are clamped).  x, y: device fp32 arrays of n elements (y written).  Enqueued
 * on `stream`.  Returns ATTN_ERR_INVALID_ARG for n < 0 or null pointers with n > 0.
 */
int attn_selftest_exp2_poly(const float* x, float* y, int n, void* stream);

/*
 * attn_selftest_wait_timeout -- launch a one-CTA kernel whose bounded mbarrier wait
 * can never complete, with a limit of `timeout_us` microseconds (1..1000000).  The
 * wait gives up, records its site and the kernel returns normally; a following
 * attn_device_status() reports ATTN_ERR_TIMEOUT.  Used to test the failure path of
 * the forward kernel's bounded waits without faulting or hanging the GPU.
 */
int attn_selftest_wait_timeout(unsigned int timeout_us, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_H_ */
