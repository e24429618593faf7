/* fa.h — C ABI of the B200 (sm_100a) exact-attention library (libfa.so).
 *
 * What is computed (forward): for every batch b, head h and query row i,
 *     S_ij  = scale * q_i . k_j                    (keys j > i left out when causal)
 *     O_i   = sum_j softmax_j(S_ij) v_j
 *     lse_i = m_i + ln l_i,  m_i = max_j S_ij,  l_i = sum_j exp(S_ij - m_i)
 * i.e. P = softmax(Q K^T / sqrt(d)) and O = P V of "Breaking the Memory Wall: A Deep Dive into
 * FlashAttention" (section "The Problem: The Memory Wall"), computed tile by tile with the
 * online-softmax running max m and running sum l of "How FlashAttention Actually Works"
 * (section "The Secret Weapon: Online Softmax") so that S and P never reach device memory.
 * The backward recomputes S and P on chip from the stored lse ("The Backward Pass:
 * Recomputation" on the same page) and returns dQ, dK, dV of the scalar loss whose gradient
 * with respect to O is dO:
 *     P = exp(S - lse), dV = P^T dO, dP = dO V^T, D_i = dO_i . O_i, dS = P o (dP - D),
 *     dQ = scale dS K, dK = scale dS^T Q.
 *
 * Layout. q, k, v, o, dO, dq, dk, dv: bf16 [B, H, N, d], contiguous (row-major, d fastest).
 * lse: fp32 [B, H, N]. Pointers are DEVICE pointers of the current CUDA device, 16-byte aligned.
 * Causal convention: square, top-left aligned — key j is visible to query i iff j <= i.
 *
 * Ownership. The caller owns every buffer, the stream and the backward workspace. The library
 * keeps, per device, one cached 4-byte status word (allocated on first use) and nothing else.
 *
 * Semantics. Calls are asynchronous on `stream` (0 = legacy default stream) and return after
 * enqueueing. Outputs are fully overwritten. Outputs must not alias inputs. There is no CPU
 * fallback: without an sm_100 device every compute call returns FA_ERR_CUDA.
 *
 * Errors. Arguments are validated before anything is launched; a failed check returns a
 * non-zero fa_status, launches nothing, and fa_last_error_string() describes it (thread-local).
 * Every wait inside the kernels is bounded; a wait that times out makes the kernel give up,
 * record FA_ERR_TIMEOUT in the device status word and return (a kernel that finds its shared
 * memory misaligned gives up the same way, with its own code in the message). fa_check_status()
 * synchronises the stream, reads and clears that word.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null or aliasing pointer, non-positive size, bad scale */
  FA_ERR_UNSUPPORTED = 2, /* head dim or sizes beyond the limits stated below */
  FA_ERR_MISALIGNED = 3,  /* a pointer not 16-byte aligned */
  FA_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed (no device, launch error) */
  FA_ERR_TIMEOUT = 5,     /* a bounded in-kernel wait expired (reported by fa_check_status) */
  FA_ERR_WORKSPACE = 6    /* backward workspace missing or smaller than fa_bwd_workspace_size */
} fa_status;

/* Limits: d in {64, 96, 128, 256} (96 runs the d = 128 kernels on zero-filled columns; the FP8
 * forward takes d <= 128; d = 256 has no dropout); B, H, N >= 1; B*H*N < 2^31;
 * B*H*ceil(N/256) < 2^31. At d = 256 the backward runs its main work in two passes over the
 * key tiles (dV, then dK and dQ), because dK and dV of a 128-key tile fill all of TMEM. */

/* Masks of the extended entry points. */
typedef enum {
  FA_MASK_NONE = 0,                /* every key visible to every query */
  FA_MASK_CAUSAL = 1,              /* key j visible to query i iff j <= i (top-left aligned) */
  FA_MASK_CAUSAL_BOTTOM_RIGHT = 2  /* iff j <= i + N_kv - N_q: the last query sees every key,
                                      as when new queries attend to a longer cached context */
} fa_mask;

/* Shape of the extended entry points: q, o, dO, dq are bf16 [B, H, N_q, d]; k, v, dk, dv are
 * bf16 [B, H_kv, N_kv, d]; lse is fp32 [B, H, N_q]. H must be a multiple of H_kv: query head h
 * uses key/value head h / (H / H_kv) (grouped heads; H_kv = 1 is a single shared K/V head),
 * and dk, dv of a key/value head sum over the query heads that share it. A query row that sees
 * no key (FA_MASK_CAUSAL_BOTTOM_RIGHT with N_q > N_kv) gets o = 0, lse = -inf and dq = 0.
 * Limits: d in {64, 96, 128, 256}; all sizes >= 1; B*H*N_q and B*H_kv*N_kv < 2^31. At d = 256
 * dropout and the FP8 forward return FA_ERR_UNSUPPORTED. */
typedef struct {
  int B, H, H_kv, N_q, N_kv, d;
  float scale; /* finite, > 0; normally 1/sqrt(d) */
  int mask;    /* an fa_mask value */
} fa_attn_shape;

/* Dropout on the attention probabilities, the pass that "How FlashAttention Actually Works"
 * ("The GPU Memory Wall: HBM vs. SRAM") places between the softmax and the product with V.
 * Inverted dropout: each entry of P is kept with probability 1 - p8/256 and scaled by
 * 256/(256 - p8), where p8 = min(255, floor(256 p + 1/2)); lse stays that of the undropped
 * softmax. No mask is stored: the forward and the backward regenerate the same decisions from
 * Philox4x32-10 (Salmon et al., "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11) with
 * counter (j/4, i/4, b*H + h, offset) and key (seed low word, seed high word) for query i and
 * key j of query head h; the entry's byte is byte (j mod 4) of output word (i mod 4), and the
 * entry is kept iff that byte >= p8. Pass the same settings to the forward and the backward.
 * A NULL fa_dropout pointer, or p8 = 0, means no dropout. */
typedef struct {
  float p;                 /* drop probability, in [0, 1) */
  unsigned long long seed; /* Philox key */
  unsigned int offset;     /* Philox counter word 3: vary it between calls that share a seed */
} fa_dropout;

/* Forward for an fa_attn_shape (fa_fwd is the case H_kv = H, N_q = N_kv = N, no dropout). The
 * pages define the square, equal-head case; these shapes apply the same definition with the
 * mask above. dropout: NULL or the settings above (FA_ERR_INVALID_ARG for p outside [0, 1)). */
fa_status fa_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                    const fa_attn_shape* shape, const fa_dropout* dropout, void* stream);

/* Workspace bytes fa_bwd_ex needs (fp32 dQ accumulator and row terms for B*H*N_q rows, and the
 * work-unit counter of the persistent backward kernel); 0 for an
 * invalid shape. */
size_t fa_bwd_ex_workspace_size(const fa_attn_shape* shape);

/* Backward for an fa_attn_shape; arguments as fa_bwd, and dropout as given to fa_fwd_ex for
 * the o and lse passed here. */
fa_status fa_bwd_ex(const void* q, const void* k, const void* v, const void* o, const void* dO,
                    const float* lse, void* dq, void* dk, void* dv, void* workspace,
                    size_t workspace_bytes, const fa_attn_shape* shape,
                    const fa_dropout* dropout, void* stream);

/* Forward. Writes o (bf16 [B,H,N,d]) and lse (fp32 [B,H,N]).
 * scale: the softmax scale (finite, > 0), normally 1/sqrt(d). causal: 0 or 1.
 * stream: a cudaStream_t passed as void*. */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int N, int d, float scale, int causal, void* stream);

/* Bytes of device workspace fa_bwd needs for these sizes (fp32 dQ accumulator [B,H,N,d], the
 * fp32 row terms D and -lse*log2(e) [B,H,N], and a counter that hands out work units to the
 * persistent backward kernel; the first kernel of each call zeroes it). Returns 0 for invalid
 * sizes. */
size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/* Backward. Inputs q, k, v, o (from fa_fwd), dO and lse (from fa_fwd); outputs dq, dk, dv
 * (bf16 [B,H,N,d]). workspace: caller-owned device memory of at least
 * fa_bwd_workspace_size(B,H,N,d) bytes, 16-byte aligned; its contents on entry do not matter.
 * Calls that share a workspace must be ordered (one stream, or events between streams). */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                 const float* lse, void* dq, void* dk, void* dv, void* workspace,
                 size_t workspace_bytes, int B, int H, int N, int d, float scale, int causal,
                 void* stream);

/* Backward that allocates nothing (no counterpart in the paper: it exists for callers).
 * Some callers cannot allocate device memory: a plugin running inside a framework that has
 * reserved the GPU's memory for its own pool and hands out no workspace, or a service that
 * must not allocate after start-up to keep its latency and memory footprint fixed. They call
 * this instead of fa_bwd: same arguments without the workspace, same results.
 * The scratch (fp32 dQ accumulator, per-row terms, work-unit counter) is a 64 MiB array built
 * into the library:
 * every GPU that loads the library holds it until the process exits. Sizes whose
 * fa_bwd_workspace_size exceeds 64 MiB (67108864 bytes) are rejected with FA_ERR_UNSUPPORTED
 * and nothing is launched. This call performs no cudaMalloc, cudaFree or other allocation.
 * Set-up: the first call on a device (with that device current) looks up the scratch's device
 * address once; make that first call before any stream capture.
 * All calls on a device share the one scratch array, which keeps the last call's contents (each
 * call rewrites what it reads before reading it): calls that overlap on the GPU (different
 * streams, or host threads, without ordering between them) race on it and must be serialised
 * by the caller. A timed-out in-kernel wait (the hang guard) is recorded in a status word
 * built into the library, which fa_check_status reads and clears (it allocates nothing). */
fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                         const void* dO, const float* lse, void* dq, void* dk, void* dv, int B,
                         int H, int N, int d, float scale, int causal, void* stream);

/* Failure-detection self-test: launches on `stream` a one-thread kernel that waits, through the
 * same bounded wait the attention kernels use, on a barrier nothing ever completes. After
 * limit_us microseconds (1 .. 10^7) the wait gives up, FA_ERR_TIMEOUT is recorded in the
 * device status word and the kernel returns; the GPU is neither faulted nor hung. A following
 * fa_check_status(stream) returns FA_ERR_TIMEOUT and clears the word. */
fa_status fa_selftest_timeout(int limit_us, void* stream);

/* Failure-detection test hook (off unless called): arms, for the calling thread, the next launch
 * of kernel kind `kind` (0 = attention forward, 2 = backward main kernel; numbering as in
 * fa_profile_read). In that launch the TMA producer of every CTA leaves out one load (for the
 * forward, K/V tile load number `skip` of the CTA; for the backward, the query tile of the
 * CTA's iteration `skip`), and the MMA warp waits at most limit_us microseconds (1 .. 10^7).
 * Its wait for the missing tile runs out; the kernel lets the copies and products it issued
 * finish, frees its tensor memory, records FA_ERR_TIMEOUT in the status word and returns,
 * without faulting or hanging the GPU. The outputs of that call are undefined; a following
 * fa_check_status returns FA_ERR_TIMEOUT. The launch disarms the hook; kind = -1 disarms it
 * without a launch. A CTA that issues fewer loads than `skip` runs normally. */
fa_status fa_debug_stall_next(int kind, int skip, int limit_us);

/* Synchronises `stream`, then reads and clears the current device's status words: the one
 * the allocating entry points write (if it has been created) and the one built into the
 * library for fa_bwd_noalloc (if that entry point has been set up on this device). Allocates
 * no device memory. Returns FA_OK, FA_ERR_TIMEOUT, or FA_ERR_CUDA. */
fa_status fa_check_status(void* stream);

/* FP8 forward: q8, k8, v8 hold E4M3 codes (OCP 8-bit floating point, the "e4m3fn" encoding:
 * bias 7, no infinities, largest finite 448) in the layouts of fa_attn_shape, one byte per
 * element; the value of each element is its E4M3 value times the tensor's descale factor
 * (finite, > 0). Computes the same O (bf16) and lse (fp32) as fa_fwd_ex on those values, with
 * both products on 8-bit tensor cores: S = Q K^T accumulates exact E4M3 products in fp32, and
 * the probabilities are rounded to E4M3 for the product with V (O is normalised by the sum of
 * the rounded weights; lse uses the unrounded sum). The pages name FP8 only as a feature of a
 * later FlashAttention version ("How does FlashAttention optimize memory and speed via
 * tiling?", "Interview tips"); this entry point is that reading of it. Forward only; no
 * dropout; d in {64, 96, 128}; B * H_kv <= 65535. The workspace (caller-owned, at least
 * fa_fwd_fp8_workspace_size bytes, 16-byte aligned; 0 for an invalid shape) receives V
 * transposed to [B, H_kv, d, N_kv rounded up to 16]. Errors as fa_fwd_ex, and
 * FA_ERR_WORKSPACE for a missing or short workspace. */
size_t fa_fwd_fp8_workspace_size(const fa_attn_shape* shape);
fa_status fa_fwd_fp8(const void* q8, const void* k8, const void* v8, float q_descale,
                     float k_descale, float v_descale, void* o, float* lse,
                     const fa_attn_shape* shape, void* workspace, size_t workspace_bytes,
                     void* stream);

/* Optional device-side timing of the library's own kernels, for benchmarks and tracing.
 * While enabled on the calling thread, every kernel the library launches is bracketed by a
 * pair of CUDA events recorded on its launch stream. fa_profile_read() waits for those events
 * and writes, per kernel kind k (0 = forward, 1 = backward preprocess, 2 = backward main,
 * 3 = backward dQ conversion, 4 = FP8 forward, 5 = FP8 V transpose, 6 = d = 256 forward,
 * 7 = d = 256 backward dV pass, 8 = d = 256 backward dK/dQ pass; FA_KERNEL_KINDS in total), the number of launches to
 * launches[k] and their summed device time in milliseconds to ms[k], then forgets them.
 * n is the length of both arrays (>= FA_KERNEL_KINDS). Events are created by the library and
 * reused; no device memory is allocated. */
#define FA_KERNEL_KINDS 9
fa_status fa_profile_enable(int on);
fa_status fa_profile_read(double* ms, long long* launches, int n);
/* Name of kernel kind k ("" if out of range). */
const char* fa_kernel_name(int kind);

/* Human-readable description of the last error returned on this thread ("" if none). */
const char* fa_last_error_string(void);

/* Library version string. */
const char* fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
