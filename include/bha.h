/*
 * libbha — block-hybrid attention for blockwise diffusion-LM decoding (C ABI).
 *
 * The operation ("Retrofitting Linear Attention into Diffusion Language Models", §3.1):
 * every query of the active block gets exact bidirectional softmax attention over the
 * block's own tokens, and reads all committed blocks only through fixed-size Hedgehog
 * linear-attention states
 *     S = sum_t phi(k_t) v_t^T   (F x d, fp32)      Z = sum_t phi(k_t)   (F, fp32)
 *     phi(x) = [softmax(xW), softmax(-xW)]           (W: d x F/2, per KV head)
 * and the two branches share one normaliser:
 *     out = (w sm_num + lin_num) / (w sm_den + lin_den),  w = sigmoid(alpha_h)
 *     sm_num = sum_{j in block} exp(q.k_j/sqrt d) v_j,  sm_den = sum_j exp(q.k_j/sqrt d)
 *     lin_num = phi(q)^T S,  lin_den = phi(q)^T Z.
 * A finished block is folded into the states by S += sum_t phi(k_t) v_t^T, Z += sum_t phi(k_t).
 *
 * Conventions shared by every call
 * --------------------------------
 * - Notation: R requests, Hq query heads, Hkv KV heads (Hq % Hkv == 0, G = Hq / Hkv), head
 *   dimension d, total feature dimension F (even; W is d x F/2), block rows b_r <= max_block.
 *   Query head h reads KV head / weight / state group g = floor(h / G).
 * - Token-major ragged activations: Q [T][Hq][d], K and V [T][Hkv][d], O [T][Hq][d];
 *   request r owns rows cu_blk[r] .. cu_blk[r+1]-1 (cu_blk is a DEVICE int32 array of R+1
 *   entries with cu_blk[0] = 0, non-decreasing, cu_blk[R] = T, each gap <= max_block).
 * - States: S [num_slots][Hkv][F][d] fp32 and Z [num_slots][Hkv][F] fp32, row-major.
 *   Request r uses slot state_slot[r] (DEVICE int32 [R]) or slot r when state_slot is NULL.
 * - W [Hkv][d][F/2] row-major in the activation dtype; alpha [Hq] fp32 or NULL (w = 1).
 * - Every call works on the CURRENT CUDA device (cudaGetDevice): its launches, tensor maps and
 *   device limits are those of that device, so all pointers and the stream must belong to it.
 * - All tensor pointers are DEVICE pointers, 16-byte aligned; the caller allocates and owns
 *   every buffer.  Outputs (O, phi) that are also 32-byte aligned are written in whole 32-byte
 *   sectors, which is faster; the results are the same bits either way.  The library allocates nothing, keeps no per-call state, never
 *   synchronises the stream, and enqueues its kernels on `stream` (a cudaStream_t; NULL is
 *   the legacy default stream).  Calls on different streams touching disjoint buffers may
 *   run concurrently.
 * - Return value: BHA_OK, or a negative bha_status from host-side validation (nothing is
 *   launched) or from the launch itself (BHA_ERR_CUDA).
 * - Device-detected problems (a malformed cu_blk, a block longer than max_block, a slot out
 *   of range, a bounded wait that ran out) are reported through dev_err: an optional DEVICE
 *   int32 that the kernels set to the first nonzero bha_status they meet (the caller
 *   zeroes it and reads it after synchronising).  The affected request is skipped; nothing
 *   traps.
 * - Outputs must not alias inputs.
 */
#ifndef BHA_H
#define BHA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BHA_OK = 0,
  BHA_ERR_INVALID = -1,     /* bad argument: null/misaligned pointer, bad dims, bad cu_blk */
  BHA_ERR_UNSUPPORTED = -2, /* valid but outside what the kernels implement               */
  BHA_ERR_CUDA = -3,        /* a CUDA runtime call or kernel launch failed                */
  BHA_ERR_TIMEOUT = -4      /* a bounded device-side wait gave up (reported via dev_err)  */
} bha_status;

typedef enum { BHA_BF16 = 0, BHA_F32 = 1 } bha_dtype;

typedef struct {
  int32_t num_requests; /* R >= 0                                                      */
  int32_t num_q_heads;  /* Hq >= 1, a multiple of num_kv_heads                         */
  int32_t num_kv_heads; /* Hkv >= 1: number of W matrices and of state heads           */
  int32_t head_dim;     /* d, 1..256                                                   */
  int32_t feature_dim;  /* F, even, 2..512; W is d x F/2                               */
  int32_t max_block;    /* B_max, 1..128: the longest active block                     */
  int32_t total_tokens; /* T = cu_blk[R], as known to the host                         */
  int32_t num_slots;    /* number of state slots in S/Z (>= R when state_slot is NULL) */
  int32_t act_dtype;    /* bha_dtype of Q, K, V, W, O and of x in bha_featuremap       */
} bha_dims;

/* Hedgehog feature map ("Retrofitting Linear Attention into Diffusion Language Models",
 * §3.1, phi(x) = [softmax(xW), softmax(-xW)], each half normalised over its F/2 entries).
 *   x    [T][x_heads][d]  activation dtype;  head h uses W[floor(h * Hkv / x_heads)]
 *   W    [Hkv][d][F/2]    activation dtype
 *   phi  [T][x_heads][F]  out_dtype (BHA_F32 or BHA_BF16)
 * Uses dims->{num_kv_heads, head_dim, feature_dim, total_tokens, act_dtype}.
 * bf16 x with d = 128, F = 256 and x_heads / num_kv_heads a power of two <= 128 (x_heads a
 * multiple of num_kv_heads) takes the tensor-core kernel; its bounded waits have no error word
 * here, so if one ever gave up the output of that call would be undefined (nothing traps).
 * bha_featuremap_checked reports that case. */
int bha_featuremap(const bha_dims* dims, const void* x, int32_t x_heads, const void* W,
                   void* phi, int32_t out_dtype, void* stream);

/* bha_featuremap with an error word: dev_err is a DEVICE int32 (4-byte aligned) or NULL.  The
 * tensor-core kernel writes BHA_ERR_TIMEOUT there if one of its bounded waits gave up (the
 * output of the call is then undefined); nothing is written otherwise, so the caller zeroes it
 * first.  Host-side validation and return values are those of bha_featuremap.  (ABI 1.01) */
int bha_featuremap_checked(const bha_dims* dims, const void* x, int32_t x_heads, const void* W,
                           void* phi, int32_t out_dtype, int32_t* dev_err, void* stream);

/* One denoising step of one block-hybrid layer (§3.1: within-block softmax sums, cross-block
 * read lin_num = phi(q)^T S, lin_den = phi(q)^T Z, and the gated shared-normaliser merge).
 *   cu_blk [R+1] device int32; state_slot [R] device int32 or NULL
 *   Q [T][Hq][d], K/V [T][Hkv][d], W [Hkv][d][F/2]: activation dtype
 *   S [num_slots][Hkv][F][d], Z [num_slots][Hkv][F]: fp32, read only
 *   alpha [Hq] fp32 or NULL (w = 1);  O [T][Hq][d] activation dtype, written
 * A row whose shared denominator is exactly 0 (w = 0 with empty states) is written as 0. */
int bha_hybrid_attn(const bha_dims* dims, const int32_t* cu_blk, const int32_t* state_slot,
                    const void* Q, const void* K, const void* V, const float* S,
                    const float* Z, const void* W, const float* alpha, void* O,
                    int32_t* dev_err, void* stream);

/* The last denoising step of a block fused with that block's commit (§3.1 block commit; in
 * §3.3 one kernel launch per step also performs the state update).
 *   Arguments, layouts and dev_err as in bha_hybrid_attn, except that S and Z are updated:
 *   O is the step's output over the states as passed in (the blocks committed before this
 *   one), and then, for each request, S += sum_t phi(k_t) v_t^T and Z += sum_t phi(k_t) over
 *   its block rows, as bha_commit_block does.  Two requests must not name the same slot.
 * The tensor-core kernel (the dims bha_hybrid_attn takes on tensor cores) reads each state
 * once for both parts; other dims run the generic decode step and commit as two launches. */
int bha_hybrid_attn_commit(const bha_dims* dims, const int32_t* cu_blk, const int32_t* state_slot,
                           const void* Q, const void* K, const void* V, float* S, float* Z,
                           const void* W, const float* alpha, void* O, int32_t* dev_err,
                           void* stream);

/* Block commit (§3.1: S_n = S_{n-1} + sum_{t in B_n} phi(k_t) v_t^T, Z_n likewise), in place.
 *   K/V [T][Hkv][d] activation dtype, W [Hkv][d][F/2]; S, Z updated in place (fp32).
 * Any b_r >= 0 is allowed (b_r = 0 leaves the slot untouched).  Two requests must not
 * name the same slot in one call.  bf16 with d = 128 and F = 256 runs on the tensor-core
 * kernel for every max_block up to 128 (its 128-row tiles hold 4, 2 or 1 requests of up to
 * 32, 64 or 128 tokens). */
int bha_commit_block(const bha_dims* dims, const int32_t* cu_blk, const int32_t* state_slot,
                     const void* K, const void* V, const void* W, float* S, float* Z,
                     int32_t* dev_err, void* stream);

/* Exact softmax attention over the whole KV cache: the softmax teacher the method replaces
 * (§2.2 softmax attention; every cached key of the request is visible, no mask), kept as
 * the comparison point for the prefix-length study (Appendix A).
 *   Q [T][Hq][d] activation dtype; O [T][Hq][d] activation dtype
 *   Kc/Vc [R][Hkv][kv_capacity][d] activation dtype; request r's keys are rows 0..kv_len[r]-1
 *   (its committed prefix followed by the active block); kv_len [R] device int32 in
 *   [0, kv_capacity]; kv_len[r] = 0 writes zeros.
 *   workspace: device scratch of at least bha_full_prefix_workspace_bytes(dims, kv_capacity)
 *   bytes (16-byte aligned), or NULL when that size is 0.  Its contents need no
 *   initialisation and are meaningless after the call. */
int bha_full_prefix_attn(const bha_dims* dims, const int32_t* cu_blk, const int32_t* kv_len,
                         const void* Q, const void* Kc, const void* Vc, int64_t kv_capacity,
                         void* O, void* workspace, size_t workspace_bytes, int32_t* dev_err,
                         void* stream);

/* Scratch bytes bha_full_prefix_attn needs for these dims and cache capacity. */
size_t bha_full_prefix_workspace_bytes(const bha_dims* dims, int64_t kv_capacity);

/* Size of the fixed scratch array behind bha_full_prefix_attn_noalloc (16 MiB). */
#define BHA_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

/* bha_full_prefix_attn without the caller-provided workspace.  The paper has no counterpart:
 * this exists for callers that cannot allocate device memory on the call path -- for
 * example a serving engine that reserves its whole memory budget up front and forbids
 * cudaMalloc inside the decode loop, or a plugin whose host owns all allocation.
 *   Arguments, layouts, results and dev_err behave exactly as in bha_full_prefix_attn.
 *   The split partials go to a file-scope device array of BHA_NOALLOC_SCRATCH_BYTES that
 *   every GPU loading the library holds until the process exits.  The call allocates
 *   nothing (no cudaMalloc / cudaFree and no allocating library routine).
 *   Returns BHA_ERR_UNSUPPORTED, launching nothing, when the call would need more scratch
 *   than that (bha_full_prefix_workspace_bytes(dims, kv_capacity) >
 *   BHA_NOALLOC_SCRATCH_BYTES).
 *   The first call on each device, with that device current, looks up the array's device
 *   address (cudaGetSymbolAddress); make that first call before any stream capture.
 *   All calls share the one array and it keeps the last call's contents (nothing in it has
 *   to start at zero), so calls whose kernels may overlap on the GPU -- different streams,
 *   or different host threads -- race on it and must be serialised by the caller. */
int bha_full_prefix_attn_noalloc(const bha_dims* dims, const int32_t* cu_blk,
                                 const int32_t* kv_len, const void* Q, const void* Kc,
                                 const void* Vc, int64_t kv_capacity, void* O, int32_t* dev_err,
                                 void* stream);

/* Self-test of the watchdog that bounds every wait inside the tensor-core kernels: launches
 * one CTA whose thread waits, through that same bounded wait, on an mbarrier nothing ever
 * arrives at.  After about limit_cycles SM cycles (1 .. 4e9) the wait gives up and the kernel
 * writes BHA_ERR_TIMEOUT to *dev_err (a DEVICE int32 the caller zeroes first), as a stalled
 * pipeline would; the context stays usable.  Returns BHA_ERR_INVALID for a NULL dev_err or a
 * limit out of range, else the launch status. */
int bha_selftest_bounded_wait(int64_t limit_cycles, int32_t* dev_err, void* stream);

/* Static description of a status code. */
const char* bha_status_string(int status);

/* Which kernel variant a call with these dims takes: 0 = generic CUDA-core kernel,
 * 1 = tensor-core (tcgen05/TMA) kernel.  which: 0 featuremap (for x_heads = num_q_heads),
 * 1 hybrid, 2 commit, 3 full prefix, 4 hybrid fused with the commit.  Negative on invalid
 * dims. */
int bha_kernel_variant(const bha_dims* dims, int32_t which);

/* Library ABI version (major * 100 + minor). */
int bha_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BHA_H */
