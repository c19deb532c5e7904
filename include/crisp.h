/*
 * crisp.h — C ABI of the CRISP sparse-prefill library (libcrisp.so) for NVIDIA B200 (sm_100a).
 *
 * The library computes the prefill hot path of CRISP ("CRISP: Cliff-awaRe Input-adaptive Sparse
 * Prefilling with Structural-Mass-Motivated Routing"): per-head index selection from a proxy
 * attention over the last query block, then causal attention restricted to the selected
 * (query block, key block) pairs.
 *
 * Conventions shared by every entry point
 *   - Q is bf16 [h_q][n][d], K and V are bf16 [h_kv][n][d], all contiguous, in device memory.
 *     GQA: q-head h reads kv-head h / (h_q / h_kv) (consecutive q-heads share a kv-head).
 *   - Supported shapes: d == 128, block == 128, anchors == 128, h_q a multiple of h_kv, any
 *     n >= 1 for attention alone (crisp_sparse_prefill, crisp_dense_prefill) and 128 <= n with
 *     N_b <= 8192 for anything that selects (crisp_select, crisp_prefill, crisp_select_noalloc).
 *     Anything else returns CRISP_ERR_UNSUPPORTED before any launch.
 *   - N_b = ceil(n / 128) is the number of blocks; when n is not a multiple of 128 the last
 *     query and key blocks are partial (their rows past n do not exist).
 *   - Ownership: the caller allocates every buffer (inputs, outputs, index, workspace); the
 *     library never allocates or frees memory and keeps no global mutable state. Calls on
 *     different streams are safe when each uses its own workspace.
 *   - All compute calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream). They return CRISP_OK once the work is enqueued. Errors found on the host are
 *     returned directly and nothing is launched; errors found on the device (a bounded wait
 *     that ran out, a failed self-check) are recorded in the workspace's status word and read
 *     with crisp_get_status().
 *   - Pointers must be 16-byte aligned (TMA requirement); the workspace 256-byte aligned.
 *   - The workspace's first 256 bytes hold the device status word: zero them once after
 *     allocating the workspace (e.g. cudaMemset); crisp_get_status() clears it after reading.
 *     The rest of the workspace needs no initialisation and may hold anything between calls.
 *   - Tracing: the launches sit inside NVTX push/pop ranges named "crisp_select" (with
 *     "proxy_pass", "route_threshold", "pooled_estimation" and "merge" nested in it),
 *     "crisp_attention", "crisp_dense_attention", "crisp_fp8_quantise" and
 *     "crisp_attention_fp8qk", so a profiler can pick a stage's kernels (for example
 *     ncu --nvtx --nvtx-include "crisp_select/"). Without a profiler attached they cost a call
 *     through a no-op pointer.
 */
#ifndef CRISP_H
#define CRISP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes: 0 is success, negative values are errors. */
enum {
  CRISP_OK = 0,
  CRISP_ERR_INVALID_ARG = -1,    /* null pointer, bad parameter value, misaligned pointer */
  CRISP_ERR_UNSUPPORTED = -2,    /* shape outside the supported set (see above) */
  CRISP_ERR_WORKSPACE = -3,      /* ws_bytes < crisp_workspace_size(...) */
  CRISP_ERR_CUDA = -4,           /* a CUDA runtime/driver call or a launch failed */
  CRISP_ERR_DEVICE_TIMEOUT = -5, /* a device-side wait exceeded its limit; the kernel exited */
  CRISP_ERR_OVERFLOW = -6,       /* sizes overflow the 32-bit index formats */
  CRISP_ERR_DEVICE_CHECK = -7    /* a device-side consistency check failed */
};

/*
 * Method parameters (CRISP paper §3.2, §4, §5; the per-head pseudocode of the rcap.io summary).
 *   block      query/key block size B (must be 128)
 *   anchors    sink window (first `anchors` keys) and recency window (last `anchors` keys) of
 *              the C_struct routing signal (must be 128)
 *   tau_proxy  route a head to Vertical-Slash iff C_struct >= tau_proxy
 *   alpha      Vertical-Slash keep rule: block j kept iff p[j] > alpha * mu (alpha >= 0)
 *   gamma      Pooled-Estimation coverage target of the global cumulative cut (gamma > 0;
 *              gamma >= 1 keeps every causal block)
 *   min_blocks minimum kept blocks per direction on Vertical-Slash heads (>= 0; 0 = off)
 * Rule switches (0 = CRISP, the default for a zero-initialised field):
 *   route_rule 0: C_struct >= tau_proxy. 1: FlexPrefill's router as the CRISP paper describes
 *              it (§2): VS iff JSD(a_bar, a_hat) >= tau_jsd, a_bar the softmax over key blocks of
 *              the last query block's mean query against the key-block means (1/sqrt(d) scale),
 *              a_hat the proxy's per-query mean pooled to blocks (p_v); natural logarithm.
 *   tau_jsd    threshold of route_rule 1 (finite, >= 0)
 *   vs_rule    0: the noise-floor keep rule above. 1: FlexPrefill's per-direction cut (§2):
 *              each direction keeps the shortest prefix of its blocks sorted (p desc, index asc)
 *              whose sum reaches gamma times the direction's total (first and last blocks are
 *              kept either way; min_blocks still tops up)
 *   floor_rule 0: mu is the mean residual mass above. 1: mu is the median of p[1..N_b-2] (the
 *              median floor of the paper's robustness discussion, §4 / Table 9)
 * Selection (crisp_select, crisp_prefill, crisp_select_noalloc) keeps per-head block arrays in
 * shared memory and supports N_b <= 8192 (n <= 1,048,576); larger n returns
 * CRISP_ERR_UNSUPPORTED. Attention alone (crisp_sparse_prefill, crisp_dense_prefill) has no
 * such limit. When n is not a multiple of 128 the proxy still takes the last 128 queries and
 * the anchors the first and last 128 keys; a partial last block pools and averages what it has.
 */
typedef struct {
  int32_t block;
  int32_t anchors;
  float tau_proxy;
  float alpha;
  float gamma;
  int32_t min_blocks;
  int32_t route_rule;
  float tau_jsd;
  int32_t vs_rule;
  int32_t floor_rule;
} crisp_params;

/*
 * Per-head index sets in CSR form, written by crisp_select / crisp_prefill and read by
 * crisp_sparse_prefill. All arrays are device memory owned by the caller.
 *   route    int32 [h_q]        1 = Vertical-Slash, 0 = Pooled-Estimation
 *   c_struct float [h_q]        C_struct of each head (CRISP §3.2)
 *   row_ptr  int32 [h_q][N_b+1] row qb of head h spans cols[h*cap + row_ptr[h][qb] ..
 *                               h*cap + row_ptr[h][qb+1]), cap = N_b*(N_b+1)/2
 *   cols     int32 [h_q][cap]   key-block indices, strictly ascending within a row, each <= qb
 *   debug    float [h_q][2*N_b+5] or NULL: p_v[N_b], p_s[N_b] (vertical and slash block
 *            masses, CRISP §4), then mu_v, mu_s, C_struct, the number of selected pairs, and
 *            the JSD of route_rule 1 (0 otherwise). With vs_rule 1, mu_v and mu_s hold the value
 *            of the last block each direction's cut kept.
 */
typedef struct {
  int32_t* route;
  float* c_struct;
  int32_t* row_ptr;
  int32_t* cols;
  float* debug;
} crisp_index;

/* Bytes of device workspace needed by every compute call for this shape (0 if unsupported). */
size_t crisp_workspace_size(int h_q, int h_kv, int n, int d, const crisp_params* params);

/*
 * Index selection (CRISP §2 proxy attention over the last query block; §3.2 C_struct routing;
 * §4 vertical/slash block pooling, noise floor mu = max(1-p[0]-p[-1],0)/(N_b-2), keep p[j] >
 * alpha*mu, union of both directions; Pooled-Estimation: pooled Q/K block scores, softmax,
 * global gamma cumulative cut). Writes every field of *out (debug if non-NULL).
 */
int crisp_select(const void* q, const void* k, int h_q, int h_kv, int n, int d,
                 const crisp_params* params, const crisp_index* out,
                 void* ws, size_t ws_bytes, void* stream);

/*
 * Block-sparse causal attention (CRISP §2: softmax(QK^T/sqrt(d) + M_S) V with M_S = 0 on the
 * selected blocks and -inf elsewhere; within a block, key j is visible to query i iff j <= i).
 * Reads idx->row_ptr and idx->cols; every row must contain at least one block <= qb. A row
 * that is empty, longer than qb+1, outside the head's column array, not strictly ascending or
 * holding a block outside [0, qb] is reported as CRISP_ERR_DEVICE_CHECK (crisp_get_status) and
 * never read out of bounds. idx->route may be NULL; when given, heads of one GQA group with the
 * same route (any non-zero value counts as 1) are scheduled together. It only affects speed.
 * o: bf16 [h_q][n][d]. lse: fp32 [h_q][n] natural-log sum-exp of the scaled logits, or NULL.
 */
int crisp_sparse_prefill(const void* q, const void* k, const void* v, int h_q, int h_kv, int n,
                         int d, const crisp_index* idx, void* o, float* lse,
                         void* ws, size_t ws_bytes, void* stream);

/*
 * Selection followed by block-sparse attention in one call. idx_out may be NULL, in which
 * case the index lives inside the workspace; otherwise it receives the index as crisp_select.
 */
int crisp_prefill(const void* q, const void* k, const void* v, int h_q, int h_kv, int n, int d,
                  const crisp_params* params, void* o, float* lse, const crisp_index* idx_out,
                  void* ws, size_t ws_bytes, void* stream);

/*
 * crisp_prefill over a batch of independent sequences packed along the token axis (a batch has
 * no counterpart on the pages, which treat one sequence; each sequence here is selected and
 * attended exactly as crisp_prefill would treat it alone).
 *   q: bf16 [h_q][total][d], k and v: bf16 [h_kv][total][d]; o: bf16 [h_q][total][d];
 *   lse: fp32 [h_q][total] or NULL. Sequence i is tokens cu_seqlens[i] .. cu_seqlens[i+1]-1 of
 *   every head.
 *   cu_seqlens: HOST int32 [n_seqs+1], cu_seqlens[0] = 0, non-decreasing, cu_seqlens[n_seqs] =
 *   total; every non-empty sequence needs >= 128 tokens (else CRISP_ERR_UNSUPPORTED); empty ones
 *   are skipped.
 *   ws: sized by crisp_workspace_size for the longest sequence; the sequences run one after
 *   another on `stream` and reuse it (their index sets live there and are not returned).
 * All checks happen before the first launch; a refused call launches nothing.
 */
int crisp_prefill_varlen(const void* q, const void* k, const void* v, int h_q, int h_kv, int total,
                         const int32_t* cu_seqlens, int n_seqs, int d, const crisp_params* params,
                         void* o, float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * Dense causal attention with the same kernel (every block <= qb selected): the reference
 * point for the sparse-versus-dense speed ratio. Same buffers as crisp_sparse_prefill.
 */
int crisp_dense_prefill(const void* q, const void* k, const void* v, int h_q, int h_kv, int n,
                        int d, void* o, float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * FP8 variant of the attention logits. The paper's pages quote an FP8 speedup only for another
 * method (FlashPrefill V2); this is an optional variant, not the headline path. Q and K are first
 * quantised to 8-bit E4M3 (the OCP 8-bit floating-point format: bias 7, 3 mantissa bits, largest
 * finite value 448) per head and 128-row block: amax = max |x|, inv = 448 / amax and
 * scale = amax / 448 (both rounded to fp32), code = E4M3(x * inv) with the product rounded to fp32
 * and the value rounded to the nearest E4M3 (ties to even, saturating at 448); an all-zero block
 * gets codes 0 and scale 1. The attention is then crisp_sparse_prefill's with S = Q K^T computed
 * on the codes (tensor cores, fp32 accumulation) and each logit multiplied by the two blocks'
 * scales: the exact attention of the dequantised Q and K up to the kernel's own rounding.
 *
 * crisp_fp8qk_buffer_size: bytes of the caller's buffer for the codes and scales, 0 for an
 *   unsupported shape. Layout, each part starting on a 256-byte boundary, in this order:
 *   Q codes uint8 [h_q][n][128], K codes uint8 [h_kv][n][128], Q scales float [h_q][N_b],
 *   K scales float [h_kv][N_b].
 * crisp_sparse_prefill_fp8qk: as crisp_sparse_prefill, plus fp8_buf (device, 256-byte aligned,
 *   at least crisp_fp8qk_buffer_size bytes; overwritten, and left holding the codes and scales).
 *   Errors as crisp_sparse_prefill; a missing or short buffer is CRISP_ERR_INVALID_ARG /
 *   CRISP_ERR_WORKSPACE.
 */
size_t crisp_fp8qk_buffer_size(int h_q, int h_kv, int n, int d);
int crisp_sparse_prefill_fp8qk(const void* q, const void* k, const void* v, int h_q, int h_kv, int n,
                               int d, const crisp_index* idx, void* o, float* lse, void* ws,
                               size_t ws_bytes, void* fp8_buf, size_t fp8_bytes, void* stream);

/*
 * Synchronises `stream`, returns the device status word of `ws` (CRISP_OK or the first device
 * error recorded since the last call) and clears it. Returns CRISP_ERR_CUDA if the
 * synchronisation itself fails.
 */
int crisp_get_status(void* ws, void* stream);

/* Static, human-readable name of a status code. */
const char* crisp_status_string(int status);

/*
 * Self-test of the device-side timeout path: launches one block that waits on a barrier
 * nothing signals, with a wait limit of `limit_ns` nanoseconds; the kernel then records
 * CRISP_ERR_DEVICE_TIMEOUT in the status word and exits. Nothing faults or hangs.
 */
int crisp_selftest_timeout(void* ws, size_t ws_bytes, uint64_t limit_ns, void* stream);

/*
 * Index selection that allocates nothing, for callers that must not call cudaMalloc: code running
 * under a memory manager that owns every device byte (a serving engine's pre-reserved pool), or a
 * latency-critical path that cannot afford the device synchronisation an allocation implies. The
 * paper has no counterpart; this is a deployment variant of crisp_select.
 *   - Same inputs and outputs as crisp_select; instead of a workspace it uses one scratch array of
 *     32 MiB inside the library (a file-scope device array: every GPU that loads the library holds
 *     it until the process exits). Shapes whose workspace (crisp_workspace_size) exceeds 32 MiB
 *     return CRISP_ERR_WORKSPACE without launching anything.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 *     that device current; make that first call before any stream capture. The address is kept
 *     for the life of the process: after cudaDeviceReset the library's module is loaded again
 *     and the kept address is stale, so a process that resets a device must not call this entry
 *     point on that device afterwards.
 *   - All calls share the array and it keeps the last call's contents; the call clears what must
 *     start at zero. Calls that overlap on the GPU (other streams, other threads) race on it.
 *   - device_status: NULL, or a device int the caller has zeroed; a device-side failure stores its
 *     negative status code there (first failure wins). With NULL such failures go unreported.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 */
int crisp_select_noalloc(const void* q, const void* k, int h_q, int h_kv, int n, int d,
                         const crisp_params* params, const crisp_index* out, int* device_status,
                         void* stream);

#ifdef __cplusplus
}
#endif

#endif /* CRISP_H */
