/*
 * pisa.h - C ABI of the B200 (sm_100a) PISA piecewise sparse attention forward.
 *
 * The method (gist.science technical summary of "PISA: Piecewise Sparse
 * Attention Is Wiser for Efficient Diffusion Transformers", section 2
 * "Method"; AI Radio episode summary of the same paper):
 *   Q, K, V are cut into blocks of B tokens.  For query block i the KV blocks
 *   split into a selected set S_i (exact softmax attention) and the rest U_i,
 *   which enter the same softmax numerator N_t and denominator D_t through a
 *   block-wise zeroth-order Taylor term (key centroid kbar_j, value sum
 *   sigma_j) plus one global first-order correction s * beta_t * (q_t Hbar),
 *   Hbar being the mean of the block-wise first-order matrices H_j and beta_t
 *   the sum of the U_i weights alpha_{t,j} = exp(s q_t . kbar_j).  o_t = N_t/D_t.
 *   S_i is the top-k of a covariance-aware score that uses M_j = ||H_j - Hbar||.
 *
 * Conventions shared by every entry point:
 *   - Tensors are dense row-major.  q, k, v, out: [batch, heads, L, d]
 *     (element type given by `dtype`; out has the input type).  Per-block
 *     statistics: [batch, heads, nb, d] float32 with nb = ceil(L / block);
 *     Hbar: [batch, heads, d, d] float32 (row = key dimension, column = value
 *     dimension); M: [batch, heads, nb] float32; sel: [batch, heads, nb, k]
 *     int32, each row ascending.
 *   - All pointers except `stream` are DEVICE pointers owned by the caller,
 *     16-byte aligned.  The library never allocates device memory; scratch
 *     space comes from the caller's `workspace` (size from the *_workspace_size
 *     query).  `stream` is a cudaStream_t passed as void* (NULL = legacy default).
 *   - Calls are asynchronous on `stream`.  Arguments are validated on the host
 *     before any launch; a rejected call launches nothing and returns an error.
 *     Launch failures return PISA_ERR_CUDA.  Device-side checks (bounded waits,
 *     index checks) record an error word read by pisa_device_status().
 *   - Supported: d in {64, 128}, block in {64, 128}, 1 <= L, 1 <= k <= nb,
 *     batch*heads >= 1.  The softmax scale is fixed at 1/sqrt(d).
 *   - Reading of the pages used throughout: scores carry the scale s=1/sqrt(d)
 *     (also inside the first-order term); H_j = sum_n (k_n - kbar_j)^T v_n (a
 *     sum, d x d); Hbar is the plain mean of H_j over all nb blocks of the
 *     (batch, head); beta_t = sum_{j in U_i} alpha_{t,j}; the norm in M_j is
 *     Frobenius; a partial last block keeps its true size n_j.
 */
#ifndef PISA_H
#define PISA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pisa_status {
  PISA_OK = 0,
  PISA_ERR_INVALID_ARG = -1,  /* null pointer, bad size, misaligned pointer */
  PISA_ERR_UNSUPPORTED = -2,  /* d or block outside the supported set      */
  PISA_ERR_WORKSPACE = -3,    /* workspace missing or smaller than needed  */
  PISA_ERR_CUDA = -4,         /* a CUDA runtime call or launch failed      */
  PISA_ERR_TIMEOUT = -5,      /* a bounded device wait ran out             */
  PISA_ERR_DEVICE_CHECK = -6  /* a device-side index check failed          */
} pisa_status;

typedef enum pisa_dtype {
  PISA_BF16 = 0,
  PISA_FP32 = 1
} pisa_dtype;

/* Routing score used by pisa_select_route. */
typedef enum pisa_route {
  PISA_ROUTE_COVARIANCE = 0,  /* s qbar.kbar + ln(n_j + s ||qbar|| M_j): the default   */
  PISA_ROUTE_POOLED = 1       /* s qbar.kbar + ln n_j: no covariance term (M unused) */
} pisa_route;

/* Text of a status code (static storage, never NULL). */
const char* pisa_status_string(pisa_status status);

/* Number of exactly computed KV blocks per query block for a keep ratio rho:
 * k = clamp(ceil(rho * nb - 1e-9), 1, nb), nb = ceil(L / block), computed in
 * double from the float argument.  Returns -1 for L < 1, block < 1 or a
 * non-finite / non-positive rho. */
int pisa_keep_count(int L, int block, float keep_ratio);

/* Scratch bytes pisa_block_stats needs (per-chunk partial sums of H_j). */
size_t pisa_stats_workspace_size(int batch, int heads, int L, int d, int block);

/* Scratch bytes pisa_attn_fwd_with_sel needs (centroid and Hbar operands in
 * the fused kernel's input format). */
size_t pisa_fused_workspace_size(int batch, int heads, int L, int d, int block);

/* Scratch bytes pisa_attn_fwd needs for all stages with k selected blocks. */
size_t pisa_workspace_size(int batch, int heads, int L, int d, int block, int k);

/* Block statistics (gist.science summary, section 2, hardware implementation:
 * the precompute of block centroids, value sums and Hbar).
 *   qbar[i] = mean of the query rows of block i   (pooled query, routing only)
 *   kbar[j] = mean of the key rows of block j      (centroid)
 *   vsum[j] = sum of the value rows of block j     (sigma_j)
 *   hbar    = (1/nb) sum_j H_j,  H_j = sum_n (k_n - kbar_j)^T v_n
 * Reads q, k, v once.  hbar is reduced in a fixed order (no float atomics), so
 * results are bit-reproducible.  workspace >= pisa_stats_workspace_size(). */
pisa_status pisa_block_stats(const void* q, const void* k, const void* v, pisa_dtype dtype,
                             int batch, int heads, int L, int d, int block,
                             float* qbar, float* kbar, float* vsum, float* hbar,
                             void* workspace, size_t workspace_bytes, void* stream);

/* Covariance norm for routing (gist.science summary, section 2,
 * covariance-aware routing): M[j] = ||H_j - Hbar||_F, recomputing each H_j from
 * k, v and the stats of pisa_block_stats instead of storing all of them. */
pisa_status pisa_cov_norm(const void* k, const void* v, pisa_dtype dtype,
                          int batch, int heads, int L, int d, int block,
                          const float* kbar, const float* vsum, const float* hbar,
                          float* M, void* stream);

/* Block-wise first-order matrices H_j, written out: H [batch, heads, nb, d, d]
 * float32.  Not on the attention path (which never stores them); for
 * inspection and tests. */
pisa_status pisa_block_first_order(const void* k, const void* v, pisa_dtype dtype,
                                   int batch, int heads, int L, int d, int block,
                                   const float* kbar, const float* vsum, float* H,
                                   void* stream);

/* Covariance-aware top-k routing (AI Radio summary: Score_{t,j}; gist.science
 * summary, section 2, covariance-aware routing).  Score of KV block j for
 * query block i:
 *     score = s * qbar_i . kbar_j + ln(n_j + s * ||qbar_i||_2 * M_j)
 * (reading: log of the block's zeroth-order mass times its size plus the
 * Cauchy-Schwarz bound of the first-order error left by Hbar).  sel[i] = the k
 * largest scores, exact ties to the smaller j, stored ascending.  Scores are
 * float32. */
pisa_status pisa_select(const float* qbar, const float* kbar, const float* M,
                        int batch, int heads, int L, int d, int block, int k,
                        int32_t* sel, void* stream);

/* Routing with a chosen score (variants of the routing reading, for
 * comparison; gist.science summary, section 2, covariance-aware routing).
 * PISA_ROUTE_COVARIANCE is exactly pisa_select.  PISA_ROUTE_POOLED drops the
 * covariance term (M_j = 0): score = s qbar_i . kbar_j + ln n_j, plain pooled
 * block-sparse routing; M is not read and may be NULL.  Any other route value
 * returns PISA_ERR_INVALID_ARG. */
pisa_status pisa_select_route(const float* qbar, const float* kbar, const float* M,
                              int batch, int heads, int L, int d, int block, int k,
                              pisa_route route, int32_t* sel, void* stream);

/* Covariance norm read as the spectral norm (gist.science summary, section
 * 2: ||H_j - Hbar||_2 as the largest singular value; the default,
 * pisa_cov_norm, reads it as the Frobenius norm).  H: the block-wise
 * matrices of pisa_block_first_order [batch, heads, nb, d, d] float32; hbar
 * from pisa_block_stats; M [batch, heads, nb] float32.  One CTA per block forms
 * G = (H_j - Hbar)^T (H_j - Hbar) and runs power iteration on it until its
 * Rayleigh quotient changes by less than 1e-7 relative (at most 4000 steps);
 * M_j = sqrt(lambda_max(G)), float32. */
pisa_status pisa_cov_norm_spectral(const float* H, const float* hbar, int batch, int heads, int L,
                                   int d, int block, float* M, void* stream);

/* The fused forward for a given selection (gist.science summary, section 2:
 * core algorithm, N_t equation; hardware implementation phases 1-3).  For
 * every query row t of block i, in one online softmax:
 *   exact:  x = s q_t . k_n for the tokens of the blocks in sel[i]
 *   approx: y = s q_t . kbar_j for the other blocks, weight e^y, mass n_j e^y,
 *           value sum vsum_j, beta_t += e^y
 *   out_t = (sum e^x v_n + sum e^y vsum_j + s beta_t (q_t hbar))
 *           / (sum e^x + sum n_j e^y)
 * kbar, vsum, hbar as produced by pisa_block_stats; sel as produced by
 * pisa_select (entries in [0, nb), ascending, no repeats).
 * workspace >= pisa_fused_workspace_size(). */
pisa_status pisa_attn_fwd_with_sel(const void* q, const void* k, const void* v, void* out,
                                   pisa_dtype dtype, int batch, int heads, int L, int d,
                                   int block, const float* kbar, const float* vsum,
                                   const float* hbar, const int32_t* sel, int k_sel,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* The whole forward: block stats -> covariance norm -> routing -> fused
 * attention, with k = pisa_keep_count(L, block, keep_ratio).
 * workspace >= pisa_workspace_size(batch, heads, L, d, block, k). */
pisa_status pisa_attn_fwd(const void* q, const void* k, const void* v, void* out,
                          pisa_dtype dtype, int batch, int heads, int L, int d, int block,
                          float keep_ratio, void* workspace, size_t workspace_bytes,
                          void* stream);

/* Device workspace bytes pisa_attn_fwd_host needs when it works through the
 * (batch, head) slices `chunk` at a time: the scratch of pisa_attn_fwd for
 * one chunk plus two device staging copies of a chunk's q, k, v and out.
 * Returns 0 for unsupported shapes or dtype, k outside [1, nb] or chunk < 1. */
size_t pisa_host_workspace_size(pisa_dtype dtype, int batch, int heads, int L, int d, int block, int k,
                                int chunk);

/* pisa_attn_fwd for tensors that live in HOST memory.  The pages describe the
 * forward only; this entry point is an interface convenience for callers whose
 * q, k, v and out are host-resident, and it overlaps the PCIe copies with the
 * compute instead of running copy, compute, copy back to back.
 *   q_host, k_host, v_host, out_host: [batch, heads, L, d] in host memory, the
 *   element type of `dtype`.  workspace: device memory owned by the caller,
 *   16-byte aligned, >= pisa_host_workspace_size(dtype, ..., k, chunk) with
 *   k = pisa_keep_count(L, block, keep_ratio).
 *   The batch*heads slices go through in chunks of `chunk` consecutive slices
 *   (the last chunk may be shorter).  For each chunk: the inputs are copied in
 *   on an internal copy stream, the whole forward (stats, covariance norm,
 *   routing, fused attention) runs on `stream`, and the output is copied back
 *   on a second internal copy stream.  Two staging buffers let the next
 *   chunk's input copy and the previous chunk's output copy run while a chunk
 *   computes.
 *   - Asynchronous: returns once everything is enqueued; `stream` reaches the
 *     end of the last output copy only when all copies and kernels are done.
 *     The host buffers must stay valid and untouched until then.
 *   - Host buffers should be page-locked (cudaHostAlloc / cudaHostRegister)
 *     for the copies to overlap; pageable memory works but copies stall the
 *     host.
 *   - Each slice is computed by the same kernels as in pisa_attn_fwd.  The
 *     fixed-order partial sums behind Hbar are grouped by the number of slices
 *     per launch, so results can differ from one whole-batch pisa_attn_fwd
 *     call in the last bits unless chunk >= batch*heads.
 *   - The library keeps, per device, two non-blocking copy streams and a few
 *     events, created on the first call on that device and kept until exit.
 *     Calls on one device are enqueued under a lock and share those streams.
 *   - Arguments are validated before any CUDA call: null pointers or chunk < 1
 *     give PISA_ERR_INVALID_ARG, a missing or small workspace
 *     PISA_ERR_WORKSPACE; a failing copy or launch gives PISA_ERR_CUDA. */
pisa_status pisa_attn_fwd_host(const void* q_host, const void* k_host, const void* v_host,
                               void* out_host, pisa_dtype dtype, int batch, int heads, int L,
                               int d, int block, float keep_ratio, int chunk, void* workspace,
                               size_t workspace_bytes, void* stream);

/* The forward with each unselected block's own first-order term instead of
 * the shared one: N_t = sum_{S_i} e^{x} v + sum_{j in U_i} alpha_{t,j}
 * (sigma_j + s q_t H_j), D_t as in pisa_attn_fwd_with_sel (gist.science
 * technical summary, section 2: the hybrid-order paragraph starts from these
 * per-block terms and replaces H_j by Hbar to avoid loading them).  For the
 * accuracy / cost comparison between the two: it costs (nb - k) d^2
 * multiply-adds per query row and reads H, so it runs on CUDA cores and is
 * meant for small shapes (a few thousand tokens); the production path is
 * pisa_attn_fwd_with_sel.
 *   H:   [batch, heads, nb, d, d] float32, the block-wise first-order
 *        matrices H_j (pisa_block_first_order).
 *   Other arguments as pisa_attn_fwd_with_sel; no workspace.  Validation
 *   errors as there. */
pisa_status pisa_attn_fwd_blockwise_with_sel(const void* q, const void* k, const void* v, void* out,
                                             pisa_dtype dtype, int batch, int heads, int L, int d,
                                             int block, const float* kbar, const float* vsum,
                                             const float* H, const int32_t* sel, int k_sel, void* stream);

/* Size in bytes of the fixed device scratch array used by
 * pisa_attn_fwd_with_sel_noalloc (32 MiB). */
#define PISA_NOALLOC_SCRATCH_BYTES (32ull * 1024ull * 1024ull)

/* pisa_attn_fwd_with_sel for callers that cannot allocate device memory: code
 * that is handed only its input and output buffers (a plugin inside another
 * framework's memory pool, a pre-allocated serving runtime, a captured
 * sequence that forbids cudaMalloc), where no workspace can be created.  The
 * paper has no counterpart; this is an interface convenience.
 *
 * Same arguments and results as pisa_attn_fwd_with_sel minus the workspace.
 * The scratch that pisa_attn_fwd_with_sel takes from the caller's workspace
 * (the tensor-core kernel's bf16 copies of kbar, vsum and Hbar) lives
 * instead in one device array of PISA_NOALLOC_SCRATCH_BYTES compiled into the
 * library; every GPU that loads the library holds that memory until the
 * process exits.
 *   - A bf16 call whose scratch need, pisa_fused_workspace_size(batch, heads,
 *     L, d, block), exceeds PISA_NOALLOC_SCRATCH_BYTES is rejected with
 *     PISA_ERR_WORKSPACE before anything is launched.  fp32 calls (the
 *     CUDA-core kernel) use no scratch and have no such limit.
 *   - The kernels and their operands are those of pisa_attn_fwd_with_sel, so
 *     the output is bit-identical to it.
 *   - It calls no allocating routine (no cudaMalloc, cudaFree or library
 *     allocator).
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.
 *   - All calls share the one array, which keeps what the last call wrote.
 *     Each call rewrites every scratch byte it later reads, so nothing needs
 *     to start at zero; but calls that overlap on the GPU (other streams,
 *     other host threads) race on the array and must be serialised by the
 *     caller. */
pisa_status pisa_attn_fwd_with_sel_noalloc(const void* q, const void* k, const void* v, void* out,
                                           pisa_dtype dtype, int batch, int heads, int L, int d,
                                           int block, const float* kbar, const float* vsum,
                                           const float* hbar, const int32_t* sel, int k_sel,
                                           void* stream);

/* Launch tuning.  A few launch parameters change only speed, never a
 * result bit: the covariance-norm kernel's blocks per CTA (each M_j comes from
 * its own block), the routing kernel's query blocks per CTA (rows are scored
 * and selected independently) and the fused kernel's persistent CTA count
 * (each pair of query tiles is computed by one CTA).  They are kept per
 * (device, batch*heads, L, d, block); 0 in a field means the built-in
 * heuristic.  Block size and the H-bar partial-sum grouping are not tuned:
 * they would change results. */
typedef struct pisa_tuning {
  int cov_blocks_per_cta;   /* >= 0 */
  int select_rows_per_cta;  /* 0..32: the tensor-core routing kernel runs 32 (values
                               above 16 or 0) or 16 (1..16) query blocks per CTA; the
                               CUDA-core one, for nb too large for the former, up to
                               what fits in shared memory */
  int fused_ctas;           /* >= 0, capped by the SM count and the pairs of query tiles */
} pisa_tuning;

/* Times candidate values of each parameter on the given inputs (one
 * parameter at a time, the others fixed; CUDA events on `stream`, three runs
 * after a warm-up), keeps the fastest for this shape on the current device and
 * returns it in `chosen` (may be NULL).  Blocking: synchronises `stream`.
 * Runs the whole forward along the way: `out` receives its result.  Same
 * arguments and workspace as pisa_attn_fwd. */
pisa_status pisa_autotune(const void* q, const void* k, const void* v, void* out, pisa_dtype dtype,
                          int batch, int heads, int L, int d, int block, float keep_ratio,
                          void* workspace, size_t workspace_bytes, void* stream, pisa_tuning* chosen);

/* Sets (t != NULL) or clears (t == NULL) the tuning of a shape on the current
 * device; fields outside their ranges give PISA_ERR_INVALID_ARG. */
pisa_status pisa_set_tuning(int batch, int heads, int L, int d, int block, const pisa_tuning* t);

/* The tuning in force for a shape on the current device (all zero when none). */
pisa_status pisa_get_tuning(int batch, int heads, int L, int d, int block, pisa_tuning* t);

/* Writes the current device's tunings to a text file (one shape per line) /
 * reads such a file into the current device's table.  A malformed file is
 * rejected whole (PISA_ERR_INVALID_ARG) and changes nothing. */
pisa_status pisa_tuning_save(const char* path);
pisa_status pisa_tuning_load(const char* path);

/* Sets the limit of the bounded waits in the tensor-core kernels on the
 * current device, in nanoseconds of the GPU's global timer; 0 restores the
 * default of 2 s.  Every mbarrier wait between the warps of a CTA (operand
 * tiles landed, MMAs done, softmax done, work list ready) gives up after this
 * long: the CTA then records PISA_ERR_TIMEOUT in the device error word,
 * lets the copies and MMAs it already issued complete (a separate fixed 2 s
 * bound that this setting does not shorten), frees its tensor memory and
 * exits, so the context stays usable.  The result of such a call is
 * undefined; pisa_device_status reports the timeout.  A limit shorter than
 * the time a healthy copy or MMA takes (microseconds) makes ordinary calls
 * time out: it exists to exercise that path in tests and to tighten the bound
 * on a stuck kernel.  Applies to kernels launched after it; blocking:
 * synchronises `stream`.  Not part of the method (the pages have no
 * counterpart).  Returns PISA_OK or PISA_ERR_CUDA. */
pisa_status pisa_set_wait_limit(uint64_t limit_ns, void* stream);

/* Reads (and, when reset != 0, clears) the device error word that bounded
 * waits and index checks set.  Synchronises `stream`.  Returns PISA_OK,
 * PISA_ERR_TIMEOUT, PISA_ERR_DEVICE_CHECK or PISA_ERR_CUDA. */
pisa_status pisa_device_status(void* stream, int reset);

#ifdef __cplusplus
}
#endif

#endif /* PISA_H */
