/*
 * libcce — Cut Cross-Entropy on NVIDIA B200 (sm_100a): the classifier matmul
 * fused with cross-entropy over a large vocabulary, forward and backward,
 * without ever writing the [N, V] logit matrix to device memory.
 *
 * What is computed (sources are web pages, cited by title and section):
 *   "The loss and the mask: Cut Cross-Entropy + FlexAttention (2 papers)",
 *   part "Cut Your Losses in Large-Vocabulary Language Models (CCE)",
 *   §Contribution: the cross-entropy of row i needs only the correct-token
 *   logit <h_i, e_{y_i}> (an indexed dot product) and the log-sum-exp of the
 *   row's logits z_ij = <h_i, e_j>, computed blockwise on chip while streaming
 *   over vocabulary tiles; loss_i = lse_i - <h_i, e_{y_i}>.  The backward
 *   recomputes the logits blockwise and drops softmax entries below bf16
 *   precision ("Cut Your Losses in Large-Vocabulary Language Models",
 *   research-map entry, §Approach).  §What transfers to us (third bullet) of
 *   the first page: a composite head composes the lse over several vocabulary
 *   segments with log-add-exp, and a dead gap between segments contributes
 *   -inf.
 *
 * Conventions shared by every entry point
 *   - Layouts are row-major and dense: H [N, D] bf16, E [V_s, D] bf16 per
 *     segment, y [N] int32.  D must be a positive multiple of 8 (16-byte rows,
 *     a TMA requirement) and at most 65536; every device pointer must be
 *     16-byte aligned.  0 <= N and 0 < V, both at most 2^31 - 257 (ids and
 *     row indices are int32 on the device).  Sizes outside these ranges give
 *     CCE_EINVAL, and a workspace size of 0.
 *   - All pointers except the ones marked "host" are device pointers.  The
 *     caller owns every buffer, including the workspace; the library never
 *     allocates device memory and never synchronises the stream.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  All work is enqueued asynchronously on it.
 *   - Return value: host-detectable errors (CCE_E*).  Errors found by the GPU
 *     while running are OR-ed as CCE_STATUS_* bits into *status (device int32,
 *     which the caller zeroes and reads after synchronising).  Device code
 *     never traps; every wait inside a kernel is bounded and reports
 *     CCE_STATUS_TIMEOUT instead of hanging.
 *   - Rows whose target equals ignore_index are skipped before any math:
 *     loss = lse = 0 and their dH row is 0.  A target outside [0, V) or inside
 *     a gap sets CCE_STATUS_BADTARGET and yields NaN loss, lse and dH row.
 */
#ifndef CCE_H_
#define CCE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes (host side). */
#define CCE_OK 0
#define CCE_EINVAL 1      /* bad shape, alignment, segment table or NULL pointer */
#define CCE_EWORKSPACE 2  /* workspace NULL or smaller than *_workspace_size()  */
#define CCE_ELAUNCH 3     /* a kernel launch or tensor-map encode failed          */
#define CCE_EDEVICE 4     /* no sm_100 device / driver entry point unavailable     */

/* Device status bits OR-ed into *status. */
#define CCE_STATUS_BADTARGET 1
#define CCE_STATUS_TIMEOUT 2

/* cce_bwd flags. */
#define CCE_KAHAN_DE 1u   /* dE += grad with a bf16 Kahan compensation buffer  */
#define CCE_FP32_GRADS 2u /* dH and dE are written as fp32 instead of bf16     */
#define CCE_FULL_DE 4u    /* filter only dH; the classifier gradient dE is full */
#define CCE_VOCAB_SHARD 8u /* E is one rank's vocabulary shard (see cce_fwd_shard) */
#define CCE_FP32_DH 16u   /* dH alone is written as fp32 (dE keeps its type)    */

#define CCE_MAX_SEGMENTS 8

/*
 * One live range of a composite classifier head.  Logical vocabulary ids
 * [vocab_begin, vocab_end) are rows 0 .. vocab_end - vocab_begin - 1 of E.
 * Ids covered by no segment form the dead gap (logit -inf).
 *   E       [vocab_end - vocab_begin, D] bf16, read only.
 *   dE      output of cce_bwd for this segment (bf16, or fp32 with
 *           CCE_FP32_GRADS); may be NULL for cce_fwd.
 *   dE_comp bf16 Kahan compensation, same shape as dE, read and updated
 *           only with CCE_KAHAN_DE (else ignored).
 * Segments must be sorted by vocab_begin, non-empty, non-overlapping and
 * inside [0, V); at most CCE_MAX_SEGMENTS.
 */
typedef struct cce_segment {
  int64_t vocab_begin;
  int64_t vocab_end;
  const void* E;
  void* dE;
  void* dE_comp;
} cce_segment;

/* Library version (major*10000 + minor*100 + patch). */
int cce_version(void);

/* Static text for a CCE_* return code. */
const char* cce_strerror(int code);

/*
 * Workspace bytes cce_fwd needs for these sizes (0 on invalid sizes).
 * n_segs = 0 means one segment [0, V).
 */
size_t cce_fwd_workspace_size(int64_t N, int64_t D, int64_t V, int32_t n_segs);

/*
 * Forward: per-row loss and log-sum-exp (natural log), fp32.
 *   H        [N, D] bf16 hidden states.
 *   E        [V, D] bf16 classifier, used when segs == NULL (one segment
 *            [0, V)); must be NULL when segs != NULL.
 *   y        [N] int32 targets (logical ids) or ignore_index.
 *   segs     host array of n_segs segments, or NULL / 0.
 *   loss,lse [N] fp32 outputs.
 *   colmax   optional [V_live] fp32 output, V_live = sum of segment sizes:
 *            the largest logit each live vocabulary row reaches over the
 *            valid rows (-inf if none), in segment order; the statistic
 *            cce_vocab_sort can order the vocabulary by.  NULL to skip.
 *   workspace, workspace_bytes  scratch of at least cce_fwd_workspace_size().
 *   status   device int32, OR-ed with CCE_STATUS_* bits.
 * Only rows with a valid target are computed; nothing of size N*V is ever
 * allocated or written.
 */
int cce_fwd(const void* H, const void* E, const int32_t* y,
            int64_t N, int64_t D, int64_t V, int32_t ignore_index,
            const cce_segment* segs, int32_t n_segs,
            float* loss, float* lse, float* colmax,
            void* workspace, size_t workspace_bytes,
            int32_t* status, void* stream);

/*
 * Forward over one vocabulary shard (vocabulary-parallel cross-entropy).
 * The live vocabulary given by E / segs is this rank's part of a vocabulary
 * of V ids split across ranks.  Per row it writes
 *   lse_part  the log-sum-exp over this shard's ids,
 *   zy_part   the correct-token logit <h_i, e_{y_i}> if this shard holds
 *             y_i, else 0.
 * Combining the ranks is plain arithmetic: lse = log-add-exp of lse_part
 * over ranks, z_y = sum of zy_part, loss = lse - z_y ("Cut Your Losses in
 * Large-Vocabulary Language Models", first page §Contribution: the loss
 * needs only the indexed logit and the log-sum-exp, and the log-sum-exp
 * composes blockwise; research-map entry §Limitations: log-add-exp of
 * partial results).  A target in [0, V) outside the shard is not an error
 * here; targets outside [0, V) set CCE_STATUS_BADTARGET and give NaN.
 * Ignored rows give 0 in both outputs.  Other arguments, the workspace
 * (cce_fwd_workspace_size) and errors as for cce_fwd.
 * The backward of a shard is cce_bwd with CCE_VOCAB_SHARD, the combined lse
 * and the same shard: it returns this shard's dE rows (complete) and this
 * shard's share of dH (to be summed over ranks); a target outside the shard
 * adds no one-hot term.
 */
int cce_fwd_shard(const void* H, const void* E, const int32_t* y,
                  int64_t N, int64_t D, int64_t V, int32_t ignore_index,
                  const cce_segment* segs, int32_t n_segs,
                  float* lse_part, float* zy_part, float* colmax,
                  void* workspace, size_t workspace_bytes,
                  int32_t* status, void* stream);

/*
 * Combine step of the vocabulary-parallel forward, run by every rank after
 * the all-gather of the shards' per-row parts.
 *   parts    [R, 2, N] fp32 device: for each of the R shards (ranks), the
 *            lse_part and zy_part rows of cce_fwd_shard.  A shard without
 *            vocabulary ids passes -inf and 0.
 *   y        [N] int32 targets.
 *   V, segs, n_segs  the whole head's logical vocabulary and live ranges
 *            (as for cce_fwd; only vocab_begin / vocab_end are read, E may
 *            be NULL); NULL / 0 = one range [0, V).
 *   loss,lse [N] fp32 outputs: lse = log-add-exp of lse_part over shards,
 *            loss = lse - sum of zy_part ("Cut Your Losses in Large-Vocabulary
 *            Language Models", research-map entry §Limitations: log-add-exp
 *            of partial results; first page §What transfers to us: the lse
 *            of a composite head composes over its parts, a dead gap adding
 *            -inf).  Ignored rows give 0; a target outside the live ranges
 *            (no shard holds it) gives NaN, as a bad target does in cce_fwd.
 * Returns CCE_EINVAL for R outside [1, 4096], bad ranges or a NULL pointer.
 */
int cce_vocab_combine(const float* parts, int32_t R, const int32_t* y, int64_t N, int64_t V,
                      int32_t ignore_index, const cce_segment* segs, int32_t n_segs,
                      float* loss, float* lse, void* stream);

/* Workspace bytes cce_bwd needs (0 on invalid sizes).  n_segs is the count
 * the cce_bwd call will pass (0 for a contiguous E): each segment can add one
 * partial vocabulary chunk to the sparse lists, so a workspace sized for fewer
 * segments than the call uses is rejected by the call with CCE_EWORKSPACE;
 * one sized for more (CCE_MAX_SEGMENTS, say) is always enough. */
size_t cce_bwd_workspace_size(int64_t N, int64_t D, int64_t V, int32_t n_segs,
                              uint32_t flags);

/*
 * The same workspace split by what each of its buffers scales with (host
 * pointers; the three add up to cce_bwd_workspace_size):
 *   rows    per-row arrays and [N, D] buffers (the compact copy of H, the
 *           fp32 dH accumulator),
 *   vocab   per-id arrays and [chunk, D] buffers of E rows,
 *   logits  buffers that hold parts of the [N, V] product: the bf16 G slab(s)
 *           of one vocabulary chunk (N x chunk width, the width capped so a
 *           slab stays below 512 MiB) and the sparse lists of kept entries.
 * The point of the method ("Cut Your Losses in Large-Vocabulary Language
 * Models", first page §Contribution: the logits are never written to global
 * memory in full) is that `logits` stays a small fraction of N x V x 2
 * bytes.  Returns CCE_OK or CCE_EINVAL.
 */
int cce_bwd_workspace_parts(int64_t N, int64_t D, int64_t V, int32_t n_segs, uint32_t flags,
                            size_t* rows, size_t* vocab, size_t* logits);

/*
 * Backward: gradients of sum_i dloss_i * loss_i.
 *   H, E, y, N, D, V, ignore_index, segs, n_segs  as for cce_fwd.
 *   lse      [N] fp32, the forward's lse output for the same inputs.
 *   dloss    [N] fp32 upstream gradient per row (1/N_valid on valid rows for
 *            a mean loss).
 *   filter_eps  softmax entries p_ij < filter_eps carry no gradient
 *            (element granularity; the target's one-hot term is never
 *            dropped); <= 0 turns filtering off.  2^-12 is bf16 precision.
 *            Tensor-core work is skipped on 16-wide blocks that are entirely
 *            zero after filtering.
 *   vocab_perm  optional [V_live] int32: for each segment, a permutation of
 *            its local rows (entries [off_s, off_s + n_s) permute
 *            0..n_s-1, off_s = sum of the sizes of earlier segments).  The
 *            backward walks the vocabulary in that order so that surviving
 *            blocks cluster; results do not depend on it beyond rounding.
 *            NULL = identity.  With a permutation the E rows of each
 *            vocabulary chunk are gathered on an internal stream (one per
 *            host thread and device, created on first use), one chunk ahead,
 *            ordered against `stream` by events; all of the call's work is
 *            still complete when work enqueued after it on `stream` runs.
 *   colmax   optional [V_live] fp32, the colmax output of cce_fwd on the
 *            same H, E, y and segments (a bound on every logit of each
 *            vocabulary row).  With filtering on (and without
 *            CCE_FULL_DE) a 128-row x 256-column tile of the backward whose
 *            bound  max colmax - min lse  over the tile lies below
 *            ln(filter_eps) by a margin is not recomputed: every softmax
 *            entry in it would be filtered, so only its one-hot entries are
 *            written: the block skip of the first page's §Contribution
 *            and of the research-map entry's §Approach, taken exactly.  The
 *            skip never changes which entries are kept.  A colmax that is not such a bound
 *            drops gradient entries.  NULL = no tile skip.
 *   flags    CCE_KAHAN_DE | CCE_FP32_GRADS | CCE_FULL_DE | CCE_VOCAB_SHARD |
 *            CCE_FP32_DH
 *            (CCE_VOCAB_SHARD: the backward of cce_fwd_shard: lse is the
 *            combined one, dH this shard's share; CCE_FP32_DH writes dH in
 *            fp32 while dE stays bf16 (or Kahan), for dH shares that are
 *            summed over ranks before rounding).  CCE_FULL_DE keeps
 *            the classifier gradient dE unfiltered while dH uses the filtered
 *            softmax (the "FullC" variant of "Cut Your Losses in
 *            Large-Vocabulary Language Models", research-map entry, §Key
 *            results / §Limitations), in every vocabulary chunk; it needs
 *            one more bf16 slab of workspace (see cce_bwd_workspace_size).
 *   dH       [N, D] output (bf16, or fp32 with CCE_FP32_GRADS).
 *   dE       [V, D] output when segs == NULL (else per-segment dE).  Written
 *            (overwritten) unless CCE_KAHAN_DE, in which case the new
 *            gradient g is added into the bf16 running sum s with the bf16
 *            compensation c (dE_comp): y' = g - c; t = s + y'; c = (t - s) - y';
 *            s = t, in fp32 arithmetic, each element owned by one thread
 *            (deterministic).  The caller zeroes s and c before the first
 *            accumulation.
 *   dE_comp  [V, D] bf16 compensation when segs == NULL and CCE_KAHAN_DE.
 *   debug_keep  optional [debug_rows, ceil(V/32)] uint32 bitmask: bit j%32 of
 *            word j/32 of row r is set when element (r, j) kept a non-zero
 *            softmax gradient (not filtered).  Rows are original row ids
 *            0..debug_rows-1.  NULL to skip.
 */
int cce_bwd(const void* H, const void* E, const int32_t* y,
            const float* lse, const float* dloss,
            int64_t N, int64_t D, int64_t V, int32_t ignore_index,
            const cce_segment* segs, int32_t n_segs,
            float filter_eps, const int32_t* vocab_perm, const float* colmax,
            uint32_t flags,
            void* dH, void* dE, void* dE_comp,
            uint32_t* debug_keep, int64_t debug_rows,
            void* workspace, size_t workspace_bytes,
            int32_t* status, void* stream);

/*
 * Soft-target KL divergence, never materialising either softmax ("The
 * Defensive Edit: Chunking Cross-Entropy Loss After an OOM Wake-Up Call",
 * §The OOM: A 12.2 GB Softmax Wall, where the soft KL between a student and a
 * teacher softmax over the vocabulary is the loss that needed chunking).
 * Per row i, with z_s = H_s E_s^T and z_t = H_t E_t^T (temperature 1; E_s and
 * E_t may be the same pointer):
 *   kl[i] = sum_j p_t,ij (log p_t,ij - log p_s,ij),  p = softmax(z).
 *   Hs, Ht   [N, D] bf16 student / teacher rows.
 *   Es, Et   [V, D] bf16 student / teacher classifiers.
 *   row_mask optional [N] int32: rows with 0 are skipped (kl = lse = 0,
 *            zero gradient); NULL = every row.
 *   kl, lse_s, lse_t  [N] fp32 outputs (the two log-sum-exps feed the
 *            backward).
 * Workspace and errors as for cce_fwd.
 */
size_t cce_kl_fwd_workspace_size(int64_t N, int64_t D, int64_t V);
int cce_kl_fwd(const void* Hs, const void* Es, const void* Ht, const void* Et,
               const int32_t* row_mask, int64_t N, int64_t D, int64_t V,
               float* kl, float* lse_s, float* lse_t,
               void* workspace, size_t workspace_bytes,
               int32_t* status, void* stream);

/*
 * Backward of sum_i dloss_i kl_i with the teacher held constant: the
 * gradients w.r.t. the student only, from G = dloss (p_s - p_t) through the
 * same dE / dH contractions as cce_bwd:
 *   dH = G E_s  ([N, D]),  dE = G^T H_s  ([V, D]).
 *   lse_s, lse_t  the forward's outputs for the same inputs.
 *   filter_eps  drops entry (i, j) when both p_s,ij and p_t,ij are below it
 *            (its gradient is then smaller than filter_eps); <= 0 = off.
 *   flags    CCE_FP32_GRADS and/or CCE_KAHAN_DE (with dE_comp) as for
 *            cce_bwd; CCE_FULL_DE and CCE_VOCAB_SHARD are rejected.
 *   debug_keep, debug_rows  optional per-element keep bits as for cce_bwd
 *            (set where the entry kept a non-zero gradient, i.e. where
 *            p_s or p_t reached filter_eps); NULL / 0 to skip.
 * Workspace: cce_kl_bwd_workspace_size(); errors as for cce_bwd.
 */
size_t cce_kl_bwd_workspace_size(int64_t N, int64_t D, int64_t V, uint32_t flags);
int cce_kl_bwd(const void* Hs, const void* Es, const void* Ht, const void* Et,
               const int32_t* row_mask, const float* lse_s, const float* lse_t,
               const float* dloss, int64_t N, int64_t D, int64_t V,
               float filter_eps, uint32_t flags, void* dH, void* dE, void* dE_comp,
               uint32_t* debug_keep, int64_t debug_rows,
               void* workspace, size_t workspace_bytes,
               int32_t* status, void* stream);

/* Workspace bytes cce_vocab_sort needs. */
size_t cce_vocab_sort_workspace_size(int64_t N, int64_t V, int32_t n_segs);

/*
 * Vocabulary sort ("Cut Your Losses in Large-Vocabulary Language Models",
 * first page §Contribution: a vocabulary sort groups the surviving blocks).
 * Writes vocab_perm [V_live] (layout as in cce_bwd): within each segment,
 * local rows ordered by descending key, ties by ascending id (stable).  The
 * key is colmax (from cce_fwd) when given, else the number of valid targets
 * that hit the row.
 */
int cce_vocab_sort(const float* colmax, const int32_t* y, int64_t N, int64_t V,
                   int32_t ignore_index, const cce_segment* segs, int32_t n_segs,
                   int32_t* vocab_perm, void* workspace, size_t workspace_bytes,
                   void* stream);

/*
 * Forward without a caller-provided workspace and without any device
 * allocation (the pages describe no such entry point; it has no counterpart
 * in the paper).  Meant for callers that cannot call cudaMalloc: code running
 * inside a host framework that owns all device memory and offers no
 * allocation hook (plugin interfaces of inference engines, C or Fortran
 * programs linking libcce without a device allocator), or code that must not
 * trigger the implicit device synchronisation an allocation can cause.
 *
 * Arguments and results are those of cce_fwd; the scratch the forward needs
 * lives in a fixed array of CCE_NOALLOC_SCRATCH_BYTES inside the library's
 * device image, which every GPU that loads libcce holds until the process
 * exits.  Returns CCE_EWORKSPACE when cce_fwd_workspace_size(N, D, V, n_segs)
 * exceeds that size (e.g. N = 4096, D = 2048, V = 128k fits; N = 8192,
 * D = 2304 does not).  The first call on each device looks up the array's
 * device address with that device current; make that first call before any
 * stream capture.  All calls on a device share the one array and the
 * forward overwrites every scratch byte it reads, so nothing needs clearing
 * between calls, but calls whose work overlaps on the GPU (other streams,
 * other host threads) race on it: serialise them.
 */
#define CCE_NOALLOC_SCRATCH_BYTES (32u << 20)
int cce_fwd_noalloc(const void* H, const void* E, const int32_t* y,
                    int64_t N, int64_t D, int64_t V, int32_t ignore_index,
                    const cce_segment* segs, int32_t n_segs,
                    float* loss, float* lse, float* colmax,
                    int32_t* status, void* stream);

/*
 * Diagnostic of the bounded waits (not needed for computing anything).
 * Launches one CTA of the tensor-core tile engine whose producer never fills
 * a stage: the MMA issuer's wait runs out after wait_ns nanoseconds of wall
 * clock, the CTA aborts, drains, frees its tensor memory and returns, and
 * CCE_STATUS_TIMEOUT is OR-ed into *status.  Every other kernel of the
 * library handles a wait that cannot complete this way (with a 2 s limit),
 * so the stream and the context stay usable.  No copy or MMA is issued.
 *   wait_ns  1 .. 1e9 (else CCE_EINVAL).
 *   status   device int32.
 */
int cce_debug_stall(uint64_t wait_ns, int32_t* status, void* stream);

/*
 * The same on one CTA pair of the cluster engine (tcgen05 cta_group::2):
 * the pair's MMA issuer waits for a stage its producers never fill, both
 * CTAs' epilogues wait for an accumulator that is never committed; each wait
 * runs out after wait_ns, both CTAs abort, hold a fixed grace period, free
 * the pair's tensor memory and return, and CCE_STATUS_TIMEOUT is OR-ed into
 * *status.  Arguments and errors as for cce_debug_stall.
 */
int cce_debug_stall_pair(uint64_t wait_ns, int32_t* status, void* stream);

/*
 * Diagnostics (not needed for computing anything).
 *
 * cce_launch_count: number of kernels libcce has enqueued in this process
 * since it was loaded (every entry point counts its launches).
 *
 * cce_timing_enable: while class_mask != 0, each launch of a selected kernel
 * class is bracketed by two CUDA events recorded on the stream the kernel is
 * launched on.  Classes: bit 0 forward tile stream, bit 1 backward G
 * producer, bit 2 backward dE contraction, bit 3 backward dH contraction,
 * bit 4 row compaction, gathers and finalize passes, bit 5 the sparse
 * gradient kernels (list counting, scans and scatter, the CSR gathers of dE
 * and dH, the dH fill).  cce_timing_read
 * synchronises on the recorded events, writes per class the summed
 * milliseconds and the number of timed launches (arrays of n_classes <= 6
 * entries, host memory), and clears the record.  Not thread-safe.  Returns
 * CCE_OK or CCE_EINVAL/CCE_ELAUNCH.
 */
uint64_t cce_launch_count(void);
int cce_timing_enable(uint32_t class_mask);
int cce_timing_read(float* ms, int64_t* launches, int32_t n_classes);

#ifdef __cplusplus
}
#endif
#endif /* CCE_H_ */
