/*
 * fp2.h -- C ABI of a B200 (sm_100a) library for FlashPrefill V2's
 * mean-corrected block-sparse causal prefill attention.
 *
 * The operation (page: "FlashPrefill V2: Block-Sparse Prefill Attention for
 * Long-Context LLM Serving", metallab.ai paper page):
 *   Figure 3  Stage 1 pools block-mean statistics of Q, K and V and writes a
 *             CSR index of the selected key blocks (per KV head, Table 7);
 *             Stage 2 runs exact attention over the selected blocks while the
 *             unselected blocks enter through the mean-correction path, and
 *             both streams merge inside one online softmax.
 *   Figure 4  a pruned block J adds |B_J| e^{s_J} (vbar_J, 1) to the softmax
 *             numerator and denominator.
 *   Abstract / Table 9  max-based dynamic thresholding with parameter alpha.
 * Backend flags (page: "128K context now demands Hopper hardware",
 * nestfrontier.com, section "A serving setup you can actually test"):
 *   attention sink, window, abs threshold, last-n-blocks, k-block-n,
 *   min sparse q len, use mean correction -> fp2_sparse_params below.
 *
 * Readings fixed by this library where the pages are silent:
 *   score       s[h,i,j] = (qbar_{i,h} . kbar_{j,g(h)}) * scale, j <= i
 *   threshold   head h keeps j iff s >= max_{j'<=i} s[h,i,j'] + ln(alpha);
 *               a KV-head row keeps the union over its G query heads
 *   forced      j < sink_blocks; j > i - max(window_blocks, 1) (so the
 *               diagonal block is always exact); i >= N - last_n_blocks;
 *               whole rows of sequences shorter than min_sparse_len;
 *               alpha == 0 keeps everything
 *   correction  pruned block j adds logit q_t . kbar_j * scale + ln n_j with
 *               value vbar_j, n_j = tokens in block j
 *
 * Conventions
 *   - Every device buffer is allocated and owned by the caller.  The library
 *     never allocates or frees memory and never synchronises a stream; all
 *     kernels are launched on the stream passed in.
 *   - Every function returns fp2_status; arguments are validated on the host
 *     before anything is launched, and nothing is launched when validation
 *     fails.  fp2_last_error() gives a message for the calling thread.
 *   - Errors that only the device can see (a page-table entry out of range,
 *     an index entry out of range, a wait that timed out) are OR-ed into a
 *     status word at the start of the scratch buffer; read it with
 *     fp2_get_device_status() after the stream has been synchronised.
 *   - Token-major layouts: Q [T, Hq, d], K/V [T, Hkv, d], O [T, Hq, d];
 *     a paged cache is [num_pages, page_size, Hkv, d] with an int32 page table
 *     [num_seqs, max_pages_per_seq] (device memory).
 *   - Supported: head_dim 64 or 128 (F32 and E4M3 inputs need 64 and 128
 *     respectively), block_size 64 or 128, page_size a power of two >= 16,
 *     Hq % Hkv == 0, up to FP2_MAX_SEQS sequences and FP2_MAX_BLOCKS key blocks
 *     per sequence.
 *   - Chunked prefill (paper page, Table 6; ResearchPod: discovery re-runs per
 *     chunk): a sequence's queries may be a chunk of its last q_len <= kv_len
 *     tokens, aligned bottom-right (chunk token t is at absolute position
 *     kv_len - q_len + t); kv_len - q_len must be a multiple of block_size, so
 *     chunk block i is absolute key block I = (kv_len - q_len) / B + i, which is
 *     what causality, the diagonal and the window refer to; last_n_blocks and
 *     min_sparse_len refer to the chunk's queries.
 */
#ifndef FP2_H_
#define FP2_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define FP2_API __attribute__((visibility("default")))
#else
#define FP2_API
#endif

#define FP2_MAX_SEQS 512
#define FP2_MAX_BLOCKS 4096

typedef enum {
  FP2_OK = 0,
  FP2_ERR_INVALID_ARG = 1,          /* a pointer, size or parameter is invalid */
  FP2_ERR_UNSUPPORTED = 2,          /* valid but outside the supported shapes */
  FP2_ERR_WORKSPACE_TOO_SMALL = 3,  /* scratch_bytes below fp2_workspace_query's figure */
  FP2_ERR_CUDA = 4,                 /* a CUDA runtime call failed (message has the CUDA error) */
  FP2_ERR_DEVICE_BOUNDS = 5,        /* device saw a page id / index entry out of range */
  FP2_ERR_TIMEOUT = 6,              /* a device-side wait ran past its time limit */
  FP2_ERR_CHECK_FAILED = 7          /* checked build: a device-side invariant failed */
} fp2_status;

typedef enum { FP2_F32 = 0, FP2_BF16 = 1, FP2_E4M3 = 2 } fp2_dtype;

/* Bits of the device status word. */
#define FP2_DEV_PAGE_OOB 0x1u      /* page_table entry outside [0, num_pages) */
#define FP2_DEV_INDEX_OOB 0x2u     /* CSR column outside [0, i] / not ascending / diagonal missing */
#define FP2_DEV_CAPACITY 0x4u      /* kept blocks exceed fp2_index.col_capacity */
#define FP2_DEV_TIMEOUT 0x8u       /* an mbarrier wait gave up */
#define FP2_DEV_CHECK 0x10u        /* checked build only: a hand-off count or an index bound did not
                                      hold where it was checked; the guarded access was skipped */

/* cudaStream_t, passed as an opaque pointer so that this header needs no CUDA include. */
typedef void* fp2_stream_t;

typedef struct {
  int32_t num_seqs;
  const int32_t* cu_seqlens_q_host;  /* HOST [num_seqs+1], token offsets of each sequence's queries in Q */
  const int32_t* cu_seqlens_k_host;  /* HOST [num_seqs+1], token offsets of each sequence's keys in K/V
                                        (NULL = same as cu_seqlens_q_host); kv_len >= q_len */
  int32_t num_q_heads, num_kv_heads, head_dim;
  fp2_dtype dtype;                   /* storage type of Q, K, V (and of the MMA operands) */
  float q_descale, k_descale, v_descale;  /* value = stored * descale; 1.0 unless E4M3 */
  float softmax_scale;               /* 0 -> 1/sqrt(head_dim) */
  const void* q;                     /* device, [T, Hq, d] with token stride q_stride_tok elements */
  const void* k;                     /* device, [T, Hkv, d] or the paged cache */
  const void* v;
  int64_t q_stride_tok;              /* elements between consecutive tokens of Q (>= Hq*d) */
  int64_t kv_stride_tok;             /* elements between consecutive tokens of K/V (>= Hkv*d) */
  const int32_t* page_table;         /* device [num_seqs, max_pages_per_seq] or NULL for contiguous K/V */
  int32_t page_size, max_pages_per_seq, num_pages;
  int32_t kv_prefix_pooled;          /* nonzero: the pooled kbar/vbar (and MMA copies) of every sequence's
                                        prefix key blocks (those before its query chunk) are already in the
                                        pooled buffers at their indices, e.g. from the previous chunk's
                                        fp2_pool, so fp2_pool pools only the chunk's key blocks.  Valid when
                                        those indices did not move (a single sequence, or earlier sequences
                                        of the batch unchanged). */
} fp2_problem;

typedef struct {
  int32_t block_size;       /* B: tokens per pooled block, and the attention key tile (64 or 128) */
  float alpha;              /* threshold parameter in [0, 1]; 0 keeps every block */
  int32_t sink_blocks;      /* leading key blocks always kept */
  int32_t window_blocks;    /* blocks ending at the diagonal always kept (at least 1) */
  int32_t last_n_blocks;    /* the last n query blocks of each sequence keep every key block */
  int32_t min_sparse_len;   /* sequences shorter than this keep every block */
  int32_t mean_correction;  /* nonzero: pruned blocks contribute their pooled term */
  int32_t kv_splits;        /* count-balanced KV splits (paper page, Table 7): a split row's key tiles
                               are cut into equal ranges processed by separate CTAs and merged by
                               their LSE.
                               >= 1: every row in this many ranges (1 = no split; at most 64);
                               < 0:  adaptive: rows with more than -kv_splits key tiles (virtual
                                     tiles of the mean correction + kept blocks) are cut into
                                     ranges of at most that many tiles (at most 64 per row), the
                                     other rows stay whole; planned on the device from the index;
                               0:    automatic: when rows x packed parts < 296, every row in up to
                                     8 ranges; below 2368 (16 waves of 148 SMs), adaptive with the
                                     range size set to the launch's total tile work over 4 x SMs
                                     (at least 32 tiles), so that no row outlasts a fraction of the
                                     launch's load per SM; longer launches are not split.
                               Adaptive splits hold at most 768 ranges per fp2_attend call; rows
                               beyond that stay whole.  Range >= -FP2_MAX_BLOCKS. */
} fp2_sparse_params;

/* Pooled block statistics and operand copies (caller-owned device buffers, written by fp2_pool). */
typedef struct {
  float* qbar;     /* [total_q_blocks, Hq, d] f32 block means of Q (dequantised) */
  float* kbar;     /* [total_kv_blocks, Hkv, d] f32 */
  float* vbar;     /* [total_kv_blocks, Hkv, d] f32 */
  void* kbar_mma;  /* [total_kv_blocks, Hkv, d] in dtype: the kbar operand of the correction MMA
                      (E4M3: mean of the stored values, rounded to e4m3, same descale as K) */
  void* vbar_mma;  /* [total_kv_blocks, Hkv, d] in the PV operand type: dtype for F32 and BF16, f16 for
                      E4M3 (mean of the stored values rounded to f16, same descale as V) */
  void* v16;       /* E4M3 only: [total_kv_tokens, Hkv, d] f16, the stored V values converted exactly
                      (every e4m3 value is an f16 value), rows in key-token order of cu_seqlens_k
                      (gathered from the page table when paged); the PV operand of fp2_attend.  With
                      kv_prefix_pooled the prefix rows must already be there, like kbar/vbar.  NULL
                      (and unused) for F32 and BF16. */
} fp2_pooled;

/* CSR index of kept key blocks: row = (q_block_offset_r + i) * Hkv + g for query block i of
 * sequence r, columns are the sequence's absolute key-block ids in ascending order. */
typedef struct {
  int32_t* row_ptr;      /* device [index_rows + 1] */
  int32_t* col_idx;      /* device [col_capacity] */
  int64_t col_capacity;  /* entries available in col_idx */
} fp2_index;

/* Sizes for one problem; every *_bytes figure is a byte count of one buffer. */
typedef struct {
  int64_t total_tokens;          /* query tokens T */
  int64_t total_kv_tokens;       /* key tokens (contiguous K/V rows) */
  int64_t total_q_blocks;        /* sum_r ceil(q_len_r / B) */
  int64_t total_kv_blocks;       /* sum_r ceil(kv_len_r / B) */
  int64_t index_rows;            /* total_q_blocks * Hkv */
  int64_t col_capacity;          /* causal worst case: sum_r Hkv sum_i (I_i + 1) */
  size_t qbar_bytes, kbar_bytes, vbar_bytes, kbar_mma_bytes, vbar_mma_bytes;
  size_t row_ptr_bytes, col_idx_bytes;
  size_t discover_scratch_bytes; /* the part of scratch that fp2_discover uses (status, kept bits, counts) */
  size_t scratch_bytes;          /* scratch for fp2_pool / fp2_discover / fp2_attend (adds KV-split partials:
                                    for adaptive splits up to 768 ranges x (128 or 256) rows x d fp32) */
  size_t prefill_scratch_bytes;  /* scratch for fp2_prefill (adds pooled and index buffers) */
  size_t v16_bytes;              /* fp2_pooled.v16 (E4M3; 0 otherwise) */
} fp2_workspace;

/* Validate a problem and report buffer sizes.  Host only; launches nothing. */
FP2_API fp2_status fp2_workspace_query(const fp2_problem* problem, const fp2_sparse_params* params,
                               fp2_workspace* out);

/* The same validation, reporting three totals for callers that carve buffers out of single
 * allocations: pooled_bytes holds the fp2_pooled buffers (five, plus v16 for E4M3) and index_bytes
 * row_ptr and col_idx,
 * each buffer starting at a 256-byte aligned offset in that order; scratch_bytes is
 * fp2_workspace.scratch_bytes.  Any output pointer may be NULL.  Host only; launches nothing. */
FP2_API fp2_status fp2_workspace_size(const fp2_problem* problem, const fp2_sparse_params* params,
                              size_t* pooled_bytes, size_t* index_bytes, size_t* scratch_bytes);

/* Stage 1a (Figure 3, "pools block-mean statistics"): one pass over Q, K, V
 * (gathered through the page table when paged) writing every field of *pooled
 * (for E4M3 also the f16 copy of V that fp2_attend reads).
 * Clears the device status word at the start of scratch. */
FP2_API fp2_status fp2_pool(const fp2_problem* problem, const fp2_sparse_params* params, const fp2_pooled* pooled,
                    void* scratch, size_t scratch_bytes, fp2_stream_t stream);

/* Stage 1b (abstract and Table 9: max-based dynamic thresholding; Table 7: CSR
 * per KV head): block scores from pooled->qbar / pooled->kbar, the threshold
 * and forced rules, and compaction into *index. */
FP2_API fp2_status fp2_discover(const fp2_problem* problem, const fp2_sparse_params* params, const fp2_pooled* pooled,
                        const fp2_index* index, void* scratch, size_t scratch_bytes, fp2_stream_t stream);

/* Stage 2 (Figure 3 and Figure 4): exact attention over the kept blocks of *index
 * with mean correction for the pruned ones.  out: [T, Hq, d] bf16 (f32 when dtype
 * is FP2_F32); lse: [Hq, T] f32 natural-log normaliser, or NULL.  The index may
 * come from fp2_discover or from the caller; every row must be ascending, within
 * [0, i] and contain the diagonal block i.  E4M3: QK runs on the e4m3 Q and K, PV on
 * the f16 copy of V in pooled->v16 (so fp2_pool must have run on the same problem). */
FP2_API fp2_status fp2_attend(const fp2_problem* problem, const fp2_sparse_params* params, const fp2_pooled* pooled,
                      const fp2_index* index, void* out, float* lse, void* scratch, size_t scratch_bytes,
                      fp2_stream_t stream);

/* The whole operator: fp2_pool, fp2_discover and fp2_attend with the pooled and
 * index buffers carved from scratch (prefill_scratch_bytes). */
FP2_API fp2_status fp2_prefill(const fp2_problem* problem, const fp2_sparse_params* params, void* out, float* lse,
                       void* scratch, size_t scratch_bytes, fp2_stream_t stream);

/* Read the device status word from scratch (a blocking 4-byte copy; call it after
 * the stream has been synchronised).  *status_out gets the raw FP2_DEV_* bits; the
 * return value maps them to FP2_ERR_DEVICE_BOUNDS / FP2_ERR_TIMEOUT, else FP2_OK. */
FP2_API fp2_status fp2_get_device_status(const void* scratch, uint32_t* status_out);

/* Size of the device buffer fp2_discover_static uses in place of caller scratch. */
#define FP2_STATIC_SCRATCH_BYTES (8u << 20)

/* Discovery for callers that cannot allocate device memory where they run it (a serving runtime
 * that reserved all memory up front and forbids allocation on the request path, or a C host with no
 * device allocator).  The paper has no counterpart: this is fp2_discover with its scratch moved into
 * a library-owned static __device__ buffer of FP2_STATIC_SCRATCH_BYTES per GPU, held until exit.
 * Inputs (pooled) and outputs (index) are still the caller's.  Returns FP2_ERR_UNSUPPORTED when the
 * problem's fp2_workspace.discover_scratch_bytes exceeds FP2_STATIC_SCRATCH_BYTES.  Calls no
 * allocator.  The first call in each CUDA context looks up the buffer's device address (cached per
 * device with the context's id, so a new context after a device reset looks it up again); with
 * CUDA's lazy module loading that first call is also when the driver places the buffer, so make it
 * at start-up, before reserving the rest of device memory and before any stream capture.  All
 * calls share the buffer: calls that overlap on the GPU race, so serialise them.  status_dev
 * (device pointer, or NULL) receives a copy of the FP2_DEV_* status word of this call. */
FP2_API fp2_status fp2_discover_static(const fp2_problem* problem, const fp2_sparse_params* params,
                                       const fp2_pooled* pooled, const fp2_index* index, uint32_t* status_dev,
                                       fp2_stream_t stream);

/* Testing hooks, process-wide, for exercising the device-side time limits without a GPU fault.
 * Not for production use.  The paper has no counterpart.
 *   FP2_DEBUG_WAIT_LIMIT_NS    limit of every wait inside the attention kernel, in ns (0 restores
 *                              the default of 1 s; otherwise 1e5 .. 1e10); draining copies in
 *                              flight at exit waits up to a fifth of it.
 *   FP2_DEBUG_WITHHOLD_K_TILE  the producer of every attention CTA skips the K load of its local
 *                              key tile `value` (-1 restores normal operation): that tile's barrier
 *                              never completes, the wait for it runs out, every role of the CTA
 *                              gives up and drains through its bounded paths, and the status word
 *                              gets FP2_DEV_TIMEOUT.  Nothing faults; the next call is unaffected.
 *   FP2_DEBUG_MISCOUNT_LOAD    checked builds only: the producer of every attention CTA counts its
 *                              K/V load `value` (-1 restores normal operation) twice in the
 *                              hand-off counters, so the consumer's check of that load fails and
 *                              the status word gets FP2_DEV_CHECK.  The data path is unchanged;
 *                              the normal build ignores it.
 * Returns FP2_ERR_INVALID_ARG for an unknown key or a value out of range. */
#define FP2_DEBUG_WAIT_LIMIT_NS 1
#define FP2_DEBUG_WITHHOLD_K_TILE 2
#define FP2_DEBUG_MISCOUNT_LOAD 3
FP2_API fp2_status fp2_debug_set(int32_t key, int64_t value);

/* Message for the last failing call on this thread ("" if none). */
FP2_API const char* fp2_last_error(void);

/* Library version as major*10000 + minor*100 + patch. */
FP2_API int32_t fp2_version(void);

/* How this library was built: FP2_BUILD_CHECKED is set in libfp2_checked.so, the same sources
 * compiled with FP2_CHECKED=1.  There every mbarrier hand-off of the attention kernel is followed
 * by a check that the producing side has signalled exactly as often as the waiter's own count says
 * (a wait that completed on a stale or a future phase of the barrier would see a different count),
 * and per-thread global stores and shared-memory indexes are bounds-checked.  A failed check sets
 * FP2_DEV_CHECK (fp2_get_device_status returns FP2_ERR_CHECK_FAILED) and skips the guarded store;
 * nothing traps.  Same arguments and results as the normal library, somewhat slower. */
#define FP2_BUILD_CHECKED 0x1u
FP2_API uint32_t fp2_build_flags(void);

#ifdef __cplusplus
}
#endif

#endif  /* FP2_H_ */
