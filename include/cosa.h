/*
 * cosa.h -- C ABI of libcosa: CoSA's prefill path on NVIDIA B200 (sm_100a).
 *
 * The method is the one of "CoSA: Accelerating Long-Context Inference via
 * Proxy-Kernel Co-Designed Sparse Attention":
 *   - the Kernel-Aware Proxy (KAP, §4.2 and Appendix C.1 / Figure A) scores
 *     every causal (q-block, key-block) pair, flags the "have rowmax" (HRM)
 *     blocks and emits, per (query head, q-block), an ordered list of key
 *     blocks: HRM blocks first, each group by score, cut to the stage-1
 *     budget (the computation-order mask M_KAP of §4.1);
 *   - the page remap (§4.3 "Any-order page visiting") turns that list into
 *     physical KV pages;
 *   - the Ordered-Skipping Kernel (OSK, §4.3, Appendix C.2 / Algorithm A,
 *     Appendix D.1) visits only those pages, in that order, with online
 *     softmax, and skips a block's value side when its logits are negligible
 *     against the running row max (the in-kernel skip of §3.3).
 *
 * Conventions for every entry point:
 *   - Pointers marked "device" are CUDA device pointers; all work is enqueued
 *     on `stream` and the call returns without synchronising (except
 *     cosa_sync_status).  The caller owns every buffer, including the
 *     workspace; the library allocates and frees nothing.
 *   - Inputs are never modified.
 *   - bf16 tensors are IEEE bfloat16, row-major, densely packed as stated.
 *   - Return value: COSA_OK or a cosa_status code below.  Argument errors are
 *     detected on the host before anything is enqueued.  Errors found on the
 *     device (a bounded wait that expired, a failed bounds check) are
 *     recorded in the workspace's status word and reported by
 *     cosa_sync_status.
 */
#ifndef COSA_H_
#define COSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define COSA_API __attribute__((visibility("default")))
#else
#define COSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (the runtime's stream handle); NULL is the legacy default stream. */
typedef struct CUstream_st* cosa_stream_t;

typedef enum cosa_status {
  COSA_OK = 0,
  COSA_ERR_INVALID_ARG = 1,  /* null pointer, size out of range, tau or budget out of range */
  COSA_ERR_UNSUPPORTED = 2,  /* shape the kernels do not implement (see cosa_shape_t) */
  COSA_ERR_WORKSPACE = 3,    /* workspace smaller than cosa_workspace_size() */
  COSA_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed */
  COSA_ERR_TIMEOUT = 5,      /* device: a bounded pipeline wait expired (kernel gave up cleanly) */
  COSA_ERR_DEVICE = 6        /* device: an index failed its bounds check (access skipped) */
} cosa_status;

/*
 * Shape of one packed prefill batch.  By default every token of a sequence is
 * a query (query length == key length); with kv_lens set, each sequence's
 * first tokens are a cached prefix that has keys and values but no queries.
 *
 *   batch              number of sequences B >= 1
 *   num_q_heads        Hq; num_kv_heads Hkv; Hq % Hkv == 0 (GQA group G = Hq/Hkv <= 8).
 *                      Query head h reads kv head h / G.
 *   head_dim           d in {64, 128}
 *   block_size         b in {64, 128}: q-block = key block (Appendix D.1 uses b = 128)
 *   page_size          b_p, a multiple of 8 that divides b (a logical block
 *                      resolves to b / b_p pages, Appendix D.1)
 *   num_pages          P, pages in the pool
 *   max_pages_per_seq  row stride of page_table
 *   total_tokens       T = sum of sequence lengths
 *   total_qblocks      NQB = sum over sequences of ceil(L_s / b)
 *   max_seqlen         max L_s (sizes the per-row lists)
 *   cu_seqlens         device int32 [B+1]: token offset of each sequence in q/out
 *   cu_qblocks         device int32 [B+1]: q-block offset of each sequence
 *   page_layout        COSA_PAGES_HND (k/v pages [P, Hkv, b_p, d]) or
 *                      COSA_PAGES_NHD ([P, b_p, Hkv, d]); both read through
 *                      the same page_table
 *
 * Prefill after a cached prefix (q_len < kv_len; the pages treat full
 * prefill only, this follows the plainest reading).  kv_lens[s] = L_s is the
 * key count of sequence s; its queries are its last Lq_s tokens, with
 * Lq_s = cu_seqlens[s+1] - cu_seqlens[s] and 1 <= Lq_s <= L_s, so query t
 * sits at position off_s + t, off_s = L_s - Lq_s, and attends to keys
 * 0 .. off_s + t.  q-blocks stay on the key-block grid: q-block i covers
 * positions [i*b, (i+1)*b) within [off_s, L_s); the q-blocks wholly inside
 * the prefix have no list row, and the first present one, floor(off_s / b),
 * may lack its leading rows (its pooled sums run over its present rows).
 * With kv_lens set:
 *   total_tokens   = sum of Lq_s (rows of q and out)
 *   cu_qblocks     counts the present q-blocks: ceil(L_s/b) - floor(off_s/b)
 *   total_qblocks  = NQB, their sum (rows of every per-row list)
 *   cu_kblocks     key-block offsets: ceil(L_s/b) per sequence
 *   total_kblocks  = NKB, their sum
 *   max_seqlen     = max L_s (the longest key sequence; sizes kmax)
 * Every list entry, key block index and page_table row refers to the whole
 * sequence (prefix included).  kv_lens NULL: L_s = Lq_s and the key blocks
 * are the q-blocks.
 *
 * The host fields must agree with the device arrays; the kernels trust them
 * for grid sizes and check every derived index against them (a tile whose
 * offsets contradict the lengths is skipped and reported as
 * COSA_ERR_DEVICE).
 */
typedef struct cosa_shape {
  int32_t batch;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t block_size;
  int32_t page_size;
  int32_t num_pages;
  int32_t max_pages_per_seq;
  int32_t total_tokens;
  int32_t total_qblocks;
  int32_t max_seqlen;
  const int32_t* cu_seqlens;
  const int32_t* cu_qblocks;
  int32_t page_layout;   /* COSA_PAGES_HND or COSA_PAGES_NHD */
  const int32_t* kv_lens;     /* NULL, or device int32 [B]: keys per sequence (see below) */
  const int32_t* cu_kblocks;  /* device int32 [B+1] when kv_lens is set, else ignored */
  int32_t total_kblocks;      /* NKB when kv_lens is set, else ignored */
} cosa_shape_t;

/* Page pool layouts of k_pages / v_pages. */
#define COSA_PAGES_HND 0   /* [P, Hkv, b_p, d]: a (page, kv head) tile is contiguous */
#define COSA_PAGES_NHD 1   /* [P, b_p, Hkv, d]: a token's kv heads are contiguous (paged-attention engines) */

/*
 * Workspace bytes needed by cosa_proxy / cosa_attn for `shape` at stage-1
 * budget `budget`, and (if kmax_out != NULL) the list length kmax every
 * per-row output array uses:
 *   kmax = max(1, ceil(ceil(max_seqlen / b) * bp / 10^4)),
 *   bp   = floor(budget * 10^4 + 0.5) (basis points, computed in double).
 * Returns 0 when the shape or budget is invalid.
 * The workspace is device memory owned by the caller, 256-byte aligned; its
 * first 256 bytes are the status block and must be zero before first use
 * (cosa_workspace_init does that).  One workspace serves one stream at a time.
 */
COSA_API size_t cosa_workspace_size(const cosa_shape_t* shape, float budget, int32_t* kmax_out);

/* Zero the workspace's status block on `stream`. */
COSA_API int cosa_workspace_init(void* workspace, size_t ws_bytes, cosa_stream_t stream);

/*
 * KAP proxy (§4.2, Appendix C.1): stage-1 selection and visit order.
 *
 *   q           device bf16 [T, Hq, d]
 *   k_pages     device bf16 [P, Hkv, b_p, d], or [P, b_p, Hkv, d] when
 *               shape->page_layout is COSA_PAGES_NHD
 *   page_table  device int32 [B, max_pages_per_seq]; entry (s, p) is the
 *               physical page of tokens [p*b_p, (p+1)*b_p) of sequence s.
 *               Entries past the sequence's last page are not read.
 *   budget      stage-1 budget, a fraction in (0, 1]
 *   kmax        list length from cosa_workspace_size
 * Outputs (device, per query head h and global q-block I):
 *   order       int32 [Hq, NQB, kmax]: key blocks (index within the
 *               sequence) in visit order; -1 after the first count entries
 *   count       int32 [Hq, NQB]: k_i = max(1, ceil((i+1) * bp / 10^4)),
 *               i the q-block index within its sequence
 *   n_hrm       int32 [Hq, NQB]: HRM entries among the kept ones (a prefix)
 *   hrm_flags   uint8 [Hq, NQB, kmax]: 1 for HRM entries, 0 otherwise/pad
 * Definitions (the pages leave the score open; these are fixed here):
 *   key block sum  = fp32 sum over its valid tokens, token by token;
 *   q sub-row sum  = fp32 sum over the valid rows of each 16-row sub-row;
 *   q-block sum    = the sub-row sums folded in order from +0;
 *   int8 quantisation per vector: M = max|v|, zero if M < 2^-126, else
 *     q = rint(v * (127 / M)) (round half to even);
 *   dot = exact integer dot product; score = fp32(dot) * ks with the key
 *     block's scale ks = (M_k / 127) / n_tok, each step one fp32 operation;
 *   HRM: key block j is HRM iff it is the argmax over j' <= i (lowest index
 *     on ties) of some valid sub-row's score;
 *   order: (HRM first, score descending, block index ascending), first k_i.
 * The workspace carries the pooled int8 keys and the intermediate results
 * between the kernels the call enqueues.  At head_dim 128: key pooling; one
 * persistent kernel that pools the queries, scores and finds the HRM blocks
 * (each row's candidate score bits and HRM blocks to the workspace); the
 * selection in registers, then the rows it leaves.  Otherwise: key pooling,
 * query pooling (the int8 query vectors to the workspace), then scoring and
 * selection in one kernel.  Both give identical lists.
 */
COSA_API int cosa_proxy(const cosa_shape_t* shape, const void* q, const void* k_pages,
               const int32_t* page_table, float budget, int32_t kmax,
               int32_t* order, int32_t* count, int32_t* n_hrm, uint8_t* hrm_flags,
               void* workspace, size_t ws_bytes, cosa_stream_t stream);

/*
 * KAP proxy with the pages' Top-p stage-1 rule (§5.1 "Hyperparameters",
 * Appendix D.1: p = 0.95 for Qwen3-8B, calibrated per context length for
 * Llama-3.1-8B) instead of a budget fraction.  Scores, HRM flags and the
 * visit order are those of cosa_proxy; each row keeps the shortest prefix
 * of its full order (all n_i = i + 1 causal candidates) whose estimated
 * attention mass reaches p of the row's total.  The pages give p but not the
 * mass; this library's reading:
 *   w_j = n_tok(j) * exp((s_j - s_max) * zscale),
 *   zscale = (M_q / 127) / (n_rows * sqrt(d)),
 * s_j the block score, M_q the max-abs of the q-block's pooled query sum
 * (the scale the ranking score drops), n_rows the q-block's query rows, so
 * s_j * zscale estimates the mean logit between the q-block and block j.
 * Masses are fp32, summed in one fixed order (deterministic run to run); a
 * prefix whose share lies within about 1e-5 of p may be cut either way.
 *   p      in (0, 1]; p = 1 keeps every candidate
 *   kmax   at least ceil(max_seqlen / b) (cosa_workspace_size with budget
 *          1.0 returns it): a row may keep every candidate
 * Outputs, workspace and errors as cosa_proxy; count[h, I] is the row's cut.
 */
COSA_API int cosa_proxy_top_p(const cosa_shape_t* shape, const void* q, const void* k_pages,
                              const int32_t* page_table, float p, int32_t kmax,
                              int32_t* order, int32_t* count, int32_t* n_hrm, uint8_t* hrm_flags,
                              void* workspace, size_t ws_bytes, cosa_stream_t stream);

/* Capacity of the static device scratch array behind cosa_proxy_noalloc. */
#define COSA_NOALLOC_SCRATCH_BYTES (4u << 20)

/*
 * cosa_proxy for callers that cannot allocate device memory.  (The paper has
 * no counterpart: this is a library convenience, not part of the method.)
 *
 * Who needs it: code that runs inside an inference engine which has already
 * reserved nearly all device memory for its own pools (a serving framework's
 * KV cache) and offers no scratch API, and code on a latency-critical path
 * where cudaMalloc, which can fail under such a reservation and can
 * synchronise the device, is not acceptable.
 *
 * Same arguments and outputs as cosa_proxy, minus the workspace.  The pooled
 * key scratch lives instead in one static device array of
 * COSA_NOALLOC_SCRATCH_BYTES bytes that every GPU loading this library holds
 * until the process exits.  Limit: shapes whose pooled keys need more
 * (num_kv_heads * NKB * (head_dim + 4) bytes, plus alignment; NKB = total_qblocks
 * without a cached prefix) are
 * rejected with COSA_ERR_WORKSPACE before anything is enqueued.
 *
 * The first call on a device (with that device current) looks up the array's
 * device address; make that first call before any stream capture.  The call
 * allocates nothing and frees nothing.  Every call shares the one array and
 * overwrites it completely, so calls that overlap on the GPU (for example on
 * two streams) race; serialise them.  Device-side bounds checks still skip a
 * bad access but, without a workspace status word, are not reported.
 */
COSA_API int cosa_proxy_noalloc(const cosa_shape_t* shape, const void* q, const void* k_pages,
                                const int32_t* page_table, float budget, int32_t kmax,
                                int32_t* order, int32_t* count, int32_t* n_hrm, uint8_t* hrm_flags,
                                cosa_stream_t stream);

/*
 * Page remap (§4.3 "Any-order page visiting"): ordered key blocks -> pages.
 *   pages  device int32 [Hq, NQB, kmax * (b / b_p)]:
 *          pages[h, I, t*ppb + u] = page_table[s, order[h,I,t]*ppb + u]
 *          when t < count[h, I] and that logical page holds tokens of the
 *          sequence, else -1.
 * cosa_attn performs the same remap inside its producer; this entry point
 * exposes it for serving frameworks that keep their own page lists.
 */
COSA_API int cosa_remap(const cosa_shape_t* shape, const int32_t* page_table, const int32_t* order,
               const int32_t* count, int32_t kmax, int32_t* pages, cosa_stream_t stream);

/*
 * OSK attention (§4.3, Appendix C.2, Appendix D.1).
 *
 *   q, k_pages, page_table, order, count, kmax: as above; v_pages like k_pages.
 *   tau      skip threshold in [0, 1).  For a visited block, with
 *            s = q.k / sqrt(d) after the causal mask, m~_r its row max and
 *            m_r the running row max before it, the block's value side
 *            (exp, row sum, P V) is skipped iff
 *            max over the tile's valid rows of (m~_r - m_r) < ln(tau).
 *            tau = 0 never skips; the first visited block is never skipped.
 * Outputs (device):
 *   out      bf16 [T, Hq, d] = (sum over kept blocks of exp(s - m) V) / l
 *            (T = total_tokens: one row per query)
 *   visited  int32 [Hq, NQB]: blocks whose QK^T was computed (= count)
 *   skipped  int32 [Hq, NQB]: visited blocks whose value side was skipped
 *   skipbits uint8 [Hq, NQB, kmax] or NULL: 1 where list entry t was skipped
 * Token slots of a page past its sequence's end may hold any values: they
 * are never read into a result.
 */
COSA_API int cosa_attn(const cosa_shape_t* shape, const void* q, const void* k_pages, const void* v_pages,
              const int32_t* page_table, const int32_t* order, const int32_t* count,
              int32_t kmax, float tau, void* out, int32_t* visited, int32_t* skipped,
              uint8_t* skipbits, void* workspace, size_t ws_bytes, cosa_stream_t stream);

/*
 * OSK attention with the pages' length-adaptive threshold (§5.1
 * "Hyperparameters", Appendix D.1 "CoSA settings"): each sequence s of the
 * batch uses tau_s = delta / L_s, L_s its length in tokens (its key count,
 * the cached prefix included), computed on the device.  delta = -1 turns the skip off (tau = 0 for every
 * sequence); otherwise delta must be > 0.  tau_s >= 1 (a sequence shorter
 * than delta) is applied as written: the skip test compares against
 * ln(tau_s) >= 0.  All other arguments, outputs and errors as cosa_attn.
 */
COSA_API int cosa_attn_delta(const cosa_shape_t* shape, const void* q, const void* k_pages, const void* v_pages,
                    const int32_t* page_table, const int32_t* order, const int32_t* count,
                    int32_t kmax, float delta, void* out, int32_t* visited, int32_t* skipped,
                    uint8_t* skipbits, void* workspace, size_t ws_bytes, cosa_stream_t stream);

/*
 * OSK attention in logical-mask execution, for the ablation of §4.3
 * "Physical jumping over pages": the kernel walks every entry of each row's
 * list and computes only those with keep[h, I, t] != 0 (device uint8
 * [Hq, NQB, kmax]); the others are passed over by each warp role with no
 * copy, MMA or vote, as a block-sparse kernel with a mask would.  With the
 * list 0, 1, ..., i of all causal blocks and keep marking the selected ones,
 * this is the same computation as cosa_attn on the selected blocks in
 * ascending order.  visited counts the computed entries; skipbits is indexed
 * by list entry (0 where keep is 0).  A row with no kept entry is written as
 * zeros.  keep must not be NULL; everything else as cosa_attn.
 */
COSA_API int cosa_attn_masked(const cosa_shape_t* shape, const void* q, const void* k_pages, const void* v_pages,
                     const int32_t* page_table, const int32_t* order, const int32_t* count,
                     int32_t kmax, const uint8_t* keep, float tau, void* out, int32_t* visited,
                     int32_t* skipped, uint8_t* skipbits, void* workspace, size_t ws_bytes,
                     cosa_stream_t stream);

/*
 * Synchronise `stream`, read and clear the workspace's status word.
 * Returns COSA_OK, COSA_ERR_TIMEOUT, COSA_ERR_DEVICE or COSA_ERR_CUDA.
 */
COSA_API int cosa_sync_status(void* workspace, cosa_stream_t stream);

/*
 * Testing hook for failure detection: cap every pipeline wait of later
 * cosa_attn launches at `spins` polls (0 restores the default, several
 * seconds).  A cap too small for the pipeline makes the kernel record
 * COSA_ERR_TIMEOUT, drain its own copies and exit; no GPU state is harmed.
 */
COSA_API void cosa_debug_set_wait_limit(uint32_t spins);

/* Static string for a status code. */
COSA_API const char* cosa_error_string(int code);

/* Library ABI version (major * 100 + minor). */
COSA_API int cosa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* COSA_H_ */
