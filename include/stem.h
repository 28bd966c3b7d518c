/*
 * stem.h — C-ABI of the Stem sparse-attention prefill library (libstem).
 *
 * The operations follow the public descriptions of Tencent Hunyuan's Stem, in
 * particular the Tencent Cloud developer article
 * "从Stem稀疏注意力看 大模型推理的架构取舍" (sections "TPD：优先级排序",
 * "OAM：价值评估", "HPC-Stem：评估选块，快几十倍", "HPC-BSA：跳块零开销的秘密").
 *
 * Conventions for every entry point
 *  - Plain pointers and sizes only.  "DEVICE" pointers are CUDA device memory of
 *    the current device; "HOST" pointers are ordinary host memory.
 *  - The caller owns every buffer, including the device workspace; the library
 *    never allocates or frees device memory.
 *  - All device work is enqueued on the caller's stream and no call synchronises,
 *    except stem_query_status().
 *  - Arguments are validated on the host before any launch; a bad argument
 *    returns STEM_ERR_INVALID / STEM_ERR_UNSUPPORTED / STEM_ERR_WORKSPACE and
 *    launches nothing.  A failed launch returns STEM_ERR_CUDA.  Errors detected
 *    on the device (a pipeline wait that timed out, an out-of-range block index)
 *    are recorded in the workspace status word and reported by
 *    stem_query_status().
 *  - Layouts are token-major: Q is [T, Hq, d], K and V are [T, Hkv, d], d
 *    contiguous, where T is the total number of tokens of the batch
 *    (sequences packed back to back as given by cu_seqlens).  Q/K/V/out base
 *    pointers must be 16-byte aligned.
 *  - Supported shapes: head_dim 64 or 128 (FP8: 128 only); block_size 64 or
 *    128; num_q_heads a multiple of num_kv_heads; at most STEM_MAX_SEQS
 *    sequences; at most STEM_MAX_BLOCKS blocks per sequence; paged caches
 *    use 64-token pages.
 */
#ifndef STEM_H_
#define STEM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define STEM_API __attribute__((visibility("default")))
#else
#define STEM_API
#endif

#define STEM_MAX_SEQS 64
#define STEM_MAX_BLOCKS 2048
#define STEM_PAGE_SIZE 64

typedef enum {
  STEM_OK = 0,
  STEM_ERR_INVALID = 1,      /* null pointer, inconsistent sizes, bad parameter */
  STEM_ERR_UNSUPPORTED = 2,  /* valid but not implemented (head_dim, block, dtype combination) */
  STEM_ERR_WORKSPACE = 3,    /* workspace null or smaller than stem_workspace_size() */
  STEM_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed */
  STEM_ERR_TIMEOUT = 5,      /* device: a pipeline wait exceeded its time limit */
  STEM_ERR_BOUNDS = 6        /* device: a block index outside its sequence was seen */
} stem_status_t;

typedef enum { STEM_DT_BF16 = 0, STEM_DT_FP8_E4M3 = 1 } stem_dtype_t;

/* One prefill problem: a batch of sequences sharing head layout and parameters. */
typedef struct {
  int num_seqs;
  const int32_t* cu_seqlens;   /* HOST [num_seqs+1]: token offsets, cu_seqlens[0] = 0 */
  int num_q_heads;             /* Hq */
  int num_kv_heads;            /* Hkv; q-head h reads kv-head h / (Hq/Hkv) */
  int head_dim;                /* d */
  int block_size;              /* B: tokens per block (selection granularity) */
  stem_dtype_t dtype;          /* storage type of Q, K, V */
  float q_scale, k_scale, v_scale; /* FP8: value = code * scale (per tensor); BF16: ignored */
  float softmax_scale;         /* sigma; <= 0 selects 1/sqrt(head_dim) */
  float beta;                  /* OAM weight of the log||V|| term (0.2 in the article) */
  double keep;                 /* fraction of causal block pairs kept, in (0, 1] */
  double mu;                   /* TPD end-to-start keep ratio (0.7 in the article), in (0, 1] */
  int shared_lists;            /* 0: one selection per q-head (the article's method).
                                  1: one selection per KV group — an extension of this library,
                                  not in the pages: the group's score of a block is the float32
                                  sum, in head order, of its q-heads' OAM scores; every q-head of
                                  the group uses the group's list (col_idx then has Hkv rows). */
} stem_problem_t;

/* Optional paged KV cache (vLLM style).  Pass NULL for contiguous K/V. */
typedef struct {
  const void* k_cache;         /* DEVICE [num_slots, page_size, Hkv, d] */
  const void* v_cache;         /* DEVICE [num_slots, page_size, Hkv, d] */
  const int32_t* block_table;  /* DEVICE [num_seqs, max_pages_per_seq]: page p of sequence b lives in slot block_table[b*max_pages_per_seq + p] */
  int page_size;               /* must be STEM_PAGE_SIZE */
  int max_pages_per_seq;
  int num_slots;
} stem_paged_kv_t;

/* Buffer sizes a caller needs for one problem. */
typedef struct {
  int64_t num_rows;            /* R = sum_b N_b, N_b = ceil(len_b / B): rows of row_ptr minus one */
  int64_t scores_per_head;     /* sum_b N_b (N_b + 1) / 2: packed causal scores per q-head */
  int64_t nnz_per_head;        /* sum_b K_b: selected (q-block, kv-block) pairs per q-head */
  int64_t total_tokens;        /* T */
  size_t workspace_bytes;      /* device workspace for any entry point of this problem */
  int64_t list_heads;          /* rows of col_idx: Hq, or Hkv with shared_lists */
} stem_sizes_t;

/* Sizes of every buffer of the problem.  Host only.  Returns STEM_ERR_* on a bad problem. */
STEM_API stem_status_t stem_query_sizes(const stem_problem_t* prob, stem_sizes_t* out);

/* Device workspace bytes (same as stem_query_sizes().workspace_bytes); 0 on a bad problem. */
STEM_API size_t stem_workspace_size(const stem_problem_t* prob);

/*
 * TPD budget plan for one sequence of n_blocks blocks (host only, no device).
 * Article section "TPD：优先级排序": the per-position top-k budget decays
 * linearly from the start to the end, the end keeping mu of the initial
 * budget, and the total is redistributed, not increased.  Readings taken:
 *   w_i = (1 - (1-mu) * i / (N-1)) * (i+1)          (w_0 = 1 when N = 1)
 *   k_i(r) = min(i+1, max(min(2, i+1), floor(r * w_i)))   (block 0 and the diagonal forced)
 *   T = clamp(floor(keep * N(N+1)/2 + 1/2), 2N-1, N(N+1)/2)
 *   r_start = midpoint of the first interval of r on which sum_i k_i(r) >= T
 *             (the interval past the last jump is represented by twice that jump).
 * Outputs: *r_start (keep fraction of block row 0), *total = sum_i k_i(r_start).
 */
STEM_API stem_status_t stem_tpd_plan(int n_blocks, double keep, double mu, double* r_start, int64_t* total);

/*
 * OAM block scores (article sections "OAM：价值评估" and "HPC-Stem").
 *   s[h, i, j] = sigma * <mean_{t in blk i} q_t[h], mean_{t in blk j} k_t[kh]>
 *              + beta * mean_{t in blk j} log ||v_t[kh]||_2,       0 <= j <= i,
 * one GEMM over per-block means, no softmax, no gather.
 * q, k, v: DEVICE (k, v ignored when paged != NULL, which then supplies them).
 * scores: DEVICE float [Hq, scores_per_head]; sequence b, row i, column j at
 *   off_b + i(i+1)/2 + j, off_b = sum_{b'<b} N_b'(N_b'+1)/2.
 * ws: DEVICE workspace of ws_bytes >= stem_workspace_size().
 */
STEM_API stem_status_t stem_score(const stem_problem_t* prob, const void* q, const void* k, const void* v,
                         const stem_paged_kv_t* paged, float* scores, void* ws, size_t ws_bytes,
                         void* stream);

/*
 * TPD budget + top-k selection fused in one kernel (article section "HPC-Stem":
 * budget generation and the selection sort are one operator).  For every
 * sequence b, q-block row i and q-head h: block 0 and block i are kept, and the
 * other k_i - min(2, i+1) blocks are the best of 1..i-1 under (score descending,
 * index ascending); NaN ranks as -inf.
 * scores: DEVICE float [Hq, scores_per_head] (layout of stem_score).
 * row_ptr: DEVICE int32 [num_rows + 1], shared by all heads (the budget does not
 *   depend on the head); row (b, i) is global row sum_{b'<b} N_b' + i.
 * col_idx: DEVICE int32 [list_heads, nnz_per_head]: ascending block indices
 *   local to the sequence, diagonal last; list l's row r is
 *   col_idx[l*nnz + row_ptr[r] ...].  list_heads = Hq (list l = q-head l) or, with
 *   shared_lists, Hkv (list l = KV group l, ranked by the group's summed scores).
 */
STEM_API stem_status_t stem_select(const stem_problem_t* prob, const float* scores, int32_t* row_ptr,
                          int32_t* col_idx, void* ws, size_t ws_bytes, void* stream);

/*
 * Scoring and selection as one operator (article section "HPC-Stem": compact
 * block representations, one pass that yields every block score, budget generation
 * fused with the top-k, no intermediate score tensor).  Pools Q, K and V into the
 * workspace, then each block row's scores (the formula of stem_score) are computed
 * inside the selection kernel and ranked there (the rules of stem_select); no score
 * matrix is written.  The lists equal stem_score followed by stem_select bit for bit
 * (same float32 operations in the same order).  Shapes the fused kernel does not
 * cover (shared_lists with more than 16 q-heads per KV group) go through the score
 * matrix in the workspace instead, with the same result.  On B200 this operator takes
 * longer than stem_score + stem_select (each row re-reads its kv-head's block means,
 * where the tiled score GEMM reuses them across rows), so stem_attention uses the latter;
 * it is for callers that cannot hold the score matrix.
 * row_ptr, col_idx: DEVICE, layouts of stem_select.  Other arguments as stem_score.
 */
STEM_API stem_status_t stem_score_select(const stem_problem_t* prob, const void* q, const void* k, const void* v,
                                         const stem_paged_kv_t* paged, int32_t* row_ptr, int32_t* col_idx,
                                         void* ws, size_t ws_bytes, void* stream);

/*
 * Block-sparse causal attention prefill (article section "HPC-BSA"): for each
 * (q-head, q-block) the kernel walks only the listed KV blocks with an online
 * softmax and no per-block branch; skipped blocks behave exactly as if all their
 * scores were -inf; only the diagonal block is token-masked.
 * col_idx: [list_heads, nnz_per_head] as stem_select writes it; q-head h walks list
 *   h / (Hq / list_heads).
 * out: DEVICE bf16 [T, Hq, d].  lse: DEVICE float [Hq, T] natural-log
 * log-sum-exp of sigma*q.k over the visited keys, or NULL.
 * FP8: Q/K/V are e4m3 codes with per-tensor scales; P is rounded to e4m3 for
 * the P.V product; out is bf16.
 */
STEM_API stem_status_t bsa_prefill(const stem_problem_t* prob, const void* q, const void* k, const void* v,
                          const stem_paged_kv_t* paged, const int32_t* row_ptr, const int32_t* col_idx,
                          void* out, float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * Dense causal attention prefill with the same kernel: every block 0..i is
 * visited (the comparator for the density sweep; equals bsa_prefill on a keep = 1
 * selection).  Arguments as bsa_prefill without the selection.
 */
STEM_API stem_status_t bsa_dense_prefill(const stem_problem_t* prob, const void* q, const void* k, const void* v,
                                const stem_paged_kv_t* paged, void* out, float* lse, void* ws,
                                size_t ws_bytes, void* stream);

/*
 * The whole prefill path: stem_score -> stem_select -> bsa_prefill (the same result
 * as stem_score_select -> bsa_prefill), with the scores and the selection kept in the
 * workspace.  Arguments as bsa_prefill.
 * If row_ptr_out / col_idx_out are non-NULL the selection is also copied there
 * (layouts of stem_select).
 */
STEM_API stem_status_t stem_attention(const stem_problem_t* prob, const void* q, const void* k, const void* v,
                             const stem_paged_kv_t* paged, void* out, float* lse, int32_t* row_ptr_out,
                             int32_t* col_idx_out, void* ws, size_t ws_bytes, void* stream);

/*
 * The whole prefill path from HOST buffers, for end-to-end use (no counterpart in
 * the pages).  q_host, k_host, v_host: HOST inputs in the layouts of q, k, v (a
 * paged cache: k_host / v_host hold whole caches of num_slots * page_size rows).
 * out_host: HOST bf16 [T, Hq, d], receives O.  The kv-heads are split into G
 * groups, G the largest divisor of Hkv not above out_groups (0: 8); each group
 * (its kv-heads and their q-heads) is a problem of its own.  When G >= 2, every group
 * holds one kv-head and a multiple of 4 q-heads, and shared_lists is 0, the first and
 * the last group each run as two halves of their q-heads (a problem each, with the
 * group's kv-head), so the first input copy and the last output copy are half as
 * large.  Per group (or half), its heads
 * are copied host -> device, the path runs on them, and their O goes back
 * device -> host; the input copies, the path and the output copies run on three
 * streams, so the copies of one group overlap the work of the others.  The results
 * (out_host, out, lse, the selection) equal stem_attention's for any G.
 * q, k, v (a paged cache: paged->k_cache, paged->v_cache) and out: DEVICE scratch
 * of the sizes of the full tensors, which this call overwrites with the inputs and
 * outputs staged group after group (each group's heads contiguous; a group run in
 * two halves holds its first half's heads, then its second half's), not in the
 * layouts above.  lse: DEVICE [Hq, T] or NULL; row_ptr_out, col_idx_out: DEVICE or
 * NULL, layouts of stem_select.  Completion of the call's work on `stream` includes
 * every copy; the device buffers are not overwritten before the caller's earlier
 * work on `stream` completes.  Host buffers should be page-locked (cudaHostAlloc /
 * cudaHostRegister): pageable ones work but their copies do not overlap.  The
 * library keeps two non-blocking copy streams per device (created on first use) and
 * creates and releases CUDA events per call; it allocates no device memory.
 * Errors as stem_attention, plus STEM_ERR_INVALID for a NULL host pointer or
 * out_groups < 0.
 */
STEM_API stem_status_t stem_attention_host(const stem_problem_t* prob, const void* q_host, const void* k_host,
                                           const void* v_host, void* q, void* k, void* v,
                                           const stem_paged_kv_t* paged, void* out_host, void* out, float* lse,
                                           int32_t* row_ptr_out, int32_t* col_idx_out, int out_groups, void* ws,
                                           size_t ws_bytes, void* stream);

/*
 * stem_attention without a caller workspace, for callers that cannot allocate
 * device memory (a plugin or custom-operator host whose framework owns every
 * byte of the GPU, a serving loop that must not allocate while it runs).  The
 * pages have no counterpart: this is a deployment convenience of this library.
 * Scratch comes from one fixed 32 MiB array compiled into the library, which
 * every device that loads the library holds until the process exits; a problem
 * whose stem_workspace_size() exceeds it is refused with STEM_ERR_WORKSPACE
 * before anything is launched.  No call allocates or frees device memory.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current), so make that first call before any stream
 * capture.  The address is kept for the life of the process: do not call this
 * entry point again on a device after a device reset (cudaDeviceReset, or its
 * primary context destroyed and recreated), which moves the array.  All calls on a device share the array and it keeps the last call's
 * contents: calls that overlap on the GPU (other streams, other threads) race
 * and must be serialised by the caller.  The status word is cleared at the start
 * of each call; status_out (DEVICE uint32, or NULL) receives this call's device
 * status word (0 = ok, bit 0 = pipeline wait timed out, bit 1 = bad block index).
 * Other arguments as stem_attention.
 */
STEM_API stem_status_t stem_attention_noalloc(const stem_problem_t* prob, const void* q, const void* k,
                                              const void* v, const stem_paged_kv_t* paged, void* out, float* lse,
                                              int32_t* row_ptr_out, int32_t* col_idx_out, uint32_t* status_out,
                                              void* stream);

/*
 * Synchronise the stream, read and clear the device status word kept in the
 * workspace.  Returns STEM_OK, STEM_ERR_TIMEOUT, STEM_ERR_BOUNDS or STEM_ERR_CUDA.
 */
STEM_API stem_status_t stem_query_status(void* ws, void* stream);

/* Zero the workspace status word (enqueued on the stream). */
STEM_API stem_status_t stem_reset_status(void* ws, void* stream);

/*
 * Failure-detection test hook (no counterpart in the pages).  mode 1 makes the next
 * bsa_prefill / bsa_dense_prefill / stem_attention launch withhold one K tile in
 * the first CTA, so that CTA's bounded pipeline wait runs out (after about 2 s):
 * the kernel records STEM_ERR_TIMEOUT in the workspace status word, releases its
 * tensor memory and exits, and the GPU context stays usable.  The launch that
 * consumes the request clears it; mode 0 cancels a pending request.
 */
STEM_API stem_status_t stem_debug_inject(int mode);

/* Static description of a status code. */
STEM_API const char* stem_status_string(stem_status_t s);

/* Text of the last error recorded by this thread (validation or CUDA), "" if none. */
STEM_API const char* stem_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* STEM_H_ */
