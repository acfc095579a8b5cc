/*
 * fb.h - C ABI of the per-denoise-step block-diffusion attention library
 * (FlashBlock cached block-external attention and the LoSA sparse variant),
 * built for NVIDIA B200 (sm_100a).
 *
 * Method sources (cited by page title and section):
 *  [FB]   "FlashBlock: Attention Caching for Efficient Long-Context Block
 *         Diffusion", technical summary (gist.science, pt and ja), section 2
 *         "Core mechanism" (block-internal / block-external split, cached
 *         (A_out, L_out = log Z_out), merge equation) and "Adaptive reuse
 *         strategies" (threshold tau, per-head gamma).
 *  [LoSA] "LoSA: Locality Aware Sparse Attention for Block-Wise Diffusion
 *         Language Models" (gist.science, es), section 2 "El Algoritmo LoSA",
 *         steps 1-4.
 *
 * Conventions for every call:
 *  - Pointers are DEVICE pointers owned by the caller unless a parameter says
 *    "host". The library never allocates device memory; scratch comes from a
 *    caller-provided workspace whose size fb_workspace_size() returns.
 *  - Calls are asynchronous on `stream` and never synchronise, except where
 *    stated (fb_device_status).
 *  - Layouts are row-major. q: [batch, B, Hq, d]; block k/v: [batch, B, Hkv, d];
 *    partials A: [batch, B, Hq, d] float32, L: [batch, B, Hq] float32.
 *    L values are natural logarithms of the softmax normaliser (log Z).
 *    q head h reads kv head h / (Hq / Hkv).
 *  - Every call validates its arguments on the host before launching and
 *    returns FB_OK (0) or a negative FB_ERR_* code; the text of the last error
 *    of the calling thread is returned by fb_last_error().
 *  - `scale` (the softmax scale applied to <q, k>) must be positive and
 *    finite; anything else is FB_ERR_ARG.
 *  - Supported: head_dim 128 (bf16 and f32) or 64; page_size a power of two in
 *    [16, 128] for paged caches; 16-byte aligned tensors. Anything else is
 *    FB_ERR_SHAPE / FB_ERR_ALIGN.
 */
#ifndef FB_H_
#define FB_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FB_OK 0
#define FB_ERR_ARG (-1)       /* null pointer, negative size, inconsistent shapes */
#define FB_ERR_SHAPE (-2)     /* unsupported head_dim, page size, group size */
#define FB_ERR_ALIGN (-3)     /* a tensor is not 16-byte aligned */
#define FB_ERR_WORKSPACE (-4) /* workspace missing or smaller than required */
#define FB_ERR_CUDA (-5)      /* launch or driver error; text in fb_last_error() */
#define FB_ERR_TIMEOUT (-6)   /* a device-side wait exceeded its budget */

typedef enum { FB_F32 = 0, FB_BF16 = 1 } fb_dtype;

/*
 * The frozen block-external KV cache (J_out in [FB] section 2).
 *  k, v        [n_slots, n_heads_kv, head_dim] rows of `dtype`.
 *  page_table  [batch, max_pages_per_seq] int32 physical page of each logical
 *              page, or NULL for a contiguous cache where sequence b's token t
 *              is row b * max_seq_len + t.
 *              Paged: token t of sequence b is row
 *                page_table[b][t / page_size] * page_size + t % page_size.
 *              Entries of pages that hold tokens must lie in
 *              [0, n_slots / page_size). Every kernel that reads through the
 *              table checks the entry first: a page outside the pool is
 *              treated as holding no tokens (nothing is read through it) and
 *              the next fb_device_status() returns FB_ERR_ARG; fb_block_commit
 *              leaves such a page unwritten and reports it the same way.
 *  seq_len     [batch] int32 tokens per sequence (<= max_seq_len), or NULL when
 *              every sequence has max_seq_len tokens.
 *  page_size   tokens per logical page (also the LoSA page granularity).
 * Rows past a sequence's end may hold any bits (NaN included): they never
 * reach an output.
 */
typedef struct fb_kv {
  const void* k;
  const void* v;
  const int32_t* page_table;
  const int32_t* seq_len;
  int64_t n_slots;
  int32_t batch;
  int32_t n_heads_kv;
  int32_t head_dim;
  int32_t page_size;
  int32_t max_pages_per_seq;
  int32_t max_seq_len;
  fb_dtype dtype;
} fb_kv;

/*
 * Bytes of workspace that fb_prefix_attn, losa_select, losa_gather and fb_step
 * need for these shapes (n_active/topk_pages may be 0 when LoSA is unused).
 * num_sms: SM count the split plan targets (0: query the current device).
 * The split plan may be tuned through the environment (FB_SPLIT_WAVES: waves
 * of resident CTAs for the streaming kernels; FB_LIST_WAVES: the same for
 * page-list key sets; FB_TC_SPLITS: splits per row tile of the tcgen05
 * kernel); query the size under the same environment as the calls that use it.
 * Returns 0 on invalid arguments.
 */
size_t fb_workspace_size(const fb_kv* kv, int32_t block, int32_t n_heads_q, int32_t n_active,
                         int32_t topk_pages, int32_t num_sms);

/*
 * Byte offset, inside a workspace sized by fb_workspace_size with the same
 * arguments, of the page scores that losa_select (and fb_step in LOSA mode)
 * leave there ([LoSA] section 2, step 3: the page bound of each active row):
 * float32 [batch, min(n_active, block), n_heads_q, pages], pages = the
 * logical page count per sequence (max_pages_per_seq for a paged cache,
 * ceil(max_seq_len / page_size) otherwise); entry (b, a, h, p) is the bound of
 * the a-th active row (rank order) under q head h over page p, written for the
 * sequence's own pages only. For inspection and tests: the next selection
 * that uses the workspace overwrites them.
 * Returns 0 on invalid arguments or when n_active or topk_pages is 0 (no
 * scores); a valid offset is never 0.
 */
size_t fb_workspace_page_scores(const fb_kv* kv, int32_t block, int32_t n_heads_q,
                                int32_t n_active, int32_t topk_pages, int32_t num_sms);

/*
 * Block-external partial ([FB] section 2: A_out and L_out = log Z_out over J_out).
 * For every block row i and q head h:
 *   L_out = log sum_{t < seq_len[b]} exp(scale * <q_i,h , k_t>)
 *   A_out = sum_t exp(scale * <q, k_t> - L_out) v_t
 * computed by split-KV flash decoding (per-split partials merged with the same
 * log-space rule as [FB]'s merge).
 *  q          [batch, B, n_heads_q, head_dim] of kv->dtype.
 *  head_mask  [batch, n_heads_q] uint8 or NULL; heads with 0 are skipped and
 *             their a_out/l_out rows are left untouched (cache reuse).
 *  a_out      [batch, B, n_heads_q, head_dim] float32 (output).
 *  l_out      [batch, B, n_heads_q] float32 (output). An empty prefix gives
 *             A_out = 0, L_out = -inf.
 *  workspace  >= fb_workspace_size(kv, B, n_heads_q, 0, 0, 0) bytes.
 */
int fb_prefix_attn(const void* q, int32_t B, int32_t n_heads_q, float scale, const fb_kv* kv,
                   const uint8_t* head_mask, float* a_out, float* l_out, void* workspace,
                   size_t workspace_bytes, cudaStream_t stream);

/*
 * fb_prefix_attn without a workspace argument, for callers that cannot allocate
 * device memory on the call path: plugin interfaces that hand the plugin no
 * scratch pointer, engines that reserve all device memory up front in their
 * own pool (a stray cudaMalloc would fail or fragment it), and latency-bound
 * loops where cudaMalloc / cudaFree may synchronise the device. The pages have
 * no counterpart to this call; it is a deployment convenience.
 * Same arguments, results and errors as fb_prefix_attn, except:
 *  - the split-KV scratch lives in one static device array of
 *    FB_NOALLOC_SCRATCH_BYTES (32 MiB), which every GPU that loads the library
 *    holds until the process exits; shapes whose split plan needs more return
 *    FB_ERR_WORKSPACE with the required size in fb_last_error();
 *  - the array's device address is looked up on the first call made with a
 *    given device current and remembered with that device's context; make that
 *    first call before any stream capture. After cudaDeviceReset the next call
 *    sees a new context and looks the address up again (also a first call in
 *    this sense);
 *  - all calls share the one array, so calls that overlap on the GPU (other
 *    streams, other host threads) race and must be serialised by the caller;
 *  - nothing is allocated: no cudaMalloc, cudaFree or allocating library call.
 */
#define FB_NOALLOC_SCRATCH_BYTES (32u << 20)
int fb_prefix_attn_noalloc(const void* q, int32_t B, int32_t n_heads_q, float scale,
                           const fb_kv* kv, const uint8_t* head_mask, float* a_out, float* l_out,
                           cudaStream_t stream);

/*
 * Block-internal partial ([FB] section 2: A_in, L_in over J_in, recomputed
 * every step). Bidirectional: every block row attends all B block tokens.
 *  q [batch, B, n_heads_q, head_dim], k_in / v_in [batch, B, n_heads_kv, head_dim]
 *  of `dtype`; a_in [batch, B, n_heads_q, head_dim], l_in [batch, B, n_heads_q]
 *  float32 outputs.
 */
int fb_block_attn(const void* q, const void* k_in, const void* v_in, int32_t batch, int32_t B,
                  int32_t n_heads_q, int32_t n_heads_kv, int32_t head_dim, float scale,
                  fb_dtype dtype, float* a_in, float* l_in, cudaStream_t stream);

/*
 * Log-space merge ([FB] section 2, merge equation):
 *   m = max(L_out, L_in)
 *   A_full = (e^{L_out-m} A_out + e^{L_in-m} A_in) / (e^{L_out-m} + e^{L_in-m})
 *   L_full = m + log(e^{L_out-m} + e^{L_in-m})
 * rows = batch * B * Hq rows of head_dim floats. l_full may be NULL. A side
 * with L = -inf contributes nothing; both -inf gives A = 0, L = -inf.
 */
int fb_merge(const float* a_out, const float* l_out, const float* a_in, const float* l_in,
             int64_t rows, int32_t head_dim, float* a_full, float* l_full, cudaStream_t stream);

/*
 * Per-page key summary for the LoSA selector (QUEST-style upper bound).
 * page_min / page_max: [batch, max_pages_per_seq, n_heads_kv, head_dim] of
 * kv->dtype: per logical page, kv head and channel, the min / max of the
 * page's keys over its valid tokens (t < seq_len). Pages past the end of a
 * sequence are not written. Exact (no rounding).
 */
int fb_page_summary(const fb_kv* kv, void* page_min, void* page_max, cudaStream_t stream);

/*
 * LoSA selection ([LoSA] steps 1 and 3), one call per denoise step s >= 1.
 *  1. locality score per block row: sum over heads and channels of
 *     (q_cur - q_prev)^2, float32, squares rounded singly and summed by the
 *     stride-halving tree over n = h * head_dim + c;
 *  2. active_rows [batch, n_active]: the n_active highest scores per sequence,
 *     in rank order (ties: lower row first); n_active is clamped to B;
 *  3. for every active row and q head, page scores
 *     u_p = tree_sum_c max(q_c * kmin_{p,c}, q_c * kmax_{p,c}) (float32) and the
 *     topk_pages best pages (ties: lower page first);
 *  4. union over active rows and the q heads of each kv head:
 *     union_bitmap [batch, n_heads_kv, ceil(max_pages/32)] uint32 (bit p%32 of
 *     word p/32), union_list [batch, n_heads_kv, max_pages_per_seq] int32 pages
 *     in ascending order, union_count [batch, n_heads_kv] int32.
 *  row_scores [batch, B] float32 receives the locality scores (may be NULL).
 *  q_cur / q_prev: [batch, B, n_heads_q, head_dim] of kv->dtype.
 */
int losa_select(const void* q_cur, const void* q_prev, int32_t B, int32_t n_heads_q,
                const void* page_min, const void* page_max, const fb_kv* kv, int32_t n_active,
                int32_t topk_pages, int32_t* active_rows, float* row_scores,
                uint32_t* union_bitmap, int32_t* union_list, int32_t* union_count,
                void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * LoSA sparse prefix partial for the active rows ([LoSA] step 3, with step 2's
 * reuse for the others): for every active row i (active_rows[b][0..n_active))
 * and q head h, (A, L) over all tokens of the union pages of kv head h / G,
 * written over a_out[b, i, h, :] and l_out[b, i, h]. Stable rows are untouched.
 *  max_union: host upper bound of any union_count entry (the split plan and
 *             the workspace are sized by it), e.g. min(n_active * G * topk_pages,
 *             pages per sequence); <= 0 means pages per sequence. Counts above
 *             it are clamped.
 */
int losa_gather(const void* q, int32_t B, int32_t n_heads_q, const int32_t* active_rows,
                int32_t n_active, const int32_t* union_list, const int32_t* union_count,
                int32_t max_union, const fb_kv* kv, float scale, float* a_out, float* l_out,
                void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Step controller ([FB] "Adaptive reuse strategies"; [LoSA] steps 1-4).
 * ------------------------------------------------------------------------- */
typedef enum { FB_THRESHOLD = 0, FB_PER_HEAD = 1, FB_LOSA = 2, FB_SPARSE_RESIDUAL = 3 } fb_mode;

typedef struct fb_policy {
  fb_mode mode;
  int32_t tau;        /* THRESHOLD: recompute sequence b when m_updated[b] >= tau
                         (tau <= 0: recompute every step, i.e. dense).
                         SPARSE_RESIDUAL: refresh the selection and the residual
                         when any sequence has m_updated[b] >= tau */
  double gamma;       /* PER_HEAD: a head that computed at steps s-1 and s stops
                         computing for the rest of the block once
                         cos(A_out^s, A_out^{s-1}) >= gamma (gamma > 1: dense) */
  int32_t n_active;   /* LOSA: active rows per step */
  int32_t topk_pages; /* LOSA: pages kept per active row and q head;
                         SPARSE_RESIDUAL: pages selected per kv head */
  float scale;        /* softmax scale applied to <q, k> */
} fb_policy;

/*
 * Caller-owned state of one (layer, block), reused across its denoise steps.
 * All arrays are device memory sized for [batch, B, Hq, d] unless noted;
 * fields a mode does not use may be NULL.
 */
typedef struct fb_cache {
  float* a_out;           /* cached block-external partial A_out */
  float* l_out;           /* its log normaliser L_out */
  float* a_out_prev;      /* PER_HEAD: A_out of the previous computing step */
  uint8_t* head_mask;     /* PER_HEAD: [batch, Hq], 1 = compute at this step */
  double* head_cos;       /* PER_HEAD: [batch, Hq] last cosine (NaN if none) */
  void* q_prev;           /* LOSA: previous step's q */
  int32_t* active_rows;   /* LOSA: [batch, n_active] */
  float* row_scores;      /* LOSA: [batch, B] (may be NULL) */
  uint32_t* union_bitmap; /* LOSA: [batch, Hkv, ceil(max_pages/32)] */
  int32_t* union_list;    /* LOSA: [batch, Hkv, max_pages] */
  int32_t* union_count;   /* LOSA: [batch, Hkv] */
  int32_t step;           /* host: index of the next step (0 = block start); fb_step advances it */
  int32_t recomputed;     /* host: sequences (THRESHOLD) whose prefix partial the last step
                             recomputed; SPARSE_RESIDUAL: batch on a refresh step, else 0 */
  float* a_res;           /* SPARSE_RESIDUAL: cached partial over the unselected pages */
  float* l_res;           /* SPARSE_RESIDUAL: its log normaliser */
  int32_t* comp_list;     /* SPARSE_RESIDUAL: [batch, Hkv, max_pages] unselected pages */
  int32_t* comp_count;    /* SPARSE_RESIDUAL: [batch, Hkv] */
} fb_cache;

/*
 * One denoise step of attention for the block:
 *   THRESHOLD: sequence b recomputes A_out (fb_prefix_attn) when step == 0 or
 *              m_updated[b] >= tau, otherwise reuses the cache;
 *   PER_HEAD:  heads with head_mask = 1 recompute (all heads at steps 0, 1);
 *              then the cosine per computing head updates head_mask on the
 *              device (no host round trip);
 *   LOSA:      step 0 computes the dense prefix partial; later steps run
 *              losa_select + losa_gather; q is copied into q_prev.
 *   SPARSE_RESIDUAL ([FB] section 2, compatibility with sparse attention: the
 *              keys a sparse method leaves out are treated as block-external and
 *              their contribution is cached): on a refresh step (step 0, tau <= 0,
 *              or any m_updated[b] >= tau) every kv head selects topk_pages pages
 *              by the head score max over block rows i and its q heads h of
 *              tree_sum_c max(q_c kmin_c, q_c kmax_c) (float32, LoSA's order;
 *              ties: lower page) into union_bitmap / union_list / union_count,
 *              the other pages into comp_list / comp_count, and the partial
 *              over the unselected pages is stored in a_res / l_res. Every step
 *              computes the partial over the selected pages with the current q
 *              and merges it with the cached residual into a_out / l_out. The
 *              head score takes every stacked row (B * Hq / Hkv per kv head), 64
 *              at a time.
 *              Workspace: fb_workspace_size with n_active = B and topk_pages =
 *              the logical page count.
 * Then the block-internal partial is computed and merged:
 *   a_full [batch, B, Hq, d] float32, l_full [batch, B, Hq] float32 (may be NULL).
 *  q, k_in, v_in: this step's block tensors (dtype of prefix->dtype).
 *  page_min / page_max: fb_page_summary output (LOSA, SPARSE_RESIDUAL).
 *  m_updated: HOST [batch] int32 rows updated since the previous step
 *             (THRESHOLD, SPARSE_RESIDUAL; may be NULL at step 0).
 */
int fb_step(const fb_policy* policy, fb_cache* cache, const void* q, const void* k_in,
            const void* v_in, int32_t B, int32_t n_heads_q, const fb_kv* prefix,
            const void* page_min, const void* page_max, const int32_t* m_updated, float* a_full,
            float* l_full, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Packed (variable-length) block rows. Several blocks or branches of different
 * sizes share one launch: the BlockBatch page (gist.science, es), "Optimizacion
 * del Sistema", packs the unmasked query positions of all active branches into
 * one variable-length buffer so that branches of different block sizes run in
 * a single forward. Here sequence b of the batch (a branch, with its own prefix
 * through kv; branches of one request may share prefix pages through the page
 * table) owns block rows cu_rows[b] .. cu_rows[b+1]-1 of every packed buffer:
 *   q, a_*      [total_rows, n_heads_q, head_dim], l_* [total_rows, n_heads_q]
 *   k_in, v_in  [total_rows, n_heads_kv, head_dim] (the block's own keys)
 * cu_rows     DEVICE [batch + 1] int32, cu_rows[0] = 0, non-decreasing,
 *             cu_rows[batch] = total_rows. A sequence may have 0 rows.
 * max_rows    HOST: the most rows any sequence has (plans the launch and sizes
 *             the workspace: fb_workspace_size(kv, max_rows, n_heads_q, 0, 0, 0)).
 * total_rows  HOST: rows of the packed buffers.
 * The kernels check every sequence's offsets: a range that leaves
 * [0, total_rows], decreases or holds more than max_rows rows is treated as
 * empty (nothing is read or written through it) and the next
 * fb_device_status() returns FB_ERR_ARG.
 * ------------------------------------------------------------------------- */

/* fb_prefix_attn over packed rows: (A_out, L_out) of every packed row over its
 * own sequence's block-external keys ([FB] section 2). No head mask. */
int fb_prefix_attn_varlen(const void* q, const int32_t* cu_rows, int32_t max_rows,
                          int32_t total_rows, int32_t n_heads_q, float scale, const fb_kv* kv,
                          float* a_out, float* l_out, void* workspace, size_t workspace_bytes,
                          cudaStream_t stream);

/* fb_block_attn over packed rows: every row of sequence b attends the B_b =
 * cu_rows[b+1] - cu_rows[b] keys of its own block (bidirectional). */
int fb_block_attn_varlen(const void* q, const void* k_in, const void* v_in,
                         const int32_t* cu_rows, int32_t batch, int32_t max_rows,
                         int32_t total_rows, int32_t n_heads_q, int32_t n_heads_kv,
                         int32_t head_dim, float scale, fb_dtype dtype, float* a_in, float* l_in,
                         cudaStream_t stream);

/* fb_step over packed rows, THRESHOLD mode only (FB_ERR_ARG otherwise): each
 * sequence recomputes its A_out when step == 0 or m_updated[b] >= tau, then
 * the block-internal partial is computed and merged ([FB] section 2). The
 * cache's a_out / l_out are packed like q ([total_rows, n_heads_q, head_dim]).
 * total_rows = 0 only advances cache->step. */
int fb_step_varlen(const fb_policy* policy, fb_cache* cache, const void* q, const void* k_in,
                   const void* v_in, const int32_t* cu_rows, int32_t max_rows,
                   int32_t total_rows, int32_t n_heads_q, const fb_kv* prefix,
                   const int32_t* m_updated, float* a_full, float* l_full, void* workspace,
                   size_t workspace_bytes, cudaStream_t stream);

/*
 * Block commit: the finished block joins the block-external cache. Block
 * diffusion is causal between blocks ([FB] abstract, section 2), so once a
 * block's tokens are final they belong to J_out of every later block; the
 * LoSA page summaries ([LoSA] step 3) then have to cover them too.
 * For every sequence b with n_b = seq_len_host[b] tokens before the call:
 *  - block row j of k_in / v_in [batch, B, n_heads_kv, head_dim] (kv->dtype)
 *    is written to the cache slot of position n_b + j (page table, or row
 *    b * max_seq_len + t of a contiguous cache);
 *  - kv->seq_len[b] (device, required) becomes n_b + B;
 *  - if page_min / page_max (fb_page_summary layout) are given, the summary
 *    of every page receiving tokens is brought up to date: a page that held
 *    tokens before folds the new keys into its min / max, a fresh page is
 *    summarised from the new keys alone (bit-exact with a full recompute).
 * seq_len_host: HOST [batch] int32 lengths before the call; it must equal the
 *   device lengths (the caller tracks them to map pages). Every n_b + B must
 *   stay within kv->max_seq_len (FB_ERR_ARG otherwise); kv->max_seq_len in turn
 *   bounds the lengths that the attention calls plan for.
 * Paged caches: the caller maps the pages of positions up to n_b + B - 1 in
 *   the page table before the call. An entry outside the pool is not written
 *   through; the kernel flags it and fb_device_status() then returns
 *   FB_ERR_ARG.
 * B = 0 is a no-op.
 */
int fb_block_commit(const fb_kv* kv, const int32_t* seq_len_host, const void* k_in,
                    const void* v_in, int32_t B, void* page_min, void* page_max,
                    cudaStream_t stream);

/*
 * Self-test of the failure path (no counterpart on the pages): launches one
 * small kernel whose single wait can never be satisfied (an mbarrier nobody
 * arrives at). Its bounded wait, the same routine every kernel of this library
 * uses, gives up after about a millisecond, sets the device error word and
 * returns; the next fb_device_status() then reports FB_ERR_TIMEOUT and the
 * context stays usable. gave_up (device int, may be NULL) receives 1.
 */
int fb_selftest_timeout(int32_t* gave_up, cudaStream_t stream);

/*
 * Reads and clears the device-side error word that bounded waits set when they
 * give up (SYNCHRONISES the current device). Returns FB_OK, FB_ERR_TIMEOUT, or
 * FB_ERR_ARG when a kernel met a page-table entry outside the pool (a read
 * path, or fb_block_commit).
 */
int fb_device_status(void);

/* Text of the calling thread's last error ("" if none). */
const char* fb_last_error(void);

/* Number of kernels this library has launched in this process (all threads). */
uint64_t fb_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* FB_H_ */
