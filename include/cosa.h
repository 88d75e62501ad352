/*
 * cosa.h — C interface of the CoSA block-sparse causal prefill attention library
 * (libcosa.so, sm_100a).
 *
 * The method: "CoSA: Accelerating Long-Context Inference via Proxy-Kernel
 * Co-Designed Sparse Attention".  Its abstract (insight.artgrammer.co.kr,
 * fugumt.com) fixes two stages: a Kernel-Aware Proxy (KAP) that selects KV
 * blocks under a moderate budget and emits an *ordered* mask, the order in
 * which the kernel's inner loop visits KV pages; and an Ordered-Skipping Kernel
 * (OSK) that applies the mask and skips further blocks from online-softmax
 * statistics.  The technical summary on gist.science/pt gives the steps:
 * §2.2 "Estágio 1: KAP" (downsampling, approximate scores, MaxPool over keys,
 * MaxNorm, HRM flags, flag-group ordering) and §2.3 "Estágio 2: OSK" (mask-
 * skipped pages via KV page remapping, in-kernel skip on local max vs running
 * max, computed pages).
 *
 * Conventions for every entry point
 *   - All tensor arguments are DEVICE pointers on the current CUDA device,
 *     allocated and owned by the caller (except the *_host arguments of
 *     cosa_attention_host, which are host memory); the library allocates no
 *     device memory per call and keeps no pointer after the call is enqueued
 *     (cosa_attention_host creates two streams and a few events per call and
 *     hands them back to CUDA before returning).
 *   - Layouts are dense, row-major (last index fastest):
 *       q          bf16  [B][H_q][N][D]
 *       k_pool     bf16  [num_phys_pages][H_kv][P][D]   (one page of one KV head
 *                                                      is a contiguous P*D block)
 *       v_pool     bf16  [num_phys_pages][H_kv][P][D]
 *       page_table int32 [B][pages_per_seq]   logical page -> physical page
 *       out        bf16  [B][H_q][N][D]
 *       lse        fp32  [B][H_q][N]          natural-log softmax normaliser
 *       order      int32 [B][H_q][nQB][k_cap] logical page ids, -1 past count
 *       count      int32 [B][H_q][nQB]
 *       scores     fp32  [B][H_q][nQB][nP]    proxy score S (0 past n_b)
 *       hrm        uint8 [B][H_q][nQB][nP]    Have-RowMax flags (0 past n_b)
 *     with N = seq_len, nP = N / P, nQB = N / Bq, and query head h reading KV
 *     head h / (H_q / H_kv).  Query i attends to keys 0..i (causal prefill).
 *   - Calls are asynchronous on `stream` (0 = legacy default stream).
 *     Argument errors are detected on the host and returned before anything
 *     is launched.  Launch failures return COSA_ERR_CUDA.  Errors detected
 *     inside a kernel (a bounded wait that ran out) are recorded in a
 *     per-device status word; read it with cosa_get_status().
 *   - Supported shapes (COSA_ERR_UNSUPPORTED otherwise): D = 128 (all kernels)
 *     or D = 64 (KAP and the attention kernels); P in {64, 128};
 *     Bq in {64, 128}; N a multiple of P and of Bq; H_q a multiple of H_kv;
 *     page_table entries in [0, num_phys_pages).  The kernels that address
 *     pages with plain loads and stores (KAP's pooling, cosa_prefill_write,
 *     cosa_osk_decode) check every entry they use: one outside the pool is
 *     recorded as COSA_ERR_INVALID_ARG in the status word and that page is
 *     neither read nor written (its pooled key vectors are zero; decode treats
 *     the list entry as invalid).  The TMA kernels (OSK, dense) read such a
 *     page as zeros, and cosa_attention_host checks its host page table before
 *     anything is queued.
 */
#ifndef COSA_H_
#define COSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* cosa_stream_t; /* a cudaStream_t */

typedef enum {
  COSA_OK = 0,
  COSA_ERR_INVALID_ARG = 1, /* null pointer, negative or inconsistent size       */
  COSA_ERR_UNSUPPORTED = 2, /* valid but outside the supported shape set        */
  COSA_ERR_CUDA = 3,        /* a CUDA runtime/driver call or a launch failed     */
  COSA_ERR_TIMEOUT = 4,     /* a kernel's bounded wait ran out (status word)     */
  COSA_ERR_WORKSPACE = 5    /* workspace missing or smaller than required        */
} cosa_status_t;

/* Problem shape shared by all entry points. */
typedef struct {
  int32_t batch;          /* B                                                  */
  int32_t num_q_heads;    /* H_q                                                */
  int32_t num_kv_heads;   /* H_kv, divides H_q                                  */
  int32_t seq_len;        /* N (prefill length; queries and keys)               */
  int32_t head_dim;       /* D                                                  */
  int32_t page_size;      /* P tokens per KV page                               */
  int32_t q_block;        /* Bq query rows per q-block (one OSK tile)           */
  int32_t pages_per_seq;  /* row stride of page_table, >= N / P                 */
  int32_t num_phys_pages; /* rows of k_pool / v_pool                            */
  float softmax_scale;    /* multiplies q.k (usually 1/sqrt(D))                 */
} cosa_shape_t;

/* Kernel-Aware Proxy parameters (gist.science/pt §2.2). */
typedef struct {
  float budget;       /* fraction of a q-block's causal pages to keep, in [0,1]; the
                         kept count is ceil(fl32(budget * n_b)), at least the forced
                         pages, at most n_b                                           */
  int32_t q_sub;      /* query rows pooled into one representative; divides Bq,
                         Bq / q_sub in {1, 2, 4, 8}                                   */
  int32_t k_sub;      /* keys pooled into one sub-key; divides P, P / k_sub in
                         {1, 2, 4, 8}                                                 */
  int32_t sink_pages; /* leading pages always kept (>= 0); the q-block's own pages
                         are always kept too                                          */
  int32_t ascending;  /* 0: list kept pages by rank (HRM first, then score
                         descending, then lower page id) — the ordered mask;
                         1: list them by page id (a binary mask's visit order)       */
} cosa_kap_params_t;

/* Ordered-Skipping Kernel parameters (gist.science/pt §2.3). */
typedef struct {
  float eps;       /* >= 0.  A listed page other than the first is skipped when, for
                      every row of the q-block that sees a key in it, (page max logit
                      - running max) < ln(eps).  0 never skips; +inf skips every page
                      after the first unless some row meets its first visible key
                      there.                                                          */
  int32_t max_run; /* >= 0.  0: the rule above alone (the pages' rule).  r > 0: once
                      r consecutive listed pages have been skipped, the rest of the
                      q-block's list is skipped without being visited (no K load,
                      no QK^T): an early break, not part of the pages' method.
                      cosa_osk_attention_group supports 0 only.                       */
} cosa_osk_params_t;

/* Status string for a status code (static storage, never NULL). */
const char* cosa_status_string(cosa_status_t status);

/* Library version as (major << 16) | (minor << 8) | patch. */
int32_t cosa_version(void);

/* Length of one ordered-page row: the largest per-q-block kept count k_b.
 * Host-only; no CUDA call. */
cosa_status_t cosa_kap_kcap(const cosa_shape_t* shape, const cosa_kap_params_t* kap,
                            int32_t* k_cap);

/* Bytes of device workspace cosa_kap_select needs (pooled queries and keys as
 * two TF32 terms each, the per-page maxima of every representative row, and
 * each row's maximum and first page attaining it).  Host-only; no CUDA call. */
cosa_status_t cosa_kap_workspace_size(const cosa_shape_t* shape, const cosa_kap_params_t* kap,
                                      size_t* bytes);

/* Stage 1, all steps (gist.science/pt §2.2 "Ranking de Blocos", "Geração de
 * Flag HRM", "Ordenação por Grupo de Flags"; abstract: "selects blocks under a
 * moderate budget and produces an ordered mask"):
 *   q^ = mean of q_sub consecutive rows, k^ = mean of k_sub consecutive keys;
 *   a[r][p] = max over causally visible sub-keys of scale * <q^_r, k^_{p,t}>;
 *   S[p] = mean_r exp(a[r][p] - max_p' a[r][p']); HRM[p] = page holding the row
 *   max of some representative (lowest page on ties);
 *   keep the forced pages (sink_pages leading pages + the q-block's own pages)
 *   plus the best-ranked others up to k_b; list them by rank (or by page id).
 * Writes order (k_cap entries per q-block, -1 padded) and count.  scores / hrm
 * may be NULL; when given, the per-page S and flags are written there too.
 * workspace: device buffer of at least cosa_kap_workspace_size bytes, 256-byte
 * aligned; its contents on entry do not matter. */
cosa_status_t cosa_kap_select(const cosa_shape_t* shape, const cosa_kap_params_t* kap,
                              const void* q, const void* k_pool, const int32_t* page_table,
                              int32_t* order, int32_t* count, float* scores, uint8_t* hrm,
                              void* workspace, size_t workspace_bytes, cosa_stream_t stream);

/* Stage 1 in two launches, for callers that time or schedule the steps apart;
 * cosa_kap_pool followed by cosa_kap_rank on the same workspace is
 * cosa_kap_select (same kernels, same results).
 *
 * cosa_kap_pool: the downsampling step alone (gist.science/pt §2.2 "Ranking de
 * Blocos": downsampling of queries and keys): q^ and k^ as above, written to the
 * workspace (at least cosa_kap_workspace_size bytes, 256-byte aligned) as two
 * TF32 terms each.  Reads Q and the K pages once: the step is bound by HBM
 * bandwidth. */
cosa_status_t cosa_kap_pool(const cosa_shape_t* shape, const cosa_kap_params_t* kap,
                            const void* q, const void* k_pool, const int32_t* page_table,
                            void* workspace, size_t workspace_bytes, cosa_stream_t stream);

/* cosa_kap_rank: the remaining Stage-1 steps (approximate scores, MaxPool over
 * keys, MaxNorm, HRM flags, budgeted selection and flag-group ordering;
 * gist.science/pt §2.2) from the pooled vectors that cosa_kap_pool left in the
 * workspace for the same shape and parameters (stream order: queue it after
 * that call).  order, count, scores and hrm as for cosa_kap_select. */
cosa_status_t cosa_kap_rank(const cosa_shape_t* shape, const cosa_kap_params_t* kap,
                            int32_t* order, int32_t* count, float* scores, uint8_t* hrm,
                            void* workspace, size_t workspace_bytes, cosa_stream_t stream);

/* The prefill's write of its attention inputs with Stage 1's downsampling fused in
 * (gist.science/pt §2.2 "Ranking de Blocos": downsampling of queries and keys).  A
 * prefill layer produces Q, K and V token-major; attention reads Q head-major and K
 * and V from the paged cache.  This call does that write and, in the same pass over
 * the rows, the pooling of cosa_kap_pool into the workspace, so Stage 1 needs no
 * second read of Q and K: cosa_kap_rank on the same workspace then finishes it, and
 * the result is bit-identical to cosa_kap_select on the written q and k_pool.
 *   q_tok bf16 [B][N][H_q][D], k_tok / v_tok bf16 [B][N][H_kv][D] (inputs);
 *   q bf16 [B][H_q][N][D], k_pool / v_pool bf16 [num_phys_pages][H_kv][P][D]
 *   (outputs: the layouts above; every page the page table names for the
 *   sequences' N tokens is written, others untouched; page-table entries of one
 *   call must be distinct).
 * workspace: a cosa_kap_select workspace (cosa_kap_workspace_size bytes, 256-byte
 * aligned) for the pooled vectors, or NULL for the plain write without pooling.
 * All buffers 16-byte aligned. */
cosa_status_t cosa_prefill_write(const cosa_shape_t* shape, const cosa_kap_params_t* kap,
                                 const void* q_tok, const void* k_tok, const void* v_tok,
                                 const int32_t* page_table, void* q, void* k_pool, void* v_pool,
                                 void* workspace, size_t workspace_bytes, cosa_stream_t stream);

/* Proxy-bound pre-skip: a variant the pages do not give (their in-kernel skip,
 * gist.science/pt §2.3 "Saltado no Kernel", still pays every listed page its K
 * load and QK^T).  It applies the same kind of test one stage earlier, on the
 * proxy's page maxima a[r][p] and the proxy's own running maximum along each
 * q-block's ordered list, and removes the pages it rejects before the kernel
 * runs: with ahat_r(j) the maximum of a[r][.] over the pages listed before
 * position j, representative r keeps position j iff a[r][p_j] > -inf and
 * (ahat_r(j) = -inf or a[r][p_j] + margin - ahat_r(j) >= ln(eps)); position
 * j >= 1 is removed iff no representative keeps it.  The survivors keep their
 * order.  Filters order / count in place: the per-head lists that
 * cosa_kap_select (or cosa_kap_rank) just wrote with this workspace, shape and
 * kap, whose page maxima the workspace still holds.  skip_log (uint8
 * [B][H_q][nQB][k_cap], may be NULL) gets 1 at the original list positions
 * removed, 0 at the others (entries past the old count untouched).  eps >= 0
 * (0 removes nothing), margin >= 0 and finite (nats).  Lists of up to 8192
 * entries (COSA_ERR_UNSUPPORTED beyond); a list entry outside the q-block's
 * causal pages leaves that list as it is and records COSA_ERR_INVALID_ARG in the
 * status word.  The pre-skip decides on proxy estimates, not bounds: the output
 * can differ from the pages' rule on the full list, and the pages' rule is
 * what cosa_osk_attention then applies to the survivors. */
cosa_status_t cosa_kap_preskip(const cosa_shape_t* shape, const cosa_kap_params_t* kap,
                               float eps, float margin, int32_t* order, int32_t* count,
                               uint8_t* skip_log, const void* workspace, size_t workspace_bytes,
                               cosa_stream_t stream);

/* Stage 1 with one list per KV head: the G query heads that read KV head h_kv
 * share one ordered list per q-block (the group-shared selection; the pages
 * describe per-head selection only, this is the next step after it).  Every
 * step up to the per-head MaxNorm scores S_h[p] and flags HRM_h[p] is that of
 * cosa_kap_select; then
 *   S[p] = max over the group's heads of S_h[p], HRM[p] = OR of HRM_h[p],
 * and the same forced pages, budget, key and order.  order is
 * int32 [B][H_kv][nQB][k_cap] (-1 padded), count int32 [B][H_kv][nQB]; scores /
 * hrm (may be NULL) get the group's S and flags, [B][H_kv][nQB][nP].  Same
 * workspace as cosa_kap_select.  kap->ascending must be 0
 * (COSA_ERR_UNSUPPORTED otherwise); G * (q_block / q_sub) > 64 is unsupported. */
cosa_status_t cosa_kap_select_group(const cosa_shape_t* shape, const cosa_kap_params_t* kap,
                                    const void* q, const void* k_pool, const int32_t* page_table,
                                    int32_t* order, int32_t* count, float* scores, uint8_t* hrm,
                                    void* workspace, size_t workspace_bytes, cosa_stream_t stream);

/* Largest workspace (cosa_kap_workspace_size) that cosa_kap_select_noalloc
 * accepts: 128 MiB, enough for a 32K-token layer with 32 query heads. */
#define COSA_KAP_NOALLOC_SCRATCH_BYTES (128u << 20)

/* cosa_kap_select for callers that cannot allocate device memory.  The paper
 * has no counterpart: this is a packaging variant of the same Stage-1 kernels.
 * Some callers cannot call cudaMalloc or hand out a workspace at call time (a
 * runtime that owns the device allocator, a plan whose memory is fixed in
 * advance), so the pooled vectors and page maxima go to a fixed 128 MiB array
 * inside the library instead.  Every GPU on which the library's kernels load
 * holds that array until the process exits.  Arguments and results are those
 * of cosa_kap_select without the workspace; the caller still allocates q,
 * k_pool, page_table, order, count and the optional scores / hrm.
 *   - Shapes whose cosa_kap_workspace_size exceeds COSA_KAP_NOALLOC_SCRATCH_BYTES
 *     return COSA_ERR_UNSUPPORTED before anything is launched.
 *   - The first call on a device looks up the array's device address (with that
 *     device current); make that first call before any stream capture.  The
 *     address is cached per CUDA context: after a device reset (a new context) the
 *     next call looks it up again, and that call too belongs before any capture.
 *   - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 *   - All calls on a device share the one array, and it keeps the last call's
 *     contents (every kernel writes what it later reads, so nothing needs
 *     clearing).  Calls whose execution overlaps on the GPU (different streams,
 *     or different host threads on the same device) race on it: serialise them. */
cosa_status_t cosa_kap_select_noalloc(const cosa_shape_t* shape, const cosa_kap_params_t* kap,
                                      const void* q, const void* k_pool,
                                      const int32_t* page_table, int32_t* order, int32_t* count,
                                      float* scores, uint8_t* hrm, cosa_stream_t stream);

/* Stage 1, selection and ordering only (gist.science/pt §2.2 "Ordenação por
 * Grupo de Flags"), from caller-given scores (fp32, >= 0) and HRM flags laid out
 * as above; entries past each q-block's causal pages are ignored.  Given the
 * same scores and flags, the result is fully determined (ties broken by page
 * id), so it is bit-reproducible.  No workspace. */
cosa_status_t cosa_kap_order(const cosa_shape_t* shape, const cosa_kap_params_t* kap,
                             const float* scores, const uint8_t* hrm, int32_t* order,
                             int32_t* count, cosa_stream_t stream);

/* Stage 2 (gist.science/pt §2.3): for every (b, h_q, q-block) visit the listed
 * pages order[0..count) in list order through the page table (unlisted pages are
 * never read), accumulate online softmax, and skip a page per the eps rule above
 * (one decision per q-block tile; skipped pages change nothing).
 * order/count as written by cosa_kap_select (or any list of distinct causal
 * pages per q-block, count >= 1, order[j] < n_b).  lse, computed (int32
 * [B][H_q][nQB], pages actually computed) and skip_log (uint8
 * [B][H_q][nQB][k_cap], 1 = skipped, entries past count untouched) may be NULL. */
cosa_status_t cosa_osk_attention(const cosa_shape_t* shape, const cosa_osk_params_t* osk,
                                 const void* q, const void* k_pool, const void* v_pool,
                                 const int32_t* page_table, const int32_t* order,
                                 const int32_t* count, int32_t k_cap, void* out, float* lse,
                                 int32_t* computed, uint8_t* skip_log, cosa_stream_t stream);

/* Stage 2 over group-shared lists (cosa_kap_select_group): every query head h
 * runs the per-head skip rule and online softmax of cosa_osk_attention on the
 * list of its KV head h / G; the result equals cosa_osk_attention given each
 * head its KV head's list.  Two query heads of a KV head run in one CTA and
 * share every K tile load.  order int32 [B][H_kv][nQB][k_cap], count int32
 * [B][H_kv][nQB]; out, lse, computed (int32 [B][H_q][nQB]) and skip_log (uint8
 * [B][H_q][nQB][k_cap]) as for cosa_osk_attention. */
cosa_status_t cosa_osk_attention_group(const cosa_shape_t* shape, const cosa_osk_params_t* osk,
                                       const void* q, const void* k_pool, const void* v_pool,
                                       const int32_t* page_table, const int32_t* order,
                                       const int32_t* count, int32_t k_cap, void* out, float* lse,
                                       int32_t* computed, uint8_t* skip_log, cosa_stream_t stream);

/* Bytes of device workspace cosa_osk_decode needs for lists of k_cap entries: the
 * listed pages' logits and local maxima, and per-chunk partial sums.  Host-only. */
cosa_status_t cosa_osk_decode_workspace_size(const cosa_shape_t* shape, int32_t k_cap,
                                             size_t* bytes);

/* Decode: one new query per sequence and head visits an ordered page list under
 * the in-kernel rule of Stage 2 (gist.science/pt §2.3), as a q-block of one row.
 * The pages leave decoding as future work (closing section); this is the plainest
 * continuation of the prefill method (for instance with the list KAP wrote for the
 * q-block that holds the query).  q bf16 [B][H_q][D]: the query of each sequence
 * and head; positions int32 [B] (device): its position t, 0 <= t < seq_len; it
 * sees keys 0..t of the paged cache (k_pool / v_pool / page_table as above,
 * holding at least t + 1 tokens).  order int32 [B][H_q][k_cap] (logical pages,
 * each <= t / P, distinct), count int32 [B][H_q].  eps in [0, 1] (the rule above;
 * eps > 1 is rejected with COSA_ERR_INVALID_ARG), max_run 0 (COSA_ERR_UNSUPPORTED
 * otherwise).  out bf16 [B][H_q][D]; lse fp32 [B][H_q], computed int32 [B][H_q]
 * and skip_log uint8 [B][H_q][k_cap] may be NULL.  workspace: at least
 * cosa_osk_decode_workspace_size(shape, k_cap) bytes, 256-byte aligned.  A list
 * entry past the query's page or naming a physical page outside the pool, or a
 * position out of range, is never read: it is recorded as COSA_ERR_INVALID_ARG
 * in the status word (an empty list, or a position out of range, gives a zero
 * output, lse -inf and 0 computed). */
cosa_status_t cosa_osk_decode(const cosa_shape_t* shape, const cosa_osk_params_t* osk,
                              const void* q, const void* k_pool, const void* v_pool,
                              const int32_t* page_table, const int32_t* positions,
                              const int32_t* order, const int32_t* count, int32_t k_cap, void* out,
                              float* lse, int32_t* computed, uint8_t* skip_log, void* workspace,
                              size_t workspace_bytes, cosa_stream_t stream);

/* Dense causal attention over the same paged cache (every causal page in page
 * order, no skipping): the comparison point for the sparse path's speedup.
 * lse may be NULL. */
cosa_status_t cosa_dense_attention(const cosa_shape_t* shape, const void* q, const void* k_pool,
                                   const void* v_pool, const int32_t* page_table, void* out,
                                   float* lse, cosa_stream_t stream);

/* Bytes of device workspace cosa_attention_host needs: the page table, two sets
 * of one KV head's Q, K pool column, V pool column and output, one KV head's
 * ordered lists and its cosa_kap_select workspace.  Host-only; no CUDA call. */
cosa_status_t cosa_attention_host_workspace_size(const cosa_shape_t* shape,
                                                 const cosa_kap_params_t* kap, size_t* bytes);

/* Both stages end to end from host memory: for every KV head, copy its column of
 * the K and V page pools to the device, and for each of its G query heads in turn
 * copy that head's Q (every sequence), run cosa_kap_select and cosa_osk_attention on
 * that query head alone (shape with H_q = 1, H_kv = 1: heads are independent in both
 * stages, so the result equals the whole-layer calls) and copy its output back to
 * its place in out_host.  The copies in and the read-backs run on two streams of
 * the call's own, overlapping the kernels, which run on `stream`; `stream` waits for
 * all of it, so synchronising `stream` means the output is in out_host.  q_host
 * bf16 [B][H_q][N][D], k_pool_host / v_pool_host
 * bf16 [num_phys_pages][H_kv][P][D], page_table_host int32 [B][pages_per_seq]
 * and out_host bf16 [B][H_q][N][D] are host memory; page-locked memory lets the
 * copies overlap the kernels (pageable memory works but the copies serialise).
 * The host buffers must stay valid and unmodified until `stream` reaches the end
 * of this call's work.  workspace: device buffer of at least
 * cosa_attention_host_workspace_size bytes, 256-byte aligned.  Argument errors
 * (a page_table_host entry outside [0, num_phys_pages) among them:
 * COSA_ERR_INVALID_ARG) return before anything is queued; a failed CUDA call returns COSA_ERR_CUDA
 * with the work queued so far still joined to `stream`; in-kernel errors go to
 * the status word as for the stage calls. */
cosa_status_t cosa_attention_host(const cosa_shape_t* shape, const cosa_kap_params_t* kap,
                                  const cosa_osk_params_t* osk, const void* q_host,
                                  const void* k_pool_host, const void* v_pool_host,
                                  const int32_t* page_table_host, void* out_host, void* workspace,
                                  size_t workspace_bytes, cosa_stream_t stream);

/* Test hook, not part of the method (the pages describe no failure handling): it
 * lets a test make one of the attention kernel's bounded waits run out on purpose
 * and check that the failure is reported and leaves the device usable.  The next
 * cosa_osk_attention call made from this host thread (and only that call: the
 * setting is consumed by it, whatever it returns) runs with
 *   - every bounded wait limited to wait_limit_ns of no progress (0 keeps the
 *     default of one second), and
 *   - when withhold_k_group >= 0, the K tile copies of that listed group (list
 *     entries 2g and 2g+1 for 64-token pages, entry g for 128-token pages) never
 *     issued in any q-block whose list reaches it, so the waits for it run out.
 * The kernel then records COSA_ERR_TIMEOUT in the status word, waits (bounded)
 * for the copies and MMAs it did issue, frees its tensor memory and returns; the
 * other CTAs of the launch stop early.  That call's outputs are undefined; the
 * following calls run normally.  That call must have max_run = 0
 * (COSA_ERR_INVALID_ARG otherwise).  withhold_k_group < -1: COSA_ERR_INVALID_ARG.
 * Host-only; no CUDA call. */
cosa_status_t cosa_debug_osk_wait_fault(int32_t withhold_k_group, uint64_t wait_limit_ns);

/* Read (and clear) the current device's status word: COSA_OK, or the first
 * in-kernel error recorded since the last call (e.g. COSA_ERR_TIMEOUT).
 * Synchronises `stream`. */
cosa_status_t cosa_get_status(cosa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* COSA_H_ */
