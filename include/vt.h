/*
 * vt.h -- C ABI of libvt: block top-k sparse decode attention over a paged KV
 * cache on NVIDIA B200 (sm_100a).
 *
 * The method (sources: "Vortex: A Flexible and Efficient Sparse Attention
 * Framework", the vortex_torch README, sections "Quick Example: Custom Sparse
 * Attention" and "Using Your Sparse Attention with SGLang"; and "Vortex:
 * Efficient and Programmable Sparse Attention Serving for AI Agents", section
 * "A dual-stage programmable abstraction"):
 *   cache side  -- when a page of 16 tokens is finished, its centroid (the
 *                  mean of its keys, one head_dim vector per KV head) is stored
 *                  in a per-page cache;
 *   query side  -- per request and KV head, the grouped query heads are
 *                  averaged, the mean is scored against the centroid of every
 *                  middle page, the top-k pages plus the reserved first `bos`
 *                  and last `eos` pages are kept, and exact softmax attention
 *                  runs over the tokens of those pages only.
 *
 * Conventions shared by every entry point
 *   - Every data pointer is DEVICE memory owned by the caller.  The library
 *     never allocates, frees or synchronises; each call enqueues its kernels
 *     on `stream` (a cudaStream_t passed as void*; NULL = legacy default
 *     stream) and returns.  Only vt_sparse_decode_fused takes a workspace
 *     (see vt_fused_workspace_size).
 *   - bf16 means IEEE bfloat16 (upper half of a binary32), fp32 is binary32.
 *   - Host-side argument checks fail fast with VT_ERR_INVALID_ARG or
 *     VT_ERR_UNSUPPORTED before anything is launched; a failed launch returns
 *     VT_ERR_CUDA.  vt_last_error_detail() gives a one-line reason (per host
 *     thread).
 *   - Checks that need device data (a page id outside [0, num_pages), a
 *     seq_len < 1 or longer than the page table, a bad sel entry) are done by
 *     the kernels: the affected unit is skipped (its outputs are zeroed) and
 *     the matching VT_DEV_* bit is OR-ed into `*status` when a status word is
 *     given.  Kernels never trap.
 *   - Page size is 16 tokens.  Supported head shapes: (head_dim, head_dim_v) =
 *     (64, 64) or (128, 128) with 1 <= Hq/Hkv <= 8, and the MLA latent form
 *     (576, 512) with Hkv == 1, Hq in {16, 32} and v_pool == k_pool (V is the
 *     first 512 dims of the K row, read from the same copy).
 */
#ifndef VT_H_
#define VT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define VT_ABI_VERSION 1
#define VT_PAGE_SIZE 16
#define VT_MAX_PAGES_PER_REQUEST 32768 /* page-table row length the kernels accept */

typedef enum {
  VT_OK = 0,
  VT_ERR_INVALID_ARG = 1, /* null pointer, negative count, inconsistent sizes */
  VT_ERR_UNSUPPORTED = 2, /* shape, stride or alignment with no kernel in this build */
  VT_ERR_CUDA = 3         /* a CUDA runtime call or a kernel launch failed */
} vt_status;

/* Bits OR-ed into the optional device status word by the kernels. */
#define VT_DEV_BAD_PAGE 1 /* a page id outside [0, num_pages); that unit/page was skipped */
#define VT_DEV_BAD_LEN 2  /* seq_len < 1, or ceil(seq_len/16) > pt_stride; unit skipped */
#define VT_DEV_BAD_SEL 4  /* n_sel or a sel entry out of range (vt_sparse_decode); unit skipped */
#define VT_DEV_BAD_ORDER 8 /* an `order` entry outside [0, B); that request slot was skipped */
#define VT_DEV_TIMEOUT 16  /* a wait for work published by another CTA gave up (never expected) */

/*
 * Paged K/V layout ("vTensor" metadata, reduced to one descriptor).
 * K element (page p, token t, kv head h, dim d) is
 *   ((const bf16*)k_pool)[p*sk_p + t*sk_t + h*sk_h + d], d < head_dim;
 * V element likewise with v_pool / sv_*, d < head_dim_v.  Strides are in
 * elements; the innermost stride is 1.  Both pools must be 16-byte aligned
 * and every stride a multiple of 8 elements (16 bytes).  For the MLA latent
 * form, V is the first 512 dims of the K row: pass v_pool == k_pool and the
 * same strides.
 */
typedef struct {
  const void* k_pool;
  const void* v_pool;
  int64_t num_pages;    /* P: physical pages in the pool */
  int32_t page_size;    /* must be VT_PAGE_SIZE */
  int32_t num_kv_heads; /* Hkv */
  int32_t head_dim;     /* D: query/key dimension */
  int32_t head_dim_v;   /* Dv: value dimension */
  int64_t sk_p, sk_t, sk_h;
  int64_t sv_p, sv_t, sv_h;
} vt_paged_kv;

/*
 * Per-step decode arguments.
 *   q           bf16 [B, Hq, D], contiguous; query head hq belongs to KV head hq / (Hq/Hkv)
 *   page_table  int32 [B, pt_stride]; entry (b, i) is the physical page of logical page i
 *   seq_lens    int32 [B]; tokens of request b INCLUDING the one being decoded (its K/V is
 *               already in the pool); logical pages n_b = ceil(seq_lens[b] / 16), the last
 *               of which holds seq_lens[b] - 16 (n_b - 1) valid tokens
 *   centroids   fp32 [P, Hkv, D], contiguous (vt_build_centroids output); read only for
 *               the candidate pages [bos, n_b - eos) of requests with n_b > topk+bos+eos
 *   topk, bos, eos  >= 0; kmax = topk + bos + eos.  A request with n_b <= kmax attends to
 *               every page; otherwise to pages {0..bos-1} U {n_b-eos..n_b-1} U the topk
 *               candidates with the highest score qm . centroid (ties -> lower index)
 *   sm_scale    softmax scale applied to q . k (e.g. 1/sqrt(D))
 *   order       optional int32 [B] permutation: the order in which requests are scheduled
 *               (vt_plan_requests output); NULL = 0..B-1.  Results do not depend on it.
 *   status      optional device int32 word receiving VT_DEV_* bits; NULL = not reported
 */
typedef struct {
  int32_t batch;       /* B */
  int32_t num_q_heads; /* Hq, a multiple of Hkv */
  const void* q;
  const int32_t* page_table;
  int64_t pt_stride;
  const int32_t* seq_lens;
  const float* centroids;
  int32_t topk, bos, eos;
  float sm_scale;
  const int32_t* order;
  int32_t* status;
} vt_decode_args;

/*
 * Cache side (README "Quick Example", forward_cache with CMean(dim=1), run
 * when a page is finished; create_cache declares one (1, head_dim) centroid
 * per page):  for each listed physical page p and KV head h,
 *   centroids[p, h, :] = (1/16) * sum_{t<16} K[p, t, h, :]
 * accumulated in fp64 and rounded once to fp32.  pages: int32 [n_pages]
 * physical ids (the finished pages, "loc"); rows of other pages are not
 * touched.  A listed id outside [0, num_pages) is skipped (VT_DEV_BAD_PAGE).
 */
vt_status vt_build_centroids(const vt_paged_kv* kv, const int32_t* pages, int32_t n_pages,
                             float* centroids, int32_t* status, void* stream);

/*
 * Indexer (README "Quick Example", forward_indexer: q.mean -> GeMV against the
 * centroids -> topK; reserved pages from vortex_page_reserved_bos/eos):
 * writes, per request b and KV head h, the selected logical page indices in
 * ascending order to sel[(b*Hkv + h)*kmax + j], j < n_sel[b*Hkv + h], and -1
 * in the remaining slots.  sel: int32 [B, Hkv, kmax]; n_sel: int32 [B, Hkv].
 * Scores are fp32 dot products of the fp32 group mean with the centroids.
 */
vt_status vt_select_pages(const vt_paged_kv* kv, const vt_decode_args* a, int32_t* sel,
                          int32_t* n_sel, void* stream);

/*
 * vt_select_pages with a workspace (vt_fused_workspace_size() bytes, 256-byte aligned, zeroed
 * once, shared with the fused call under the same rules): for B <= 2048 the selection then
 * runs on the fused call's persistent CTAs (GQA heads: scan items only, the unit's last
 * counted chunk merging its candidates; the MLA form: scan items and one merge item per
 * request) ("a workload planner for balanced GPU scheduling", rndamp.com article, "A
 * dual-stage programmable abstraction").  Same results and errors as vt_select_pages;
 * without a workspace, or for B > 2048, it is vt_select_pages.
 */
vt_status vt_select_pages_ws(const vt_paged_kv* kv, const vt_decode_args* a, int32_t* sel,
                             int32_t* n_sel, void* workspace, size_t workspace_bytes,
                             void* stream);

/*
 * The indexer's lossy mode ("stochastic radix top-k": a lossy, early-terminating top-k for
 * the indexing stage, rndamp.com article, "A dual-stage programmable abstraction"), as
 * vt_select_pages with the exact top-k replaced by one radix pass that stops there:
 *   - the candidates' fp32 scores go into 1024 bins linear between their smallest and
 *     largest score (IEEE fp32: bin = min(1023, (int)((s - lo) * (1024 / (hi - lo)))), one
 *     bin when hi == lo);
 *   - every candidate in a bin above the bin B of the topk-th largest score is kept;
 *   - B is not refined: its remaining slots go to its candidates in cyclic order of their
 *     position c = i - bos, starting at splitmix64(seed + b*Hkv + h) mod m (m candidates;
 *     SplitMix64's output step, Steele, Lea and Flood 2014).
 * The selected set always has topk candidates plus the reserved pages (same sel / n_sel
 * layout as vt_select_pages), and every candidate scoring a bin width or more above the
 * exact topk-th score is in it; pages of the same bin as the topk-th score may differ from
 * the exact top-k.  Same arguments, errors and status bits as vt_select_pages.
 */
vt_status vt_select_pages_approx(const vt_paged_kv* kv, const vt_decode_args* a, uint64_t seed,
                                 int32_t* sel, int32_t* n_sel, void* stream);

/*
 * Sparse attention over a given selection ("performs the actual attention" on
 * the selected blocks through the paged layout): for each query head hq of
 * request b, exact softmax(sm_scale * q K^T) V over the valid tokens of the
 * logical pages sel[b, hq/G, 0:n_sel[b, hq/G]] (any order, no duplicates).
 * out: bf16 [B, Hq, Dv]; lse: fp32 [B, Hq] natural-log sum of exp of the
 * scaled scores, or NULL.  Accumulation is fp32.  a->centroids, topk/bos/eos
 * are not used except kmax = topk+bos+eos, the row length of sel.
 */
vt_status vt_sparse_decode(const vt_paged_kv* kv, const vt_decode_args* a, const int32_t* sel,
                           const int32_t* n_sel, void* out, float* lse, void* stream);

/*
 * vt_sparse_decode with a workspace (as for vt_select_pages_ws): for B <= 2048 (GQA heads and
 * the MLA form) the attention then runs on the fused call's persistent CTAs, attention items
 * only, reading the given selection.  Same results and errors as vt_sparse_decode; without a
 * workspace, or for B > 2048, it is vt_sparse_decode.
 */
vt_status vt_sparse_decode_ws(const vt_paged_kv* kv, const vt_decode_args* a, const int32_t* sel,
                              const int32_t* n_sel, void* out, float* lse, void* workspace,
                              size_t workspace_bytes, void* stream);

/*
 * The whole query side in one call: selection + attention ("kernel fusion",
 * and "a workload planner for balanced GPU scheduling", rndamp.com article,
 * same section).  Same results as vt_select_pages followed by
 * vt_sparse_decode up to fp32 rounding (and, where two candidate pages score
 * within that rounding of each other, which of them is kept).  sel / n_sel
 * receive the selection when not NULL (both or neither).
 *
 * For B <= 2048 the work runs as one launch of persistent CTAs fed from a
 * queue of small scan and attention items that the CTAs derive from seq_lens
 * themselves (a->order is not used there), which keeps every SM busy on
 * batches of very uneven lengths; it needs `workspace`: device memory of vt_fused_workspace_size()
 * bytes, 256-byte aligned, ZERO-FILLED ONCE when allocated.  Every call
 * leaves it ready for the next one with the same B * Hkv, so it is zeroed
 * only once (its counter arrays are laid out for B * Hkv units: zero it again
 * before a call with another B * Hkv).  Calls that share a workspace must not
 * overlap on the GPU (use one stream, or one workspace per stream); after a
 * call that reported VT_DEV_TIMEOUT, zero it again.  When
 * vt_fused_workspace_size() is 0 (B > 2048) no workspace is used and
 * `workspace` may be NULL.
 */
vt_status vt_sparse_decode_fused(const vt_paged_kv* kv, const vt_decode_args* a, void* out,
                                 float* lse, int32_t* sel, int32_t* n_sel, void* workspace,
                                 size_t workspace_bytes, void* stream);

/*
 * One decode step of one layer in one launch: the cache-side centroid build of the pages
 * that filled at this step (as vt_build_centroids on fill_pages[0, n_fill)) and
 * vt_sparse_decode_fused, for a serving loop that runs both every step (README "Using Your
 * Sparse Attention with SGLang": the engine replays each step as a captured CUDA graph).
 * The build items run on the same persistent CTAs, ahead of the scans, and are not waited
 * for: a page filled at this step is its request's last page, which with eos >= 1 is a
 * reserved page that no score of this step reads.  So n_fill > 0 needs eos >= 1
 * (VT_ERR_UNSUPPORTED otherwise), `centroids` must be the cache args->centroids points to,
 * and fill_pages must hold only pages that this step does not score (the last page of their
 * request); other pages would be read while they are written.  Same workspace, results and
 * errors as vt_sparse_decode_fused; out-of-range fill_pages entries set VT_DEV_BAD_PAGE.
 * Where the fused call needs no workspace (B > 2048) the build is its own launch first.
 */
vt_status vt_sparse_decode_step(const vt_paged_kv* kv, const vt_decode_args* a,
                                const int32_t* fill_pages, int32_t n_fill, float* centroids,
                                void* out, float* lse, int32_t* sel, int32_t* n_sel,
                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * Bytes of workspace vt_sparse_decode_fused needs for these arguments (0 if
 * none); depends only on the shapes (B, Hq, Hkv, head dims, pt_stride, topk,
 * bos, eos), not on the data (args->centroids may be NULL).  Returns 0 as
 * well for arguments that vt_sparse_decode_fused would reject otherwise.  It sizes the
 * workspace of vt_select_pages_ws and vt_sparse_decode_ws too, for their own arguments.
 */
size_t vt_fused_workspace_size(const vt_paged_kv* kv, const vt_decode_args* a);

/*
 * vt_sparse_decode_fused on a scratch buffer held inside the library instead
 * of a caller-provided workspace, for callers that cannot allocate or keep
 * one.  The method's pages have no counterpart to this call: it is a
 * deployment convenience of this library.  Arguments, results and errors are
 * those of vt_sparse_decode_fused without workspace / workspace_bytes.
 *
 * The scratch is one file-scope device array of VT_STATIC_SCRATCH_BYTES on
 * each device the library is used on, placed and zero-filled by CUDA when the
 * library's module is loaded there (the library itself never allocates).
 * What must start at zero -- the work-queue and per-unit counters at the
 * start of the scratch -- is zero at load, and every complete call leaves it
 * zero again; the candidate and partial arrays after them are always written
 * before they are read.  A call whose vt_fused_workspace_size() exceeds
 * VT_STATIC_SCRATCH_BYTES fails with VT_ERR_UNSUPPORTED before anything is
 * launched; shapes that need no workspace (B > 2048) run as
 * vt_sparse_decode_fused does.
 *
 * The array's device address is looked up (cudaGetSymbolAddress) on every
 * call, in the current device's current context, so it stays right when a
 * context is destroyed and created again.  The first call on a device may
 * load the library's module there: make that first call before any stream
 * capture on the device.
 *
 * Races: every call on one device shares the one scratch.  Two calls that can
 * be on the GPU at the same time (different streams with no event ordering
 * them, e.g. from two host threads) take work items from each other's queue:
 * their results are wrong and their waits may end in VT_DEV_TIMEOUT.  Order
 * such calls (one stream, or events), or use vt_sparse_decode_fused with one
 * workspace per stream.  After a call that reported VT_DEV_TIMEOUT the
 * counters may be left nonzero, and later calls on that device may fail the
 * same way; only a new CUDA context (a new process) starts from zero again.
 */
#define VT_STATIC_SCRATCH_BYTES (32u << 20)
vt_status vt_sparse_decode_fused_static(const vt_paged_kv* kv, const vt_decode_args* a,
                                        void* out, float* lse, int32_t* sel, int32_t* n_sel,
                                        void* stream);

/*
 * Workload planner ("a workload planner for balanced GPU scheduling", same
 * article and section): writes to order[0..B) the request indices sorted by
 * page count, longest first (equal counts keep index order), so that long
 * scans start first.  The order can be computed once per decode step and
 * reused by every layer.  seq_lens, order: device int32 [B]; B <= 65536.
 */
vt_status vt_plan_requests(const int32_t* seq_lens, int32_t batch, int32_t* order, void* stream);

/* Static name of a status code. */
const char* vt_status_string(vt_status s);

/* One-line reason for the last non-OK status returned on this host thread ("" if none). */
const char* vt_last_error_detail(void);

/* VT_ABI_VERSION of the loaded library. */
int32_t vt_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* VT_H_ */
