/*
 * vt_oracle.c -- plain, slow, fp64 CPU oracle for block top-k sparse decode
 * attention over a paged KV cache (the "Vortex" block top-k flow).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the correctness reference that the
 * CUDA library is checked against.  Only the test suite, the smoke check and
 * the CPU-baseline leg of the benchmark may load it.  It shares no source,
 * header, table or helper with the CUDA path, and the CUDA path never calls it.
 *
 * What it computes follows the sources' description of the method:
 *   - "Vortex: A Flexible and Efficient Sparse Attention Framework" (GitHub
 *     README of vortex_torch), section "Quick Example: Custom Sparse
 *     Attention": the cache-side op CMean(dim=1) builds a per-page centroid
 *     (shape (1, head_dim) per page, declared by create_cache) when a page is
 *     finished; the indexer-side ops take the mean of the query heads, score
 *     it against the centroids with GeMV and keep the top-k pages.
 *   - same README, section "Using Your Sparse Attention with SGLang": page
 *     size 16, vortex_topk_val, vortex_page_reserved_bos/eos (first/last
 *     pages always attended).
 *   - "Vortex: Efficient and Programmable Sparse Attention Serving for AI
 *     Agents" (rndamp.com article), section "A dual-stage programmable
 *     abstraction": query-independent preprocessing builds block centroids;
 *     query-dependent execution scores, selects the top-k blocks and performs
 *     the actual attention over the paged layout.
 *
 * Readings where the sources are silent (each one is listed in the design
 * notes of the repository):
 *   - the query mean is taken per KV head over its GQA group of G = Hq/Hkv
 *     query heads (for Hkv = 1 this is the README's mean over all heads);
 *   - the score is the raw dot product (no softmax scale);
 *   - top-k counts only the middle pages [bos, n-eos); the reserved pages are
 *     added on top, so at most k+bos+eos pages are attended;
 *   - a request with n <= k+bos+eos pages attends to all of its pages;
 *   - equal scores are broken toward the lower logical page index;
 *   - centroids are stored as fp32 (the fp64 page sum divided by the page
 *     size, rounded once to nearest);
 *   - seq_len counts the token being decoded (its K/V is already in the pool);
 *   - the selected pages are written in ascending logical order, -1 padded.
 *
 * Precision: every sum, dot product, exponential and division is done in
 * fp64 from the stored bf16/fp32 inputs.  Inputs in bf16 are passed as their
 * raw 16-bit patterns (a bf16 value is the upper half of an IEEE binary32).
 */
#include <stdint.h>
#include <tgmath.h> /* exp and log follow the argument type (fp64 unless VTO_REAL says otherwise) */
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define VTO_OK 0
#define VTO_ERR_ARG 1       /* a size, count or pointer argument is invalid */
#define VTO_ERR_LEN 2       /* a seq_len is < 1 or needs more pages than the page table holds */
#define VTO_ERR_PAGE 3      /* a page id is outside [0, num_pages) */

/* The arithmetic type.  fp64 is the oracle; -DVTO_REAL=float builds a timing-only copy that
 * the benchmark uses as a CPU baseline without the fp64 handicap (never as a reference). */
#ifndef VTO_REAL
#define VTO_REAL double
#endif
typedef VTO_REAL vto_real;

static int g_threads = 0; /* 0: OpenMP default */

void vto_set_threads(int n) { g_threads = n; }

int vto_get_threads(void) {
#ifdef _OPENMP
  return g_threads > 0 ? g_threads : omp_get_max_threads();
#else
  return 1;
#endif
}

/* bf16 -> the arithmetic type (exact).  A bf16 value is the upper 16 bits of a binary32. */
static vto_real bf16_to_f64(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (vto_real)f;
}

static int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

/* ------------------------------------------------------------------------ */
/* Cache side: CMean(dim=1) over the tokens of each finished page.           */
/* ------------------------------------------------------------------------ */

/*
 * centroids[p, h, d] = (float)( (sum_{t < page_size} K[p, t, h, d]) / page_size )
 * for every physical page p listed in pages[0..n_pages).  Rows of pages not
 * listed are left untouched.  K element (p,t,h,d) is at
 * k_pool[p*sk_p + t*sk_t + h*sk_h + d]; centroids is [num_pages, Hkv, D].
 */
int vto_build_centroids(const uint16_t* k_pool, int64_t num_pages, int32_t page_size,
                        int32_t num_kv_heads, int32_t head_dim, int64_t sk_p, int64_t sk_t,
                        int64_t sk_h, const int32_t* pages, int32_t n_pages, float* centroids) {
  if (!k_pool || !centroids || (n_pages > 0 && !pages)) return VTO_ERR_ARG;
  if (num_pages < 1 || page_size < 1 || num_kv_heads < 1 || head_dim < 1 || n_pages < 0)
    return VTO_ERR_ARG;
  for (int32_t i = 0; i < n_pages; ++i)
    if (pages[i] < 0 || pages[i] >= num_pages) return VTO_ERR_PAGE;
  const int64_t rows = (int64_t)n_pages * num_kv_heads;
#pragma omp parallel for schedule(static) num_threads(vto_get_threads())
  for (int64_t r = 0; r < rows; ++r) {
    const int64_t p = pages[r / num_kv_heads];
    const int64_t h = r % num_kv_heads;
    float* out = centroids + (p * num_kv_heads + h) * head_dim;
    for (int32_t d = 0; d < head_dim; ++d) {
      vto_real sum = 0.0;
      for (int32_t t = 0; t < page_size; ++t)
        sum += bf16_to_f64(k_pool[p * sk_p + t * sk_t + h * sk_h + d]);
      out[d] = (float)(sum / (vto_real)page_size);
    }
  }
  return VTO_OK;
}

/* ------------------------------------------------------------------------ */
/* Query side: group mean -> GeMV against centroids -> topK (+ reserved).    */
/* ------------------------------------------------------------------------ */

typedef struct {
  vto_real score;
  int32_t index; /* logical page index */
} vto_cand;

/* Order: higher score first; equal scores -> lower logical index first. */
static int cand_cmp(const void* a, const void* b) {
  const vto_cand* x = (const vto_cand*)a;
  const vto_cand* y = (const vto_cand*)b;
  if (x->score > y->score) return -1;
  if (x->score < y->score) return 1;
  return (x->index > y->index) - (x->index < y->index);
}

static int check_lengths(const int32_t* seq_lens, int32_t batch, int32_t page_size,
                         int64_t pt_stride) {
  for (int32_t b = 0; b < batch; ++b) {
    if (seq_lens[b] < 1) return VTO_ERR_LEN;
    if (ceil_div64(seq_lens[b], page_size) > pt_stride) return VTO_ERR_LEN;
  }
  return VTO_OK;
}

/*
 * Per request b and KV head h (G = Hq / Hkv):
 *   n    = ceil(seq_lens[b] / page_size)
 *   qm   = (1/G) * sum_{j<G} q[b, h*G + j, :]
 *   if n <= topk + bos + eos: selected = {0 .. n-1}
 *   else: s_i = qm . centroids[page_table[b, i], h, :] for i in [bos, n-eos);
 *         selected = {0..bos-1} U {n-eos..n-1} U the topk candidates ranked by
 *         (s descending, i ascending).
 * sel is [B, Hkv, kmax] (kmax = topk+bos+eos), ascending logical indices,
 * -1 padded; n_sel is [B, Hkv].  If scores is not NULL it is [B, Hkv, pt_stride]
 * and receives s_i at the candidates of sparse requests and NaN elsewhere.
 */
int vto_select_pages(const uint16_t* q, int32_t batch, int32_t num_q_heads,
                     int32_t num_kv_heads, int32_t head_dim, const int32_t* page_table,
                     int64_t pt_stride, const int32_t* seq_lens, const float* centroids,
                     int64_t num_pages, int32_t page_size, int32_t topk, int32_t bos,
                     int32_t eos, int32_t* sel, int32_t* n_sel, double* scores) {
  if (!q || !page_table || !seq_lens || !centroids || !sel || !n_sel) return VTO_ERR_ARG;
  if (batch < 0 || num_kv_heads < 1 || num_q_heads < num_kv_heads ||
      num_q_heads % num_kv_heads != 0 || head_dim < 1 || page_size < 1 || topk < 0 ||
      bos < 0 || eos < 0 || pt_stride < 1)
    return VTO_ERR_ARG;
  int rc = check_lengths(seq_lens, batch, page_size, pt_stride);
  if (rc) return rc;
  for (int32_t b = 0; b < batch; ++b) {
    const int64_t n = ceil_div64(seq_lens[b], page_size);
    for (int64_t i = 0; i < n; ++i) {
      const int32_t p = page_table[(int64_t)b * pt_stride + i];
      if (p < 0 || p >= num_pages) return VTO_ERR_PAGE;
    }
  }
  const int32_t G = num_q_heads / num_kv_heads;
  const int32_t kmax = topk + bos + eos;
  const int64_t units = (int64_t)batch * num_kv_heads;
  if (scores)
    for (int64_t i = 0; i < units * pt_stride; ++i) scores[i] = NAN;

#pragma omp parallel num_threads(vto_get_threads())
  {
    vto_real* qm = (vto_real*)malloc(sizeof(vto_real) * (size_t)head_dim);
    vto_cand* cand = (vto_cand*)malloc(sizeof(vto_cand) * (size_t)pt_stride);
    char* keep = (char*)malloc((size_t)pt_stride);
#pragma omp for schedule(dynamic, 1)
    for (int64_t u = 0; u < units; ++u) {
      const int32_t b = (int32_t)(u / num_kv_heads);
      const int32_t h = (int32_t)(u % num_kv_heads);
      const int32_t n = (int32_t)ceil_div64(seq_lens[b], page_size);
      int32_t* out = sel + u * kmax;
      for (int32_t j = 0; j < kmax; ++j) out[j] = -1;

      if (n <= kmax) { /* dense rule: every page is attended */
        for (int32_t i = 0; i < n; ++i) out[i] = i;
        n_sel[u] = n;
        continue;
      }
      /* q.mean over the G query heads of this KV head */
      for (int32_t d = 0; d < head_dim; ++d) {
        vto_real s = 0.0;
        for (int32_t j = 0; j < G; ++j)
          s += bf16_to_f64(q[((int64_t)b * num_q_heads + (int64_t)h * G + j) * head_dim + d]);
        qm[d] = s / (vto_real)G;
      }
      /* GeMV against the centroid of every middle page */
      int32_t m = 0;
      for (int32_t i = bos; i < n - eos; ++i) {
        const int64_t p = page_table[(int64_t)b * pt_stride + i];
        const float* c = centroids + (p * num_kv_heads + h) * head_dim;
        vto_real s = 0.0;
        for (int32_t d = 0; d < head_dim; ++d) s += qm[d] * (vto_real)c[d];
        cand[m].score = s;
        cand[m].index = i;
        ++m;
        if (scores) scores[u * pt_stride + i] = s;
      }
      /* topK: full sort by (score desc, index asc), keep the first topk */
      qsort(cand, (size_t)m, sizeof(vto_cand), cand_cmp);
      memset(keep, 0, (size_t)n);
      for (int32_t i = 0; i < bos; ++i) keep[i] = 1;
      for (int32_t i = n - eos; i < n; ++i) keep[i] = 1;
      for (int32_t j = 0; j < topk && j < m; ++j) keep[cand[j].index] = 1;
      int32_t c = 0;
      for (int32_t i = 0; i < n; ++i)
        if (keep[i]) out[c++] = i;
      n_sel[u] = c;
    }
    free(qm);
    free(cand);
    free(keep);
  }
  return VTO_OK;
}

/* ------------------------------------------------------------------------ */
/* Lossy mode of the indexer: an early-terminating ("stochastic radix") top-k. */
/* ------------------------------------------------------------------------ */

/* SplitMix64's output step (Steele, Lea and Flood, "Fast splittable pseudorandom number
 * generators", OOPSLA 2014): advance by the golden gamma, then the two xor-shift-multiply
 * rounds.  The counter-based generator the lossy mode draws its random start from. */
static uint64_t vto_splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

/*
 * The indexer's "stochastic radix top-k" (rndamp.com article, "A dual-stage programmable
 * abstraction": a lossy top-k with early termination, for the indexing stage), read as:
 * one radix pass over the candidates' scores, then stop.  Per unit with n > kmax:
 *   - scores s_i as in vto_select_pages, rounded to fp32 (f_i; the kernels decide in fp32);
 *   - lo, hi = the smallest and largest f_i; if hi > lo (and finite) each candidate gets
 *     bin_i = min(1023, (int)((f_i - lo) * (1024 / (hi - lo)))), every step in fp32;
 *     otherwise every candidate is in bin 0;
 *   - B = the bin holding the topk-th largest score (counting bins from the top);
 *   - every candidate in a bin above B is kept; instead of refining inside B the pass
 *     ends there: the remaining need slots go to B's candidates in cyclic order of their
 *     position c = i - bos, starting at r = splitmix64(seed + b*Hkv + h) mod m.
 * The reserved pages and the dense rule are those of vto_select_pages.
 */
int vto_select_pages_approx(const uint16_t* q, int32_t batch, int32_t num_q_heads,
                            int32_t num_kv_heads, int32_t head_dim, const int32_t* page_table,
                            int64_t pt_stride, const int32_t* seq_lens, const float* centroids,
                            int64_t num_pages, int32_t page_size, int32_t topk, int32_t bos,
                            int32_t eos, uint64_t seed, int32_t* sel, int32_t* n_sel) {
  if (batch < 0 || num_q_heads < 1 || num_kv_heads < 1 || head_dim < 1 || page_size < 1 ||
      pt_stride < 1 || topk < 0 || bos < 0 || eos < 0 || num_q_heads % num_kv_heads != 0)
    return VTO_ERR_ARG;
  int rc = check_lengths(seq_lens, batch, page_size, pt_stride);
  if (rc) return rc;
  const int32_t G = num_q_heads / num_kv_heads;
  const int32_t kmax = topk + bos + eos;
  const int64_t units = (int64_t)batch * num_kv_heads;
  int bad_page = 0;
#pragma omp parallel num_threads(vto_get_threads()) reduction(| : bad_page)
  {
    vto_real* qm = (vto_real*)malloc(sizeof(vto_real) * (size_t)head_dim);
    float* f = (float*)malloc(sizeof(float) * (size_t)pt_stride);
    int32_t* bin = (int32_t*)malloc(sizeof(int32_t) * (size_t)pt_stride);
    char* keep = (char*)malloc((size_t)pt_stride);
#pragma omp for schedule(dynamic, 1)
    for (int64_t u = 0; u < units; ++u) {
      const int32_t b = (int32_t)(u / num_kv_heads);
      const int32_t h = (int32_t)(u % num_kv_heads);
      const int32_t n = (int32_t)ceil_div64(seq_lens[b], page_size);
      int32_t* out = sel + u * kmax;
      for (int32_t j = 0; j < kmax; ++j) out[j] = -1;
      if (n <= kmax) {
        for (int32_t i = 0; i < n; ++i) out[i] = i;
        n_sel[u] = n;
        continue;
      }
      for (int32_t d = 0; d < head_dim; ++d) {
        vto_real s = 0.0;
        for (int32_t j = 0; j < G; ++j)
          s += bf16_to_f64(q[((int64_t)b * num_q_heads + (int64_t)h * G + j) * head_dim + d]);
        qm[d] = s / (vto_real)G;
      }
      const int32_t m = n - bos - eos;
      float lo = INFINITY, hi = -INFINITY;
      for (int32_t c = 0; c < m; ++c) {
        const int64_t p = page_table[(int64_t)b * pt_stride + bos + c];
        if (p < 0 || p >= num_pages) {
          bad_page = 1;
          f[c] = -INFINITY;
          continue;
        }
        const float* cr = centroids + (p * num_kv_heads + h) * head_dim;
        vto_real s = 0.0;
        for (int32_t d = 0; d < head_dim; ++d) s += qm[d] * (vto_real)cr[d];
        f[c] = (float)s;
        if (f[c] < lo) lo = f[c];
        if (f[c] > hi) hi = f[c];
      }
      const float width = hi - lo;
      const int linear = hi > lo && isfinite(width);
      const float inv = linear ? 1024.0f / width : 0.0f;
      int32_t count[1024];
      memset(count, 0, sizeof count);
      for (int32_t c = 0; c < m; ++c) {
        int32_t k = 0;
        if (linear) {
          const float x = (f[c] - lo) * inv;
          k = x >= 1023.0f ? 1023 : (int32_t)x;
        }
        bin[c] = k;
        count[k] += 1;
      }
      int32_t B = 1023, above = 0;
      while (B > 0 && above + count[B] < topk) above += count[B--];
      int32_t need = topk - above;
      memset(keep, 0, (size_t)n);
      for (int32_t i = 0; i < bos; ++i) keep[i] = 1;
      for (int32_t i = n - eos; i < n; ++i) keep[i] = 1;
      for (int32_t c = 0; c < m; ++c)
        if (bin[c] > B) keep[bos + c] = 1;
      const int32_t r = (int32_t)(vto_splitmix64(seed + (uint64_t)u) % (uint64_t)m);
      for (int32_t t = 0; t < m && need > 0; ++t) {
        const int32_t c = (r + t) % m;
        if (bin[c] == B) {
          keep[bos + c] = 1;
          --need;
        }
      }
      int32_t cnt = 0;
      for (int32_t i = 0; i < n; ++i)
        if (keep[i]) out[cnt++] = i;
      n_sel[u] = cnt;
    }
    free(qm);
    free(f);
    free(bin);
    free(keep);
  }
  return bad_page ? VTO_ERR_PAGE : VTO_OK;
}

/* ------------------------------------------------------------------------ */
/* Exact softmax attention over the selected pages.                          */
/* ------------------------------------------------------------------------ */

/*
 * For request b, query head hq (KV head h = hq / G), over every token t of
 * every selected logical page i (the last page n-1 holds only
 * seq_lens[b] - page_size*(n-1) valid tokens):
 *   z    = sm_scale * q[b,hq,:] . K[page_table[b,i], t, h, :]
 *   out  = sum softmax(z) * V[page_table[b,i], t, h, 0:Dv]
 *   lse  = log(sum exp(z))        (natural log)
 * sel / n_sel as produced by vto_select_pages (any order, no duplicates).
 * out is [B, Hq, Dv] fp64, lse is [B, Hq] fp64 (may be NULL).
 */
int vto_sparse_attention(const uint16_t* q, int32_t batch, int32_t num_q_heads,
                         int32_t num_kv_heads, int32_t head_dim, int32_t head_dim_v,
                         const uint16_t* k_pool, int64_t sk_p, int64_t sk_t, int64_t sk_h,
                         const uint16_t* v_pool, int64_t sv_p, int64_t sv_t, int64_t sv_h,
                         int64_t num_pages, int32_t page_size, const int32_t* page_table,
                         int64_t pt_stride, const int32_t* seq_lens, const int32_t* sel,
                         const int32_t* n_sel, int32_t kmax, double sm_scale, double* out,
                         double* lse) {
  if (!q || !k_pool || !v_pool || !page_table || !seq_lens || !sel || !n_sel || !out)
    return VTO_ERR_ARG;
  if (batch < 0 || num_kv_heads < 1 || num_q_heads < num_kv_heads ||
      num_q_heads % num_kv_heads != 0 || head_dim < 1 || head_dim_v < 1 || page_size < 1 ||
      kmax < 0 || pt_stride < 1)
    return VTO_ERR_ARG;
  int rc = check_lengths(seq_lens, batch, page_size, pt_stride);
  if (rc) return rc;
  const int32_t G = num_q_heads / num_kv_heads;
  const int64_t units = (int64_t)batch * num_kv_heads;
  for (int64_t u = 0; u < units; ++u) {
    const int32_t b = (int32_t)(u / num_kv_heads);
    const int32_t n = (int32_t)ceil_div64(seq_lens[b], page_size);
    if (n_sel[u] < 0 || n_sel[u] > kmax) return VTO_ERR_ARG;
    for (int32_t j = 0; j < n_sel[u]; ++j) {
      const int32_t i = sel[u * kmax + j];
      if (i < 0 || i >= n) return VTO_ERR_ARG;
      const int32_t p = page_table[(int64_t)b * pt_stride + i];
      if (p < 0 || p >= num_pages) return VTO_ERR_PAGE;
    }
  }

#pragma omp parallel num_threads(vto_get_threads())
  {
    const int64_t max_tokens = (int64_t)kmax * page_size;
    vto_real* z = (vto_real*)malloc(sizeof(vto_real) * (size_t)(max_tokens > 0 ? max_tokens : 1));
    vto_real* acc = (vto_real*)malloc(sizeof(vto_real) * (size_t)(head_dim_v > 0 ? head_dim_v : 1));
    const uint16_t** vrow =
        (const uint16_t**)malloc(sizeof(uint16_t*) * (size_t)(max_tokens > 0 ? max_tokens : 1));
#pragma omp for schedule(dynamic, 1)
    for (int64_t u = 0; u < units; ++u) {
      const int32_t b = (int32_t)(u / num_kv_heads);
      const int32_t h = (int32_t)(u % num_kv_heads);
      const int32_t L = seq_lens[b];
      const int32_t n = (int32_t)ceil_div64(L, page_size);
      for (int32_t j = 0; j < G; ++j) {
        const int64_t hq = (int64_t)h * G + j;
        const uint16_t* qrow = q + ((int64_t)b * num_q_heads + hq) * head_dim;
        int64_t T = 0;
        vto_real zmax = -INFINITY;
        for (int32_t s = 0; s < n_sel[u]; ++s) {
          const int32_t i = sel[u * kmax + s];
          const int64_t p = page_table[(int64_t)b * pt_stride + i];
          const int32_t valid = (i == n - 1) ? L - page_size * (n - 1) : page_size;
          for (int32_t t = 0; t < valid; ++t) {
            const uint16_t* krow = k_pool + p * sk_p + t * sk_t + h * sk_h;
            vto_real dot = 0.0;
            for (int32_t d = 0; d < head_dim; ++d) dot += bf16_to_f64(qrow[d]) * bf16_to_f64(krow[d]);
            z[T] = (vto_real)sm_scale * dot;
            vrow[T] = v_pool + p * sv_p + t * sv_t + h * sv_h;
            if (z[T] > zmax) zmax = z[T];
            ++T;
          }
        }
        double* o = out + ((int64_t)b * num_q_heads + hq) * head_dim_v;
        for (int32_t d = 0; d < head_dim_v; ++d) acc[d] = 0.0;
        vto_real l = 0.0;
        for (int64_t t = 0; t < T; ++t) {
          const vto_real w = exp(z[t] - zmax);
          l += w;
          for (int32_t d = 0; d < head_dim_v; ++d) acc[d] += w * bf16_to_f64(vrow[t][d]);
        }
        for (int32_t d = 0; d < head_dim_v; ++d) o[d] = (T > 0) ? acc[d] / l : 0.0;
        if (lse) lse[(int64_t)b * num_q_heads + hq] = (T > 0) ? zmax + log(l) : -INFINITY;
      }
    }
    free(z);
    free(acc);
    free((void*)vrow);
  }
  return VTO_OK;
}

/* One whole decode step: select the pages, then attend over them. */
int vto_decode_step(const uint16_t* q, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                    int32_t head_dim, int32_t head_dim_v, const uint16_t* k_pool, int64_t sk_p,
                    int64_t sk_t, int64_t sk_h, const uint16_t* v_pool, int64_t sv_p,
                    int64_t sv_t, int64_t sv_h, int64_t num_pages, int32_t page_size,
                    const int32_t* page_table, int64_t pt_stride, const int32_t* seq_lens,
                    const float* centroids, int32_t topk, int32_t bos, int32_t eos,
                    double sm_scale, int32_t* sel, int32_t* n_sel, double* out, double* lse) {
  int rc = vto_select_pages(q, batch, num_q_heads, num_kv_heads, head_dim, page_table, pt_stride,
                            seq_lens, centroids, num_pages, page_size, topk, bos, eos, sel, n_sel,
                            NULL);
  if (rc) return rc;
  return vto_sparse_attention(q, batch, num_q_heads, num_kv_heads, head_dim, head_dim_v, k_pool,
                              sk_p, sk_t, sk_h, v_pool, sv_p, sv_t, sv_h, num_pages, page_size,
                              page_table, pt_stride, seq_lens, sel, n_sel, topk + bos + eos,
                              sm_scale, out, lse);
}
