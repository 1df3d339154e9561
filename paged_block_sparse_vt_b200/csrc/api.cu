// api.cu -- the C ABI of libvt (include/vt.h): host-side argument checks, kernel choice and
// launch.  No allocation, no synchronisation: every call only enqueues work on `stream`.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <atomic>

#include "decode_params.cuh"

namespace vt {
cudaError_t launch_build_centroids(const vt_paged_kv& kv, const int32_t* pages, int n_pages,
                                   float* centroids, int32_t* status, cudaStream_t stream);
cudaError_t launch_gqa_decode(const DecodeParams& p, int mode, int D, int G, int C,
                              cudaStream_t s);
int gqa_smem_bytes(int D, int G, int cand_cap, int key_cap, int kmax);
cudaError_t launch_mla_decode(const DecodeParams& p, int mode, int G, int C, cudaStream_t s);
int mla_smem_bytes(int G, int cand_cap, int key_cap, int kmax, int pages_per_cta);
int mla_max_pages_per_cta();
cudaError_t launch_plan(const int32_t* seq_lens, int B, int32_t* order, cudaStream_t s);
size_t persist_workspace_bytes(const DecodeParams& p, int G, int Dv, int64_t unit_cap);
int persist_smem_bytes(const DecodeParams& p, int D, int G);
int persist_max_batch();
size_t mla_persist_workspace_bytes(const DecodeParams& p, int G, int64_t unit_cap);
int mla_persist_smem_bytes(const DecodeParams& p, int G);
int mla_persist_max_batch();
cudaError_t launch_mla_persist(const DecodeParams& p, int G, void* ws, int64_t unit_cap,
                               int sm_count, cudaStream_t s, int mode);
cudaError_t launch_persist_fused(const DecodeParams& p, int D, int G, void* ws, int64_t unit_cap,
                                 int sm_count, cudaStream_t s, int mode);
}  // namespace vt

using namespace vt;

namespace {

thread_local char g_detail[256] = "";

vt_status fail(vt_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_detail, sizeof g_detail, fmt, ap);
  va_end(ap);
  return s;
}

vt_status ok() {
  g_detail[0] = '\0';
  return VT_OK;
}

vt_status cuda_fail(cudaError_t e, const char* what) {
  return fail(VT_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

enum Path { kPathGqa = 1, kPathMla = 2 };

struct Shape {
  Path path;
  int D, Dv, G;
};

vt_status check_kv(const vt_paged_kv* kv) {
  if (!kv) return fail(VT_ERR_INVALID_ARG, "kv descriptor is NULL");
  if (!kv->k_pool || !kv->v_pool) return fail(VT_ERR_INVALID_ARG, "k_pool/v_pool is NULL");
  if (kv->page_size != VT_PAGE_SIZE)
    return fail(VT_ERR_UNSUPPORTED, "page_size %d (only %d is supported)", kv->page_size,
                VT_PAGE_SIZE);
  if (kv->num_pages < 1) return fail(VT_ERR_INVALID_ARG, "num_pages %lld < 1", (long long)kv->num_pages);
  if (kv->num_pages > (int64_t)INT32_MAX)
    return fail(VT_ERR_UNSUPPORTED, "num_pages above 2^31-1");
  if (kv->num_kv_heads < 1) return fail(VT_ERR_INVALID_ARG, "num_kv_heads < 1");
  if (kv->head_dim < 1 || kv->head_dim_v < 1) return fail(VT_ERR_INVALID_ARG, "head dims < 1");
  if (!aligned16(kv->k_pool) || !aligned16(kv->v_pool))
    return fail(VT_ERR_UNSUPPORTED, "k_pool/v_pool not 16-byte aligned");
  const int64_t st[6] = {kv->sk_p, kv->sk_t, kv->sk_h, kv->sv_p, kv->sv_t, kv->sv_h};
  for (int i = 0; i < 6; ++i)
    if (st[i] < 0 || st[i] % 8 != 0)
      return fail(VT_ERR_UNSUPPORTED, "pool strides must be non-negative multiples of 8 elements");
  return ok();
}

vt_status classify(const vt_paged_kv* kv, int Hq, Shape* sh) {
  const int Hkv = kv->num_kv_heads;
  if (Hq < Hkv || Hq % Hkv != 0)
    return fail(VT_ERR_INVALID_ARG, "num_q_heads %d is not a multiple of num_kv_heads %d", Hq, Hkv);
  const int G = Hq / Hkv;
  const int D = kv->head_dim, Dv = kv->head_dim_v;
  if ((D == 64 || D == 128) && Dv == D) {
    if (G > 8) return fail(VT_ERR_UNSUPPORTED, "GQA group %d > 8 with head_dim %d", G, D);
    *sh = Shape{kPathGqa, D, Dv, G};
    return ok();
  }
  if (D == 576 && Dv == 512) {
    if (Hkv != 1) return fail(VT_ERR_UNSUPPORTED, "MLA latent form needs num_kv_heads == 1");
    if (G != 16 && G != 32)
      return fail(VT_ERR_UNSUPPORTED, "MLA latent form supports 16 or 32 query heads, got %d", G);
    if (kv->v_pool != kv->k_pool || kv->sv_p != kv->sk_p || kv->sv_t != kv->sk_t ||
        kv->sv_h != kv->sk_h)
      return fail(VT_ERR_UNSUPPORTED, "MLA latent form needs v_pool == k_pool with equal strides");
    *sh = Shape{kPathMla, D, Dv, G};
    return ok();
  }
  return fail(VT_ERR_UNSUPPORTED, "head shape (%d, %d) has no kernel", D, Dv);
}

// SMs of the current device, looked up once per device.
int sm_count() {
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  std::atomic<int>& slot = cached[dev & 63];
  int n = slot.load(std::memory_order_relaxed);
  if (n > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
    return 148;
  slot.store(n, std::memory_order_relaxed);
  return n;
}

// Cluster size: CTAs that share one (request, KV head) unit.
int pick_cluster(const Shape& sh, int64_t units, int kmax) {
  if (sh.path == kPathMla) {
    int C = 8;
    while (C < 16 && (kmax + C - 1) / C > mla_max_pages_per_cta()) C *= 2;
    return C;
  }
  // One deep CTA per unit as soon as the units alone cover every SM (fewer, longer
  // pipelines beat more, shorter ones); otherwise split units so that every SM has work.
  const int64_t sms = sm_count();
  if (units >= sms) return 1;
  if (units * 2 >= sms) return 2;
  if (units * 4 >= sms) return 4;
  return 8;
}

vt_status fill_params(const vt_paged_kv* kv, const vt_decode_args* a, bool need_centroids,
                      Shape* sh, DecodeParams* p) {
  vt_status s = check_kv(kv);
  if (s != VT_OK) return s;
  if (!a) return fail(VT_ERR_INVALID_ARG, "args is NULL");
  if (a->batch < 0) return fail(VT_ERR_INVALID_ARG, "batch < 0");
  if (a->batch > 0) {
    if (!a->q || !a->page_table || !a->seq_lens)
      return fail(VT_ERR_INVALID_ARG, "q/page_table/seq_lens is NULL");
    if (need_centroids && !a->centroids) return fail(VT_ERR_INVALID_ARG, "centroids is NULL");
  }
  s = classify(kv, a->num_q_heads, sh);
  if (s != VT_OK) return s;
  if (a->pt_stride < 1 || a->pt_stride > VT_MAX_PAGES_PER_REQUEST)
    return fail(VT_ERR_UNSUPPORTED, "pt_stride %lld outside [1, %d]", (long long)a->pt_stride,
                VT_MAX_PAGES_PER_REQUEST);
  if (a->topk < 0 || a->bos < 0 || a->eos < 0)
    return fail(VT_ERR_INVALID_ARG, "topk/bos/eos must be >= 0");
  const int64_t kmax = (int64_t)a->topk + a->bos + a->eos;
  if (kmax < 1) return fail(VT_ERR_INVALID_ARG, "topk + bos + eos must be >= 1");
  if (kmax > 4096) return fail(VT_ERR_UNSUPPORTED, "topk + bos + eos > 4096");
  if (!std::isfinite(a->sm_scale)) return fail(VT_ERR_INVALID_ARG, "sm_scale is not finite");
  if (a->q && !aligned16(a->q)) return fail(VT_ERR_UNSUPPORTED, "q not 16-byte aligned");
  if (a->centroids && !aligned16(a->centroids))
    return fail(VT_ERR_UNSUPPORTED, "centroids not 16-byte aligned");
  const int64_t units = (int64_t)a->batch * kv->num_kv_heads;
  if (units * 16 > (int64_t)INT32_MAX) return fail(VT_ERR_UNSUPPORTED, "batch too large");

  *p = DecodeParams{};
  p->k_pool = static_cast<const __nv_bfloat16*>(kv->k_pool);
  p->v_pool = static_cast<const __nv_bfloat16*>(kv->v_pool);
  p->num_pages = kv->num_pages;
  p->Hkv = kv->num_kv_heads;
  p->sk_p = kv->sk_p; p->sk_t = kv->sk_t; p->sk_h = kv->sk_h;
  p->sv_p = kv->sv_p; p->sv_t = kv->sv_t; p->sv_h = kv->sv_h;
  p->B = a->batch;
  p->Hq = a->num_q_heads;
  p->q = static_cast<const __nv_bfloat16*>(a->q);
  p->page_table = a->page_table;
  p->pt_stride = a->pt_stride;
  p->seq_lens = a->seq_lens;
  p->centroids = a->centroids;
  p->topk = a->topk;
  p->bos = a->bos;
  p->eos = a->eos;
  p->kmax = (int)kmax;
  p->qscale = a->sm_scale * kLog2e;
  p->order = a->order;
  p->status = a->status;
  return ok();
}

// The fused call runs on persistent CTAs (and needs a workspace) up to this many requests.
bool use_persistent(const Shape& sh, const vt_decode_args* a) {
  if (a->batch < 1) return false;
  if (sh.path == kPathMla) return a->batch <= mla_persist_max_batch();
  return sh.path == kPathGqa && a->batch <= persist_max_batch();
}

// Workspace of the persistent fused path (its counters laid out for unit_cap units, 0: B*Hkv).
size_t persist_bytes(const Shape& sh, const DecodeParams& p, int64_t unit_cap) {
  return sh.path == kPathMla ? mla_persist_workspace_bytes(p, sh.G, unit_cap)
                             : persist_workspace_bytes(p, sh.G, sh.Dv, unit_cap);
}

// unit_cap: units the persistent path's counter arrays are laid out for (0: exactly B * Hkv)
vt_status launch_query_side(const vt_paged_kv* kv, const vt_decode_args* a, int mode,
                            int32_t* sel, int32_t* n_sel, void* out, float* lse, void* ws,
                            size_t ws_bytes, void* stream, int64_t unit_cap = 0,
                            bool approx = false, uint64_t seed = 0,
                            const int32_t* fill_pages = nullptr, int n_fill = 0,
                            float* cent_out = nullptr, bool split_on_persistent = false) {
  Shape sh;
  DecodeParams p;
  vt_status s = fill_params(kv, a, mode != kDecode, &sh, &p);
  if (s != VT_OK) return s;
  if (mode != kSelect && !out) return fail(VT_ERR_INVALID_ARG, "out is NULL");
  if (mode == kSelect && (!sel || !n_sel)) return fail(VT_ERR_INVALID_ARG, "sel/n_sel is NULL");
  if (mode == kDecode && (!sel || !n_sel)) return fail(VT_ERR_INVALID_ARG, "sel/n_sel is NULL");
  if (mode == kFused && ((sel == nullptr) != (n_sel == nullptr)))
    return fail(VT_ERR_INVALID_ARG, "sel and n_sel must both be given or both be NULL");
  if (a->batch == 0) {
    if (n_fill > 0) {
      cudaError_t e = launch_build_centroids(*kv, fill_pages, n_fill, cent_out, a->status,
                                             static_cast<cudaStream_t>(stream));
      if (e != cudaSuccess) return cuda_fail(e, "build_centroids launch");
    }
    return ok();
  }
  p.sel = sel;
  p.n_sel = n_sel;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.approx = approx ? 1 : 0;
  p.seed = seed;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (n_fill > 0 && !(mode == kFused && use_persistent(sh, a))) {
    // no persistent launch to fold the build into: it runs first, as its own launch
    cudaError_t e = launch_build_centroids(*kv, fill_pages, n_fill, cent_out, a->status, st);
    if (e != cudaSuccess) return cuda_fail(e, "build_centroids launch");
    n_fill = 0;
  }
  p.fill_pages = fill_pages;
  p.n_fill = n_fill;
  p.cent_out = cent_out;
  // the select-only and decode-only calls given a workspace run as modes of the persistent
  // kernels
  const bool persistent = use_persistent(sh, a) && (mode == kFused || (split_on_persistent && ws));
  if (persistent) {
    const size_t need = persist_bytes(sh, p, unit_cap);
    if (!ws || ws_bytes < need)
      return fail(VT_ERR_INVALID_ARG, "workspace of %zu bytes needed, %zu given", need,
                  ws ? ws_bytes : (size_t)0);
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
      return fail(VT_ERR_INVALID_ARG, "workspace not 256-byte aligned");
    const int bytes = sh.path == kPathMla ? mla_persist_smem_bytes(p, sh.G)
                                          : persist_smem_bytes(p, sh.D, sh.G);
    if (bytes > 227 * 1024) return fail(VT_ERR_UNSUPPORTED, "shared memory need %d B too large", bytes);
    cudaError_t e = sh.path == kPathMla
                        ? launch_mla_persist(p, sh.G, ws, unit_cap, sm_count(), st, mode)
                        : launch_persist_fused(p, sh.D, sh.G, ws, unit_cap, sm_count(), st, mode);
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return ok();
  }
  const int64_t units = (int64_t)a->batch * kv->num_kv_heads;
  const int C = pick_cluster(sh, units, p.kmax);
  const int max_cand = (int)std::max<int64_t>(1, a->pt_stride - a->bos - a->eos);
  p.key_cap = max_cand;
  p.cand_cap = (max_cand + C - 1) / C;
  cudaError_t e;
  if (sh.path == kPathGqa) {
    const int bytes = gqa_smem_bytes(sh.D, sh.G, p.cand_cap, p.key_cap, p.kmax);
    if (bytes > 227 * 1024) return fail(VT_ERR_UNSUPPORTED, "shared memory need %d B too large", bytes);
    e = launch_gqa_decode(p, mode, sh.D, sh.G, C, st);
  } else {
    const int ppc = (p.kmax + C - 1) / C;
    if (ppc > mla_max_pages_per_cta())
      return fail(VT_ERR_UNSUPPORTED, "topk+bos+eos %d too large for the MLA kernel", p.kmax);
    const int bytes = mla_smem_bytes(sh.G, p.cand_cap, p.key_cap, p.kmax, ppc);
    if (bytes > 227 * 1024) return fail(VT_ERR_UNSUPPORTED, "shared memory need %d B too large", bytes);
    e = launch_mla_decode(p, mode, sh.G, C, st);
  }
  if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
  return ok();
}

// ---- the library-owned scratch of vt_sparse_decode_fused_static ----------------------------

// One per device the module is loaded on, zero-filled by CUDA at load.  The persistent
// kernel leaves its counters at zero after every complete call, so it is never cleared here.
static __device__ __align__(256) unsigned char g_static_scratch[VT_STATIC_SCRATCH_BYTES];
// Its per-unit counters are laid out for this many units whatever the call's shape, so they
// sit at the same offsets in every call and never overlap another call's data.
constexpr int64_t kStaticUnitCap = 65536;

// Device address of g_static_scratch in the current device's current context.  In host code
// the array's name only stands in for it, so it is looked up, and it is looked up on every
// call rather than cached: a context that is destroyed and created again (cudaDeviceReset)
// reloads the module, and the array may then sit at another address.
cudaError_t static_scratch_address(void** addr) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
  if (e != cudaSuccess) return e;
  *addr = p;
  return cudaSuccess;
}

}  // namespace

extern "C" {

vt_status vt_build_centroids(const vt_paged_kv* kv, const int32_t* pages, int32_t n_pages,
                             float* centroids, int32_t* status, void* stream) {
  vt_status s = check_kv(kv);
  if (s != VT_OK) return s;
  if (n_pages < 0) return fail(VT_ERR_INVALID_ARG, "n_pages < 0");
  if (n_pages == 0) return ok();
  if (!pages || !centroids) return fail(VT_ERR_INVALID_ARG, "pages/centroids is NULL");
  if (kv->head_dim % 8 != 0) return fail(VT_ERR_UNSUPPORTED, "head_dim must be a multiple of 8");
  if (!aligned16(centroids)) return fail(VT_ERR_UNSUPPORTED, "centroids not 16-byte aligned");
  if ((int64_t)n_pages * kv->num_kv_heads * (kv->head_dim / 8) > (int64_t)UINT32_MAX * 256)
    return fail(VT_ERR_UNSUPPORTED, "too many pages in one call");
  cudaError_t e = launch_build_centroids(*kv, pages, n_pages, centroids, status,
                                         static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "build_centroids launch");
  return ok();
}

vt_status vt_select_pages(const vt_paged_kv* kv, const vt_decode_args* a, int32_t* sel,
                          int32_t* n_sel, void* stream) {
  return launch_query_side(kv, a, kSelect, sel, n_sel, nullptr, nullptr, nullptr, 0, stream);
}

vt_status vt_select_pages_ws(const vt_paged_kv* kv, const vt_decode_args* a, int32_t* sel,
                             int32_t* n_sel, void* workspace, size_t workspace_bytes,
                             void* stream) {
  return launch_query_side(kv, a, kSelect, sel, n_sel, nullptr, nullptr, workspace,
                           workspace_bytes, stream, 0, false, 0, nullptr, 0, nullptr, true);
}

vt_status vt_sparse_decode_ws(const vt_paged_kv* kv, const vt_decode_args* a, const int32_t* sel,
                              const int32_t* n_sel, void* out, float* lse, void* workspace,
                              size_t workspace_bytes, void* stream) {
  return launch_query_side(kv, a, kDecode, const_cast<int32_t*>(sel), const_cast<int32_t*>(n_sel),
                           out, lse, workspace, workspace_bytes, stream, 0, false, 0, nullptr, 0,
                           nullptr, true);
}

vt_status vt_select_pages_approx(const vt_paged_kv* kv, const vt_decode_args* a, uint64_t seed,
                                 int32_t* sel, int32_t* n_sel, void* stream) {
  return launch_query_side(kv, a, kSelect, sel, n_sel, nullptr, nullptr, nullptr, 0, stream, 0,
                           true, seed);
}

vt_status vt_sparse_decode(const vt_paged_kv* kv, const vt_decode_args* a, const int32_t* sel,
                           const int32_t* n_sel, void* out, float* lse, void* stream) {
  return launch_query_side(kv, a, kDecode, const_cast<int32_t*>(sel),
                           const_cast<int32_t*>(n_sel), out, lse, nullptr, 0, stream);
}

vt_status vt_sparse_decode_fused(const vt_paged_kv* kv, const vt_decode_args* a, void* out,
                                 float* lse, int32_t* sel, int32_t* n_sel, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  return launch_query_side(kv, a, kFused, sel, n_sel, out, lse, workspace, workspace_bytes,
                           stream);
}

size_t vt_fused_workspace_size(const vt_paged_kv* kv, const vt_decode_args* a) {
  Shape sh;
  DecodeParams p;
  if (fill_params(kv, a, false, &sh, &p) != VT_OK) return 0;  // (centroids are not needed)
  if (!use_persistent(sh, a)) return 0;
  return persist_bytes(sh, p, 0);
}

vt_status vt_sparse_decode_fused_static(const vt_paged_kv* kv, const vt_decode_args* a,
                                        void* out, float* lse, int32_t* sel, int32_t* n_sel,
                                        void* stream) {
  // 0 for arguments the fused call rejects (it then reports why) and for shapes that need
  // no workspace
  size_t need = 0;
  {
    Shape sh;
    DecodeParams p;
    if (fill_params(kv, a, true, &sh, &p) == VT_OK && use_persistent(sh, a)) {
      if ((int64_t)a->batch * kv->num_kv_heads > kStaticUnitCap)
        return fail(VT_ERR_UNSUPPORTED, "B * Hkv > %lld units for the static scratch",
                    (long long)kStaticUnitCap);
      need = persist_bytes(sh, p, kStaticUnitCap);
    }
  }
  if (need > (size_t)VT_STATIC_SCRATCH_BYTES)
    return fail(VT_ERR_UNSUPPORTED, "needs %zu bytes of scratch; the static scratch holds %zu",
                need, (size_t)VT_STATIC_SCRATCH_BYTES);
  void* ws = nullptr;
  size_t ws_bytes = 0;
  if (need > 0) {
    // the call-level checks of the fused call, before any CUDA call
    if (!out) return fail(VT_ERR_INVALID_ARG, "out is NULL");
    if ((sel == nullptr) != (n_sel == nullptr))
      return fail(VT_ERR_INVALID_ARG, "sel and n_sel must both be given or both be NULL");
    cudaError_t e = static_scratch_address(&ws);
    if (e != cudaSuccess) return cuda_fail(e, "static scratch address");
    ws_bytes = VT_STATIC_SCRATCH_BYTES;
  }
  return launch_query_side(kv, a, kFused, sel, n_sel, out, lse, ws, ws_bytes, stream,
                           kStaticUnitCap);
}

vt_status vt_sparse_decode_step(const vt_paged_kv* kv, const vt_decode_args* a,
                                const int32_t* fill_pages, int32_t n_fill, float* centroids,
                                void* out, float* lse, int32_t* sel, int32_t* n_sel,
                                void* workspace, size_t workspace_bytes, void* stream) {
  if (n_fill < 0) return fail(VT_ERR_INVALID_ARG, "n_fill < 0");
  if (n_fill > 0) {
    if (!fill_pages || !centroids) return fail(VT_ERR_INVALID_ARG, "fill_pages/centroids is NULL");
    if (!a || centroids != a->centroids)
      return fail(VT_ERR_INVALID_ARG, "centroids must be the cache args->centroids points to");
    if (a->eos < 1)
      return fail(VT_ERR_UNSUPPORTED,
                  "filled pages are built beside the scans: needs eos >= 1 (the last page is "
                  "then never scored)");
  }
  return launch_query_side(kv, a, kFused, sel, n_sel, out, lse, workspace, workspace_bytes,
                           stream, 0, false, 0, fill_pages, n_fill, centroids);
}

vt_status vt_plan_requests(const int32_t* seq_lens, int32_t batch, int32_t* order, void* stream) {
  if (batch < 0) return fail(VT_ERR_INVALID_ARG, "batch < 0");
  if (batch == 0) return ok();
  if (!seq_lens || !order) return fail(VT_ERR_INVALID_ARG, "seq_lens/order is NULL");
  if (batch > 65536) return fail(VT_ERR_UNSUPPORTED, "batch > 65536");
  cudaError_t e = launch_plan(seq_lens, batch, order, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "plan launch");
  return ok();
}

const char* vt_status_string(vt_status s) {
  switch (s) {
    case VT_OK: return "VT_OK";
    case VT_ERR_INVALID_ARG: return "VT_ERR_INVALID_ARG";
    case VT_ERR_UNSUPPORTED: return "VT_ERR_UNSUPPORTED";
    case VT_ERR_CUDA: return "VT_ERR_CUDA";
  }
  return "VT_ERR_UNKNOWN";
}

const char* vt_last_error_detail(void) { return g_detail; }

int32_t vt_abi_version(void) { return VT_ABI_VERSION; }

}  // extern "C"
