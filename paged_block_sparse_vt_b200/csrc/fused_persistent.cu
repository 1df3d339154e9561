// fused_persistent.cu -- the whole query side of block top-k sparse decode for GQA heads in one
// launch of persistent CTAs that pull small work items from a queue, so that a batch of
// requests with very different lengths keeps every SM busy until the end.
//
// Sources: "Vortex: A Flexible and Efficient Sparse Attention Framework" (vortex_torch
// README), "Quick Example" (forward_indexer: q.mean -> GeMV against the centroids -> topK)
// and "Using Your Sparse Attention with SGLang" (page size 16, vortex_topk_val, reserved
// bos/eos pages); "Vortex: Efficient and Programmable Sparse Attention Serving for AI Agents",
// "A dual-stage programmable abstraction" (a workload planner for balanced GPU scheduling
// and kernel fusion); the thread on digg.com, closing reply (batch heterogeneity is where
// sparse-attention speedups are lost).
//
// Work items, claimed in order through one global counter (a CTA claims its next item when
// the streaming part of the current one is ending, so the counter's latency is hidden by the
// current item's tail and the queue order still follows the CTAs' actual progress):
//   scan items   -- (request, KV head, chunk of kChunk candidate pages), in request order,
//                   each unit's chunks consecutive.  Every warp streams its rows of the
//                   chunk's fp32 centroids through a cp.async ring and dots them with the
//                   fp32 mean of the unit's G query heads; the CTA then takes the exact top-k
//                   of the chunk in shared memory and stores those candidates (ordered
//                   score key and offset, ascending by page) before counting the chunk done.
//                   When the next item is a scan item too, its page ids and query rows load
//                   while that top-k runs, and its first batches go out right after it
//                   (issuing them before the top-k measured slower).
//                   The union of the chunks' top-k holds the unit's top-k: a key outside its
//                   chunk's top-k has k keys above it in that chunk alone;
//   attention    -- (unit, piece of at most kPiecePages selected pages), after every scan item.  The
//   items           CTA waits until all of the unit's chunks are counted (every chunk was
//                   claimed before this item and scan items never wait, so the wait ends),
//                   merges the candidates with the same exact top-k, attends the pages of its
//                   piece on the tensor cores (eight per warp through a kAttSlots-slot ring) and
//                   stores a partial (max, sum, acc); the piece that is counted last for
//                   its unit merges the partials and writes the bf16 output and the lse.
// The schedule (scan items per request and their prefix) is computed by every CTA from the
// sequence lengths at start, so the call is one launch.  The per-unit counters are reset by
// the CTA that last uses them and the claim counter runs on across launches (each launch
// numbers its items from where the previous one stopped), so the workspace needs
// zero-filling only once and no CTA waits for the others on its way out.
#include "centroid_chunk.cuh"
#include "decode_params.cuh"
#include "gqa_attend.cuh"
#include "topk.cuh"

namespace vt {

constexpr int kPersistThreads = 128;
constexpr int kPersistWarps = kPersistThreads / 32;
constexpr int kChunk = 256;      // candidate pages per scan item (64 per warp)
constexpr int kScanRing = 4;     // 8-row centroid batches per warp ring (3 landing)
constexpr int kPiecePages = 32;  // most selected pages per attention item (8 per warp)
constexpr int kTailPiecePages = 16;  // the same for the units attended last
constexpr int kAttSlots = 2;     // page slots per warp's attention ring (kAttSlots - 1 landing)
constexpr int kMaxPlanB = 2048;  // requests the persistent path takes (schedule kept in smem)
constexpr int kPersistMinCtas = 3;  // CTAs per SM the registers must allow (<= 168 per thread)

// ---- sizes derived from the call ----------------------------------------------------------

struct PersistGeom {
  int max_cand;  // middle (candidate) pages of a full page-table row, >= 1
  int nch_max;   // chunks of such a row
  int kc;        // candidates a chunk keeps: min(topk, kChunk)
  int A;         // attention pieces of each unit attended before the last ones
  int pp;        // their selected pages per piece: kmax split evenly, at most kPiecePages
  int A2, pp2;   // the same for the units attended last (at most kTailPiecePages): their
                 // attention runs at the end of the launch, where more, shorter items keep
                 // more CTAs busy
  int cmax;      // candidates one unit merges at most
};

__host__ __device__ inline PersistGeom persist_geom(int64_t pt_stride, int topk, int bos, int eos,
                                                    int kmax) {
  PersistGeom g;
  const int64_t mc = pt_stride - bos - eos;
  g.max_cand = mc > 1 ? (int)mc : 1;
  g.nch_max = (g.max_cand + kChunk - 1) / kChunk;
  g.kc = topk < kChunk ? (topk > 0 ? topk : 1) : kChunk;
  g.A = (kmax + kPiecePages - 1) / kPiecePages;
  g.pp = (kmax + g.A - 1) / g.A;
  g.A2 = (kmax + kTailPiecePages - 1) / kTailPiecePages;
  g.pp2 = (kmax + g.A2 - 1) / g.A2;
  const int64_t c = (int64_t)g.nch_max * g.kc;
  g.cmax = c < g.max_cand ? (int)c : g.max_cand;
  return g;
}

// Scan items of one request per KV head: none when nothing is ranked (invalid length, a
// dense request, or topk == 0), otherwise one per chunk of the candidate pages.
__host__ __device__ inline int chunks_of(int L, int64_t pt_stride, int topk, int bos, int eos,
                                         int kmax) {
  const int n = (L + kPage - 1) / kPage;
  if (L < 1 || n > pt_stride || n <= kmax || topk < 1) return 0;
  return (n - bos - eos + kChunk - 1) / kChunk;
}

// ---- workspace ----------------------------------------------------------------------------

struct PersistWs {
  uint32_t* ctr;       // [2]: claims ever made (mod 2^32), the claim count when this launch began
  int32_t* unit_done;  // [U]: chunks of the unit whose candidates are stored
  int32_t* att_cnt;    // [U]: attention pieces of the unit done
  uint32_t* ckey;      // [U][nch_max][kc]: ordered score keys of each chunk's top-k
  uint16_t* coff;      // [U][nch_max][kc]: their offsets in the chunk, ascending
  int32_t* cpid;       // [U][nch_max][kc]: their page ids (-1 where the id was out of range)
  float* part;         // [U][A2][G][Dv+2]: attention partials
  PersistGeom g;
  int mode;            // kFused, kSelect (scan items only) or kDecode (attention items only)
  int units;
};

struct PersistWsLayout {
  size_t ctr, unit_done, att_cnt, ckey, coff, cpid, part, total;
};

static inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// unit_cap >= B * Hkv: units the counter arrays are laid out for.  The counters are the only
// part that must be zero before a call; with a fixed unit_cap they sit at the same offsets for
// every shape, so calls of different shapes can share one buffer.
static PersistWsLayout persist_ws_layout(const DecodeParams& p, int G, int Dv, int64_t unit_cap) {
  const PersistGeom g = persist_geom(p.pt_stride, p.topk, p.bos, p.eos, p.kmax);
  const size_t U = (size_t)p.B * p.Hkv;
  const size_t cap = unit_cap > (int64_t)U ? (size_t)unit_cap : U;
  const size_t cand = U * g.nch_max * g.kc;
  PersistWsLayout L;
  size_t o = 0;
  L.ctr = o;       o += align256(2 * sizeof(uint32_t));
  L.unit_done = o; o += align256(cap * sizeof(int32_t));
  L.att_cnt = o;   o += align256(cap * sizeof(int32_t));
  L.ckey = o;      o += align256(cand * sizeof(uint32_t));
  L.coff = o;      o += align256(cand * sizeof(uint16_t));
  L.cpid = o;      o += align256(cand * sizeof(int32_t));
  L.part = o;      o += align256(U * g.A2 * G * (Dv + 2) * sizeof(float));
  L.total = o;
  return L;
}

// ---- memory-order helpers (gpu scope) --------------------------------------------------

__device__ __forceinline__ void red_release_add(int32_t* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;\n" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ int atom_acq_rel_add(int32_t* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;\n" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ int ld_acquire(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Page id of row i (any lane-dependent i < 64) from ids held as (row l, row l + 32) by lane l.
__device__ __forceinline__ int page_of_lane(int pidA, int pidB, int i) {
  const int a = __shfl_sync(kFull, pidA, i & 31);
  const int b = __shfl_sync(kFull, pidB, i & 31);
  return i < 32 ? a : b;
}

// ---- the persistent kernel ---------------------------------------------------------------

template <int D>
struct PersistShape : PageTile<D> {
  static constexpr int C_ROW = D * 4;  // fp32 centroid row
};

struct PersistSmem {
  int prefix, keys, pids, sel, phys, misc, region, total;
};

__host__ __device__ inline PersistSmem persist_smem_layout(int D, int G, int B,
                                                           const PersistGeom& g) {
  PersistSmem s;
  int o = 0;
  s.prefix = o; o += align16((B + 1) * 4);
  s.keys = o;   o += align16(kChunk * 4);
  s.pids = o;   o += align16(kChunk * 4);
  s.sel = o;    o += align16(kPiecePages * 4);
  s.phys = o;   o += align16(kPiecePages * 4);
  s.misc = o;   o += align16(64 * 4);
  o = (o + 127) & ~127;
  s.region = o;  // one of: scan rings | top-k scratch | page rings | attention partials
  // scan rings, plus the chunk top-k scratch where it does not fit in one ring slot
  const int scan = kPersistWarps * kScanRing * 8 * D * 4 +
                   (8 * D * 4 >= SmallTopk<kPersistThreads>::BYTES ? 0 : SmallTopk<kPersistThreads>::BYTES);
  const int att = kPersistWarps * kAttSlots * 2 * kPage * (D + 8) * 2;
  // merge of up to 2 NT candidates: keys, logical and physical pages, small_topk scratch;
  // of more: keys, offsets, block_topk scratch
  const int merge_small = 3 * 2 * kPersistThreads * 4 + SmallTopk<kPersistThreads>::BYTES;
  const int merge_big = align16(g.cmax * 4) + align16(g.cmax * 2) + align16((kTopkBins + 64) * 4);
  const int merge = merge_small > merge_big ? merge_small : merge_big;
  const int comb = align16(kPersistWarps * G * (D + 2) * 4) + align16(G * (D + 2) * 4) +
                   align16(g.A2 * G * (D + 2) * 4);
  int r = scan;
  if (att > r) r = att;
  if (merge > r) r = merge;
  if (comb > r) r = comb;
  s.total = o + r;
  return s;
}

template <int D, int G>
__global__ void __launch_bounds__(kPersistThreads, kPersistMinCtas) persist_fused_kernel(const DecodeParams p,
                                                                        const PersistWs w) {
  using S = PersistShape<D>;
  constexpr int NT = kPersistThreads;
  constexpr int NW = kPersistWarps;
  constexpr int LPR_S = D / 4;     // lanes per centroid row
  constexpr int RPS = 32 / LPR_S;  // centroid rows per warp step
  constexpr int SN = 8 / RPS;      // values per lane per batch of 8 rows
  static_assert(D == 64 || D == 128, "GQA path covers head_dim 64 and 128");
  static_assert(kPiecePages <= kPersistThreads, "one thread per page of a piece");

  extern __shared__ __align__(128) unsigned char smem[];
  const PersistGeom gm = w.g;
  const PersistSmem Ls = persist_smem_layout(D, G, p.B, gm);
  int* s_prefix = reinterpret_cast<int*>(smem + Ls.prefix);
  uint32_t* s_keys = reinterpret_cast<uint32_t*>(smem + Ls.keys);
  int* s_pids = reinterpret_cast<int*>(smem + Ls.pids);  // page ids of the chunk's rows
  int* s_sel = reinterpret_cast<int*>(smem + Ls.sel);
  int* s_phys = reinterpret_cast<int*>(smem + Ls.phys);
  int* s_misc = reinterpret_cast<int*>(smem + Ls.misc);  // [0] item, [1] flag, [8..] scan
  unsigned char* region = smem + Ls.region;
  const uint32_t region_u32 = smem_u32(region);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // Launched as a programmatic dependent of the previous kernel on the stream: the CTAs may
  // be placed while that kernel still runs, and nothing in global memory is touched before it
  // has completed.  The next such launch may likewise be placed early.
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

  uint32_t qbase = 0;  // thread 0: the claim count when this launch began
  // items are numbered from -n_fill: the build items of the pages filled at this step first
  auto claim = [&]() { return (int)(atomicAdd(w.ctr + 0, 1u) - qbase) - p.n_fill; };

  // ---- schedule: exclusive prefix of scan items over the requests, in request order
  {
    // the first item, claimed now so that the claim overlaps the prefix.  Items are numbered
    // from the claim count at which this launch began (qbase), so the counter is never reset:
    // the launch's last claim stores the next launch's qbase.
    int first = 0;
    if (tid == 0) {
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];\n" : "=r"(qbase) : "l"(w.ctr + 1) : "memory");
      first = claim();
    }
    const int per = (p.B + NT - 1) / NT;
    const int i0 = min(p.B, tid * per), i1 = min(p.B, i0 + per);
    int run = 0;
    for (int i = i0; i < i1; ++i) {
      const int c = p.Hkv * chunks_of(p.seq_lens[i], p.pt_stride, p.topk, p.bos, p.eos, p.kmax);
      s_prefix[i] = c;
      run += c;
    }
    int x = run;
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) s_misc[8 + warp] = x;
    __syncthreads();
    int base = 0;
    for (int k = 0; k < warp; ++k) base += s_misc[8 + k];
    int acc = base + x - run;
    for (int i = i0; i < i1; ++i) {
      const int c = s_prefix[i];
      s_prefix[i] = acc;
      acc += c;
    }
    if (tid == NT - 1) s_prefix[p.B] = base + x;
    if (tid == 0) s_misc[0] = first;
    __syncthreads();
  }
  const int scan_items = w.mode == kDecode ? 0 : s_prefix[p.B];
  // Units from u_split on take gm.A2 (shorter) pieces: only the attention that runs at the
  // end of the launch, where shorter items keep more CTAs busy, is split.  Measured: splitting
  // the last gridDim.x / 4 units (at least half of them) against the last half of the units:
  // 35.8 us both at the Qwen3-0.6B-like layer (256 units), 342 -> 324 us at 32K contexts
  // (1024 units), 260 -> 237 us on the heterogeneous batch (16384 units).
  const int u_split = max(w.units / 2, w.units - (int)gridDim.x / 4);
  const int total_items =
      scan_items + (w.mode == kSelect ? 0 : u_split * gm.A + (w.units - u_split) * gm.A2);
  if (w.mode == kSelect) {
    // the units that rank nothing (dense, reserved only, or invalid): their selection here
    for (int u = blockIdx.x; u < w.units; u += gridDim.x) {
      const int b = u / p.Hkv;
      const int L = p.seq_lens[b];
      if (chunks_of(L, p.pt_stride, p.topk, p.bos, p.eos, p.kmax) > 0) continue;
      const int n = (L + kPage - 1) / kPage;
      const bool valid = L >= 1 && n <= p.pt_stride;
      const int ns = !valid ? 0 : (n <= p.kmax ? n : p.kmax);
      const bool resv = valid && n > p.kmax;
      for (int j = tid; j < p.kmax; j += NT)
        p.sel[(int64_t)u * p.kmax + j] =
            j >= ns ? -1 : ((!resv || j < p.bos) ? j : n - p.eos + (j - p.bos));
      if (tid == 0) {
        p.n_sel[u] = ns;
        if (!valid && u % p.Hkv == 0) flag(p.status, VT_DEV_BAD_LEN);
      }
    }
  }

  // ---- scan items: where an item's rows lie, and its per-lane state.  A scan item whose
  // predecessor was a scan item finds its page ids and query mean already in registers and
  // its first kScanRing - 1 batches in flight (prepared during the predecessor's top-k).
  struct ScanItem {
    int b, h, c, u, cnt, c0, myrows, batches, nch;
  };
  auto scan_item = [&](int t) {
    ScanItem it;
    int lo = 0, hi = p.B - 1;  // largest k with prefix[k] <= t: a request with items
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_prefix[mid] <= t) lo = mid; else hi = mid - 1;
    }
    it.b = lo;
    const int r = t - s_prefix[it.b];
    const int n = (p.seq_lens[it.b] + kPage - 1) / kPage;
    const int m = n - p.bos - p.eos;
    const int nch = (m + kChunk - 1) / kChunk;
    it.nch = nch;
    it.h = r / nch;
    it.c = r - it.h * nch;
    it.u = it.b * p.Hkv + it.h;
    it.c0 = it.c * kChunk;
    it.cnt = min(kChunk, m - it.c0);
    // warp w: rows w + NW i, i < 64 of the chunk, streamed in batches of 8
    it.myrows = (it.cnt - warp + NW - 1) / NW;
    it.batches = (it.myrows + 7) / 8;
    return it;
  };
  const int sub = lane / LPR_S, ch = lane % LPR_S;
  bool prepared = false;
  int pidA = -1, pidB = -1;  // lane l: page ids of its warp's rows l and l + 32
  float4 qv = make_float4(0.f, 0.f, 0.f, 0.f);  // fp32 group mean of q, this lane's float4
  // The query rows are loaded ahead with the page ids only for small groups (registers).
  constexpr bool kQAhead = G <= 2;
  uint2 qraw[G];  // this lane's 4 query values of each head of the group, as loaded
  auto load_q = [&](const ScanItem& it) {
    const __nv_bfloat16* q0 = p.q + ((int64_t)it.b * p.Hq + (int64_t)it.h * G) * D + ch * 4;
#pragma unroll
    for (int j = 0; j < G; ++j) qraw[j] = *reinterpret_cast<const uint2*>(q0 + (int64_t)j * D);
  };
  // loads of an item's page ids (and query rows), not yet used, so that they may be in
  // flight while other work proceeds ...
  auto scan_load = [&](const ScanItem& it) {
    const int32_t* ptrow = p.page_table + (int64_t)it.b * p.pt_stride + p.bos + it.c0 + warp;
    pidA = lane < it.myrows ? ptrow[NW * lane] : -1;
    pidB = lane + 32 < it.myrows ? ptrow[NW * (lane + 32)] : -1;
    if (kQAhead) load_q(it);
  };
  // ... and their use: the fp32 group mean, and the page ids checked
  auto scan_check = [&](const ScanItem& it) {
    if (!kQAhead) load_q(it);
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < G; ++j) {
      a.x += bf_lo(qraw[j].x);
      a.y += bf_hi(qraw[j].x);
      a.z += bf_lo(qraw[j].y);
      a.w += bf_hi(qraw[j].y);
    }
    qv = make_float4(a.x / (float)G, a.y / (float)G, a.z / (float)G, a.w / (float)G);
    if (pidA >= p.num_pages || pidA < -1 || pidB >= p.num_pages || pidB < -1 ||
        (lane < it.myrows && pidA < 0) || (lane + 32 < it.myrows && pidB < 0)) {
      flag(p.status, VT_DEV_BAD_PAGE);
      if (pidA < 0 || pidA >= p.num_pages) pidA = -1;
      if (pidB < 0 || pidB >= p.num_pages) pidB = -1;
    }
  };
  constexpr int CPRS = S::C_ROW / 16;  // 16-byte chunks per centroid row
  const int64_t cstride = (int64_t)p.Hkv * D;
  auto scan_issue = [&](const ScanItem& it, int bt) {
    if (bt < it.batches) {
      const uint32_t dst = region_u32 + (warp * kScanRing + bt % kScanRing) * 8 * S::C_ROW;
      const float* cbase = p.centroids + (int64_t)it.h * D;
#pragma unroll
      for (int t8 = 0; t8 < 8; ++t8) {
        const int i = bt * 8 + t8;  // uniform, < 64
        const int pg = __shfl_sync(kFull, i < 32 ? pidA : pidB, i & 31);
#pragma unroll
        for (int kk = lane; kk < CPRS; kk += 32)
          if (pg >= 0)
            cp_async16(dst + t8 * S::C_ROW + kk * 16, cbase + (int64_t)pg * cstride + kk * 4, 16);
      }
    }
    cp_async_commit();
  };
  // ---- select-only launches: the unit's selection, taken by the CTA whose chunk was counted
  // last for the unit: the exact top-k of the chunks' candidates (the union of the chunks'
  // top-k holds the unit's top-k) plus the reserved pages, written to sel / n_sel in ascending
  // logical order.
  auto merge_unit = [&](int b, int u, int nch) {
    const int n = (p.seq_lens[b] + kPage - 1) / kPage;
    const int m = n - p.bos - p.eos;
    const int kc = gm.kc;
    const int C = (nch - 1) * kc + min(kc, m - (nch - 1) * kChunk);
    const int64_t cb = (int64_t)u * gm.nch_max * kc;  // chunks are contiguous
    const int bos = p.bos, topk = p.topk;
    const int32_t* ptrow = p.page_table + (int64_t)b * p.pt_stride;
    int32_t* selrow = p.sel + (int64_t)u * p.kmax;
    if (tid == 0) p.n_sel[u] = p.kmax;
    auto checked = [&](int pg) {
      if (pg < 0 || pg >= p.num_pages) flag(p.status, VT_DEV_BAD_PAGE);
    };
    // the reserved pages (their page-id loads in flight with the candidates' loads)
    const int nres = bos + p.eos;
    int rlp = -1, rpg = -1;
    if (tid < nres) {
      rlp = tid < bos ? tid : n - p.eos + (tid - bos);
      rpg = ptrow[rlp];
    }
    // candidate j of chunk j / kc sits at offset coff[j] of it; candidates are in ascending
    // page order, so ties (lowest position) go to the lowest page
    if (C <= 2 * NT) {
      uint32_t* keys = reinterpret_cast<uint32_t*>(region);
      int* lps = reinterpret_cast<int*>(region + 2 * NT * 4);
      int* pids = reinterpret_cast<int*>(region + 4 * NT * 4);
      unsigned char* tkm = region + 6 * NT * 4;
      for (int i = tid; i < SmallTopk<NT>::HIST / 4; i += NT)
        reinterpret_cast<int4*>(tkm)[i] = make_int4(0, 0, 0, 0);
      const bool h0 = tid < C, h1 = tid + NT < C;
      uint32_t key0 = 0, key1 = 0;
      int off0 = 0, off1 = 0, pid0 = -1, pid1 = -1;
      if (h0) {
        key0 = __ldcg(w.ckey + cb + tid);
        off0 = __ldcg(w.coff + cb + tid);
        pid0 = __ldcg(w.cpid + cb + tid);
      }
      if (h1) {
        key1 = __ldcg(w.ckey + cb + tid + NT);
        off1 = __ldcg(w.coff + cb + tid + NT);
        pid1 = __ldcg(w.cpid + cb + tid + NT);
      }
      uint32_t klo = 0xffffffffu, khi = 0u;
      if (h0) {
        keys[tid] = key0;
        lps[tid] = bos + (tid / kc) * kChunk + off0;
        pids[tid] = pid0;
        klo = key0;
        khi = key0;
      }
      if (h1) {
        const int j = tid + NT;
        keys[j] = key1;
        lps[j] = bos + (j / kc) * kChunk + off1;
        pids[j] = pid1;
        klo = min(klo, key1);
        khi = max(khi, key1);
      }
      klo = __reduce_min_sync(kFull, klo);
      khi = __reduce_max_sync(kFull, khi);
      if (lane == 0) {
        s_misc[16 + warp] = (int)klo;
        s_misc[16 + NW + warp] = (int)khi;
      }
      __syncthreads();
#pragma unroll
      for (int k = 0; k < NW; ++k) {
        klo = min(klo, (uint32_t)s_misc[16 + k]);
        khi = max(khi, (uint32_t)s_misc[16 + NW + k]);
      }
      small_topk<NT>(keys, C, topk, klo, khi, tkm, [&](int j, int pos) {
        selrow[bos + pos] = lps[j];
      });
    } else {
      uint32_t* keys = reinterpret_cast<uint32_t*>(region);
      uint16_t* offs = reinterpret_cast<uint16_t*>(region + align16(gm.cmax * 4));
      int* hist = reinterpret_cast<int*>(region + align16(gm.cmax * 4) + align16(gm.cmax * 2));
      for (int j = tid; j < C; j += NT) {
        keys[j] = __ldcg(w.ckey + cb + j);
        offs[j] = __ldcg(w.coff + cb + j);
      }
      __syncthreads();
      block_topk<NT>(keys, C, topk, hist, hist + kTopkBins, [&](int j, int pos) {
        selrow[bos + pos] = bos + (j / kc) * kChunk + offs[j];
      });
    }
    if (tid < nres) {
      const int pos = tid < bos ? tid : bos + topk + (tid - bos);
      checked(rpg);
      selrow[pos] = rlp;
    }
    __syncthreads();
    if (tid == 0) w.unit_done[u] = 0;  // every chunk of u is counted: the counter is free again
  };
  // scratch of a chunk's top-k: warp 0's last ring slot where it is large enough (the next
  // item's first batches fill the other slots meanwhile), else past the rings
  unsigned char* tk = region + (8 * S::C_ROW >= SmallTopk<NT>::BYTES
                                    ? (kScanRing - 1) * 8 * S::C_ROW
                                    : NW * kScanRing * 8 * S::C_ROW);
  for (;;) {
    const int t = s_misc[0];
    __syncthreads();  // every thread has read the item before the next claim is stored
    if (t >= total_items) {
      // Every CTA makes one claim per item plus one that ends it, so the launch's claims are
      // numbered -n_fill .. total_items + gridDim.x - 1.  The CTA holding the last one knows
      // that every CTA has read qbase, and sets it for the next launch.
      if (tid == 0 && t == total_items + (int)gridDim.x - 1)
        w.ctr[1] = qbase + (uint32_t)(p.n_fill + total_items) + gridDim.x;
      break;
    }
    // the next item, claimed by thread 0 once this item's streaming is done (or at its end)
    int next = -1;

    if (t < 0) {
      // ---------------------------------------------------------------- build item
      // the centroids of one page filled at this step (every KV head), which no score of
      // this step reads: the page is its request's reserved last page
      const int64_t pg = p.fill_pages[t + p.n_fill];
      if (pg < 0 || pg >= p.num_pages) {
        if (tid == 0) flag(p.status, VT_DEV_BAD_PAGE);
      } else {
        for (int idx = tid; idx < p.Hkv * (D / 8); idx += NT)
          build_centroid_chunk(p.k_pool, pg, idx / (D / 8), idx % (D / 8), p.sk_p, p.sk_t,
                               p.sk_h, p.Hkv, D, p.cent_out);
      }
      if (tid == 0) next = claim();
    } else if (t < scan_items) {
      // ---------------------------------------------------------------- scan item
      const ScanItem it = scan_item(t);
      if (!prepared) {
        scan_load(it);
        scan_check(it);
#pragma unroll
        for (int bt = 0; bt < kScanRing - 1; ++bt) scan_issue(it, bt);
      }
      // the rows' page ids for the top-k's emit (the previous item's top-k has passed its
      // closing barrier)
      if (lane < it.myrows) s_pids[warp + NW * lane] = pidA;
      if (lane + 32 < it.myrows) s_pids[warp + NW * (lane + 32)] = pidB;
      const uint32_t ring = region_u32 + warp * kScanRing * 8 * S::C_ROW;
      uint32_t klo = 0xffffffffu, khi = 0u;  // range of the keys this lane stores
      for (int bt = 0; bt < it.batches; ++bt) {
        scan_issue(it, bt + kScanRing - 1);
        // the next item is claimed as warp 0's last batch lands (warp 0 has the most rows),
        // so that the claim's latency hides under it
        if (tid == 0 && bt == it.batches - 1) next = claim();
        cp_async_wait<kScanRing - 1>();
        __syncwarp();
        const uint32_t src = ring + (bt % kScanRing) * 8 * S::C_ROW;
        float v[SN];
#pragma unroll
        for (int qq = 0; qq < SN; ++qq) {
          const int tt = qq * RPS + sub;  // row of the batch
          float4 cv;
          asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];\n"
                       : "=f"(cv.x), "=f"(cv.y), "=f"(cv.z), "=f"(cv.w)
                       : "r"(src + tt * S::C_ROW + ch * 16));
          float d = cv.x * qv.x;
          d = fmaf(cv.y, qv.y, d);
          d = fmaf(cv.z, qv.z, d);
          v[qq] = fmaf(cv.w, qv.w, d);
        }
        exchange_reduce<SN, LPR_S>(v, lane);
        const int i = bt * 8 + exchange_index<SN, LPR_S>(lane) * RPS + sub;
        const int pg = page_of_lane(pidA, pidB, i);
        if ((ch % (LPR_S / SN)) == 0 && i < it.myrows) {
          const uint32_t key = score_key(pg >= 0 ? v[0] : -INFINITY);
          s_keys[warp + NW * i] = key;
          klo = min(klo, key);
          khi = max(khi, key);
        }
        __syncwarp();  // every lane is done with the slot before it is refilled
      }
      cp_async_wait<0>();
      if (tid == 0 && next < 0) next = claim();
      klo = __reduce_min_sync(kFull, klo);
      khi = __reduce_max_sync(kFull, khi);
      if (lane == 0) {
        s_misc[16 + warp] = (int)klo;
        s_misc[16 + NW + warp] = (int)khi;
      }
      if (warp == 0)
        for (int i = lane; i < SmallTopk<NT>::HIST / 4; i += 32)
          reinterpret_cast<int4*>(tk)[i] = make_int4(0, 0, 0, 0);
      if (tid == 0) s_misc[0] = next;
      __syncthreads();  // all scores of the chunk are in s_keys; the rings are free
      // A scan item next: the loads of its page ids and query rows are issued now and land
      // while this chunk's top-k runs; its first batches follow the top-k.
      const int t2 = s_misc[0];
      prepared = t2 < scan_items;
      const ScanItem it2 = scan_item(prepared ? t2 : t);
      if (prepared) scan_load(it2);
      next = t2;
      klo = 0xffffffffu;
      khi = 0u;
#pragma unroll
      for (int k = 0; k < NW; ++k) {
        klo = min(klo, (uint32_t)s_misc[16 + k]);
        khi = max(khi, (uint32_t)s_misc[16 + NW + k]);
      }
      // exact top-kc of the chunk, stored in ascending page order
      const int kc = min(gm.kc, it.cnt);
      const int64_t cb = ((int64_t)it.u * gm.nch_max + it.c) * gm.kc;
      uint32_t* ck = w.ckey + cb;
      uint16_t* co = w.coff + cb;
      int32_t* cp = w.cpid + cb;
      small_topk<NT>(s_keys, it.cnt, kc, klo, khi, tk, [&](int j, int pos) {
        ck[pos] = s_keys[j];
        co[pos] = (uint16_t)j;
        cp[pos] = s_pids[j];
      });
      // count the chunk as soon as its candidates are stored (the barrier orders every
      // thread's stores before thread 0's release), then put the next chunk's first batches
      // in flight
      __syncthreads();
      if (w.mode == kSelect) {  // the chunk counted last for the unit takes its selection
        if (tid == 0) s_misc[2] = atom_acq_rel_add(w.unit_done + it.u, 1) == it.nch - 1;
        __syncthreads();
        if (s_misc[2]) merge_unit(it.b, it.u, it.nch);
      } else if (tid == 0) {
        red_release_add(w.unit_done + it.u, 1);
      }
      if (prepared) {
        scan_check(it2);
#pragma unroll
        for (int bt = 0; bt < kScanRing - 1; ++bt) scan_issue(it2, bt);
      }
    } else {
      // ---------------------------------------------------------------- attention item
      const int a = t - scan_items;
      const bool early = a < u_split * gm.A;
      const int A = early ? gm.A : gm.A2, pp = early ? gm.pp : gm.pp2;
      const int a2 = early ? a : a - u_split * gm.A;
      const int u = (early ? 0 : u_split) + a2 / A, piece = a2 % A;
      const int b = u / p.Hkv, h = u - b * p.Hkv;
      const int L = p.seq_lens[b];
      const int n = (L + kPage - 1) / kPage;
      const bool valid = L >= 1 && n <= p.pt_stride;
      const bool dense = n <= p.kmax;
      const bool dec = w.mode == kDecode;  // the selection is an input (sel, n_sel)
      const int nch = dec ? 0 : chunks_of(L, p.pt_stride, p.topk, p.bos, p.eos, p.kmax);
      int ns = !valid ? 0 : (dense ? n : p.kmax);
      if (dec) {
        // every piece checks the unit's whole row, so that a bad entry anywhere zeroes all of
        // the unit's outputs
        const int nsi = valid ? p.n_sel[u] : 0;
        int bad = valid && (nsi < 0 || nsi > p.kmax);
        if (!bad)
          for (int j = tid; j < nsi; j += NT) {
            const int v = p.sel[(int64_t)u * p.kmax + j];
            bad |= v < 0 || v >= n;
          }
        bad = __syncthreads_or(bad);
        if (bad && tid == 0 && piece == 0) flag(p.status, VT_DEV_BAD_SEL);
        ns = bad ? 0 : nsi;
      }
      const int j0 = piece * pp;
      const int np = max(0, min(ns - j0, pp));
      const bool write_sel = piece == 0 && p.sel != nullptr && !dec;
      int32_t* selrow = write_sel ? p.sel + (int64_t)u * p.kmax : nullptr;
      if (tid == 0 && piece == 0) {
        if (!valid && h == 0) flag(p.status, VT_DEV_BAD_LEN);
        if (p.n_sel && !dec) p.n_sel[u] = ns;
      }
      int ok = 1;
      if (nch > 0) {
        // wait until every chunk of u has stored its candidates
        if (tid == 0) {
          if (ld_acquire(w.unit_done + u) < nch) {
            const unsigned long long t0 = global_ns();
            for (;;) {
              __nanosleep(32);
              if (ld_acquire(w.unit_done + u) >= nch) break;
              if (global_ns() - t0 > kWaitNs) {
                flag(p.status, kDevTimeout);
                ok = 0;
                break;
              }
            }
          }
          s_misc[1] = ok;
        }
        __syncthreads();
        ok = s_misc[1];
      }
      if (ok) {
        // ---- the logical pages of this piece into s_sel[0, np), their page ids into s_phys
        const int32_t* ptrow = p.page_table + (int64_t)b * p.pt_stride;
        auto checked = [&](int pg) {
          if (pg < 0 || pg >= p.num_pages) {
            flag(p.status, VT_DEV_BAD_PAGE);
            pg = -1;
          }
          return pg;
        };
        bool have_phys = false;
        if (nch > 0) {
          const int m = n - p.bos - p.eos;
          const int kc = gm.kc;
          const int C = (nch - 1) * kc + min(kc, m - (nch - 1) * kChunk);
          const int64_t cb = (int64_t)u * gm.nch_max * kc;  // chunks are contiguous
          const int bos = p.bos, topk = p.topk;
          // thread q < np: the piece's q-th page if it is a reserved one (np <= NT).  Its page
          // id is loaded now and checked only once the candidates' loads below are issued, so
          // that both take one round trip.
          int rlp = -1, rpg = -1;
          if (tid < np) {
            const int pos = j0 + tid;
            if (pos < bos || pos >= bos + topk) {
              rlp = pos < bos ? pos : n - p.eos + (pos - bos - topk);
              rpg = ptrow[rlp];
            }
          }
          if (write_sel) {
            for (int j = tid; j < bos; j += NT) selrow[j] = j;
            for (int j = tid; j < p.eos; j += NT) selrow[bos + topk + j] = n - p.eos + j;
          }
          // candidate j of chunk j / kc sits at offset coff[j] of it; candidates are in
          // ascending page order, so ties (lowest position) go to the lowest page
          if (C <= 2 * NT) {
            // keys, logical pages and page ids of the candidates, fetched together
            uint32_t* keys = reinterpret_cast<uint32_t*>(region);
            int* lps = reinterpret_cast<int*>(region + 2 * NT * 4);
            int* pids = reinterpret_cast<int*>(region + 4 * NT * 4);
            unsigned char* tk = region + 6 * NT * 4;
            for (int i = tid; i < SmallTopk<NT>::HIST / 4; i += NT)
              reinterpret_cast<int4*>(tk)[i] = make_int4(0, 0, 0, 0);
            // candidates tid and tid + NT: every load in flight before any is used
            const bool h0 = tid < C, h1 = tid + NT < C;
            uint32_t key0 = 0, key1 = 0;
            int off0 = 0, off1 = 0, pid0 = -1, pid1 = -1;
            if (h0) {
              key0 = __ldcg(w.ckey + cb + tid);
              off0 = __ldcg(w.coff + cb + tid);
              pid0 = __ldcg(w.cpid + cb + tid);
            }
            if (h1) {
              key1 = __ldcg(w.ckey + cb + tid + NT);
              off1 = __ldcg(w.coff + cb + tid + NT);
              pid1 = __ldcg(w.cpid + cb + tid + NT);
            }
            if (rlp >= 0) {
              s_sel[tid] = rlp;
              s_phys[tid] = checked(rpg);
            }
            uint32_t klo = 0xffffffffu, khi = 0u;
            if (h0) {
              keys[tid] = key0;
              lps[tid] = bos + (tid / kc) * kChunk + off0;
              pids[tid] = pid0;
              klo = key0;
              khi = key0;
            }
            if (h1) {
              const int j = tid + NT;
              keys[j] = key1;
              lps[j] = bos + (j / kc) * kChunk + off1;
              pids[j] = pid1;
              klo = min(klo, key1);
              khi = max(khi, key1);
            }
            klo = __reduce_min_sync(kFull, klo);
            khi = __reduce_max_sync(kFull, khi);
            if (lane == 0) {
              s_misc[16 + warp] = (int)klo;
              s_misc[16 + NW + warp] = (int)khi;
            }
            __syncthreads();
#pragma unroll
            for (int k = 0; k < NW; ++k) {
              klo = min(klo, (uint32_t)s_misc[16 + k]);
              khi = max(khi, (uint32_t)s_misc[16 + NW + k]);
            }
            auto put = [&](int j, int pos) {
              const int q = bos + pos - j0;
              if (q >= 0 && q < np) {
                s_sel[q] = lps[j];
                int pg = pids[j];
                if (pg < 0 || pg >= p.num_pages) {
                  flag(p.status, VT_DEV_BAD_PAGE);
                  pg = -1;
                }
                s_phys[q] = pg;
              }
              if (write_sel) selrow[bos + pos] = lps[j];
            };
            small_topk<NT>(keys, C, topk, klo, khi, tk, put);
            have_phys = true;
          } else {
            if (rlp >= 0) s_sel[tid] = rlp;  // page ids of the whole piece are looked up below
            uint32_t* keys = reinterpret_cast<uint32_t*>(region);
            uint16_t* offs = reinterpret_cast<uint16_t*>(region + align16(gm.cmax * 4));
            int* hist = reinterpret_cast<int*>(region + align16(gm.cmax * 4) + align16(gm.cmax * 2));
            for (int j = tid; j < C; j += NT) {
              keys[j] = __ldcg(w.ckey + cb + j);
              offs[j] = __ldcg(w.coff + cb + j);
            }
            __syncthreads();
            block_topk<NT>(keys, C, topk, hist, hist + kTopkBins, [&](int j, int pos) {
              const int lp = bos + (j / kc) * kChunk + offs[j];
              const int q = bos + pos - j0;
              if (q >= 0 && q < np) s_sel[q] = lp;
              if (write_sel) selrow[bos + pos] = lp;
            });
          }
        } else {
          // dense (every page, in order) or, with topk == 0, the reserved pages alone; or, in
          // a decode-only launch, the given selection
          const bool resv = valid && !dense;
          auto page_at = [&](int pos) {
            return (!resv || pos < p.bos) ? pos : n - p.eos + (pos - p.bos);
          };
          for (int q = tid; q < np; q += NT)
            s_sel[q] = dec ? p.sel[(int64_t)u * p.kmax + j0 + q] : page_at(j0 + q);
          if (write_sel)
            for (int j = tid; j < p.kmax; j += NT) selrow[j] = j < ns ? page_at(j) : -1;
        }
        __syncthreads();
        if (!have_phys) {
          if (tid < np) s_phys[tid] = checked(ptrow[s_sel[tid]]);
          __syncthreads();
        }
        // ---- warp w: pages w + NW i of the piece through a kAttSlots-slot ring
        const int last_valid = L - kPage * (n - 1);
        const uint32_t ring = region_u32 + warp * kAttSlots * S::SLOT;
        auto rows_of = [&](int j) {
          return s_phys[j] < 0 ? 0 : (s_sel[j] == n - 1 ? last_valid : kPage);
        };
        const int npw = (np - warp + NW - 1) / NW;
        auto issue = [&](int i) {
          if (i < npw) {
            const int j = warp + NW * i;
            const int64_t pg = s_phys[j] < 0 ? 0 : s_phys[j];
            stage_page<D>(ring + (i % kAttSlots) * S::SLOT, p.k_pool + pg * p.sk_p + (int64_t)h * p.sk_h,
                          p.v_pool + pg * p.sv_p + (int64_t)h * p.sv_h, p.sk_t, p.sv_t,
                          rows_of(j), p.k_pool, lane);
          }
          cp_async_commit();
        };
#pragma unroll
        for (int i = 0; i < kAttSlots - 1; ++i) issue(i);
        WarpAttention<D, G> att;
        const int64_t orow = (int64_t)b * p.Hq + (int64_t)h * G;
        att.init(p.q + orow * D, lane);
        for (int i = 0; i < npw; ++i) {
          issue(i + kAttSlots - 1);
          cp_async_wait<kAttSlots - 1>();
          __syncwarp();
          att.page(ring + (i % kAttSlots) * S::SLOT, rows_of(warp + NW * i), p.qscale);
          __syncwarp();
        }
        cp_async_wait<0>();
        if (tid == 0) next = claim();
        __syncthreads();  // every warp is done with the staged tiles: partials may reuse them
        float* s_wp = reinterpret_cast<float*>(region);  // [NW][G][D+2]
        float* s_cp = s_wp + NW * G * (D + 2);            // [G][D+2]
        float* s_all = s_cp + G * (D + 2);                // [A][G][D+2]
        att.store(s_wp + warp * G * (D + 2), lane);
        __syncthreads();
        merge_partials<G, D>(s_wp, NW, s_cp, tid, NT);
        __syncthreads();
        int fin = 1;
        if (A > 1) {
          // every piece publishes its partial and counts itself; the piece that arrives last
          // merges all A of them, so no piece ever waits for another
          float* dst = w.part + ((int64_t)u * gm.A2 + piece) * G * (D + 2);
          for (int i = tid; i < G * (D + 2); i += NT) dst[i] = s_cp[i];
          __syncthreads();
          if (tid == 0) {
            // release: the CTA's partial stores (ordered by the barrier); acquire: the partials
            // of the pieces counted before
            const int before = atom_acq_rel_add(w.att_cnt + u, 1);
            s_misc[1] = before == A - 1;
          }
          __syncthreads();
          fin = s_misc[1];
          if (fin) {
            // the A partials into s_all (this piece's own from s_cp), eight loads in flight
            // per thread
            const float* src = w.part + (int64_t)u * gm.A2 * G * (D + 2);
            const int tot = A * G * (D + 2), own0 = piece * G * (D + 2), own1 = own0 + G * (D + 2);
            for (int i0 = 0; i0 < tot; i0 += 8 * NT) {
              float v[8];
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                const int i = i0 + k * NT + tid;
                v[k] = i < tot && (i < own0 || i >= own1) ? __ldcg(src + i) : 0.0f;
              }
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                const int i = i0 + k * NT + tid;
                if (i < tot) s_all[i] = i >= own0 && i < own1 ? s_cp[i - own0] : v[k];
              }
            }
            __syncthreads();
            merge_partials<G, D>(s_all, A, s_cp, tid, NT);
            __syncthreads();
            if (tid == 0) {  // every piece of u is past its waits: reset u's counters
              w.att_cnt[u] = 0;
              w.unit_done[u] = 0;
            }
          }
        } else if (tid == 0 && nch > 0) {
          w.unit_done[u] = 0;
        }
        if (fin) {
          for (int idx = tid; idx < G * D; idx += NT) {
            const int gg = idx / D, d = idx - gg * D;
            const float* pc = s_cp + gg * (D + 2);
            const float Lsum = pc[D + 1];
            p.out[(orow + gg) * D + d] = __float2bfloat16(Lsum > 0.0f ? pc[d] / Lsum : 0.0f);
            if (d == 0 && p.lse)
              p.lse[orow + gg] = Lsum > 0.0f ? (pc[D] + log2f(Lsum)) * kLn2 : -INFINITY;
          }
        }
      }
    }
    if (tid == 0) s_misc[0] = next >= 0 ? next : claim();
    __syncthreads();
  }

}

// ---- host side ----------------------------------------------------------------------------

size_t persist_workspace_bytes(const DecodeParams& p, int G, int Dv, int64_t unit_cap) {
  return persist_ws_layout(p, G, Dv, unit_cap).total;
}

int persist_smem_bytes(const DecodeParams& p, int D, int G) {
  return persist_smem_layout(D, G, p.B, persist_geom(p.pt_stride, p.topk, p.bos, p.eos, p.kmax))
      .total;
}

int persist_max_batch() { return kMaxPlanB; }

template <int D, int G>
static cudaError_t launch_persist_t(const DecodeParams& p, const PersistWs& w, int sm_count,
                                    cudaStream_t stream) {
  auto kern = persist_fused_kernel<D, G>;
  const int smem = persist_smem_layout(D, G, p.B, w.g).total;
  static std::atomic<int> optin[64];
  cudaError_t e = ensure_smem_optin(kern, smem, false, optin);
  if (e != cudaSuccess) return e;
  static std::atomic<long long> occ[64];
  int per_sm = 0;
  e = blocks_per_sm(kern, kPersistThreads, smem, occ, &per_sm);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sm_count * per_sm);
  cfg.blockDim = dim3(kPersistThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p, w);
}

template <int D>
static cudaError_t dispatch_persist_g(const DecodeParams& p, const PersistWs& w, int G,
                                      int sm_count, cudaStream_t s) {
  switch (G) {
    case 1: return launch_persist_t<D, 1>(p, w, sm_count, s);
    case 2: return launch_persist_t<D, 2>(p, w, sm_count, s);
    case 3: return launch_persist_t<D, 3>(p, w, sm_count, s);
    case 4: return launch_persist_t<D, 4>(p, w, sm_count, s);
    case 5: return launch_persist_t<D, 5>(p, w, sm_count, s);
    case 6: return launch_persist_t<D, 6>(p, w, sm_count, s);
    case 7: return launch_persist_t<D, 7>(p, w, sm_count, s);
    case 8: return launch_persist_t<D, 8>(p, w, sm_count, s);
    default: return cudaErrorInvalidValue;
  }
}

// Launch the persistent kernel on `ws` (persist_workspace_bytes() bytes for the same
// unit_cap, counters zero): as many CTAs as fit on the sm_count SMs at once.
cudaError_t launch_persist_fused(const DecodeParams& p, int D, int G, void* ws, int64_t unit_cap,
                                 int sm_count, cudaStream_t s, int mode) {
  const PersistWsLayout L = persist_ws_layout(p, G, D, unit_cap);
  unsigned char* base = static_cast<unsigned char*>(ws);
  PersistWs w;
  w.ctr = reinterpret_cast<uint32_t*>(base + L.ctr);
  w.unit_done = reinterpret_cast<int32_t*>(base + L.unit_done);
  w.att_cnt = reinterpret_cast<int32_t*>(base + L.att_cnt);
  w.ckey = reinterpret_cast<uint32_t*>(base + L.ckey);
  w.coff = reinterpret_cast<uint16_t*>(base + L.coff);
  w.cpid = reinterpret_cast<int32_t*>(base + L.cpid);
  w.part = reinterpret_cast<float*>(base + L.part);
  w.g = persist_geom(p.pt_stride, p.topk, p.bos, p.eos, p.kmax);
  w.units = p.B * p.Hkv;
  w.mode = mode;
  if (D == 64) return dispatch_persist_g<64>(p, w, G, sm_count, s);
  if (D == 128) return dispatch_persist_g<128>(p, w, G, sm_count, s);
  return cudaErrorInvalidValue;
}

}  // namespace vt
