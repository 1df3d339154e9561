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
// Work items, claimed in order through one global counter (each CTA claims its next item
// before it starts on the current one, so the counter's latency is hidden):
//   scan items   -- (request, KV head, chunk of kChunk candidate pages), in request order,
//                   each unit's chunks consecutive.  Every warp streams its rows of the
//                   chunk's fp32 centroids through a cp.async ring and dots them with the
//                   fp32 mean of the unit's G query heads; the CTA then takes the exact top-k
//                   of the chunk in shared memory and stores those candidates (ordered
//                   score key and offset, ascending by page) before counting the chunk done.
//                   The union of the chunks' top-k holds the unit's top-k: a key outside its
//                   chunk's top-k has k keys above it in that chunk alone;
//   attention    -- (unit, piece of kPiecePages selected pages), after every scan item.  The
//   items           CTA waits until all of the unit's chunks are counted (every chunk was
//                   claimed before this item and scan items never wait, so the wait ends),
//                   merges the candidates with the same exact top-k, attends the pages of its
//                   piece on the tensor cores (four per warp through a two-slot ring) and
//                   stores a partial (max, sum, acc); the CTA that completes a unit's last
//                   piece merges the partials and writes the bf16 output and the lse.
// The schedule (scan items per request and their prefix) is computed by every CTA from the
// sequence lengths at start, so the call is one launch.  Every counter is reset by the CTA
// that last uses it, so the workspace needs zero-filling only once.
#include "decode_params.cuh"
#include "gqa_attend.cuh"
#include "topk.cuh"

namespace vt {

constexpr int kPersistThreads = 128;
constexpr int kPersistWarps = kPersistThreads / 32;
constexpr int kChunk = 256;      // candidate pages per scan item (64 per warp)
constexpr int kScanRing = 4;     // 8-row centroid batches per warp ring (3 landing)
constexpr int kPiecePages = 16;  // selected pages per attention item (4 per warp)
constexpr int kMaxPlanB = 2048;  // requests the persistent path takes (schedule kept in smem)

// ---- sizes derived from the call ----------------------------------------------------------

struct PersistGeom {
  int max_cand;  // middle (candidate) pages of a full page-table row, >= 1
  int nch_max;   // chunks of such a row
  int kc;        // candidates a chunk keeps: min(topk, kChunk)
  int A;         // attention pieces per unit
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
  int32_t* ctr;        // [2]: items claimed, CTAs finished
  int32_t* unit_done;  // [U]: chunks of the unit whose candidates are stored
  int32_t* att_cnt;    // [U]: attention pieces of the unit done
  uint32_t* ckey;      // [U][nch_max][kc]: ordered score keys of each chunk's top-k
  uint16_t* coff;      // [U][nch_max][kc]: their offsets in the chunk, ascending
  float* part;         // [U][A][G][Dv+2]: attention partials
  PersistGeom g;
  int units;
};

struct PersistWsLayout {
  size_t ctr, unit_done, att_cnt, ckey, coff, part, total;
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
  L.ctr = o;       o += align256(2 * sizeof(int32_t));
  L.unit_done = o; o += align256(cap * sizeof(int32_t));
  L.att_cnt = o;   o += align256(cap * sizeof(int32_t));
  L.ckey = o;      o += align256(cand * sizeof(uint32_t));
  L.coff = o;      o += align256(cand * sizeof(uint16_t));
  L.part = o;      o += align256(U * g.A * G * (Dv + 2) * sizeof(float));
  L.total = o;
  return L;
}

// ---- memory-order helpers (gpu scope) --------------------------------------------------

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
  int prefix, keys, sel, phys, misc, region, total;
};

__host__ __device__ inline PersistSmem persist_smem_layout(int D, int G, int B,
                                                           const PersistGeom& g) {
  PersistSmem s;
  int o = 0;
  s.prefix = o; o += align16((B + 1) * 4);
  s.keys = o;   o += align16(kChunk * 4);
  s.sel = o;    o += align16(kPiecePages * 4);
  s.phys = o;   o += align16(kPiecePages * 4);
  s.misc = o;   o += align16(64 * 4);
  o = (o + 127) & ~127;
  s.region = o;  // one of: scan rings | top-k scratch | page rings | attention partials
  const int scan = kPersistWarps * kScanRing * 8 * D * 4;
  const int att = kPersistWarps * 2 * 2 * kPage * (D + 8) * 2;
  const int merge = align16(g.cmax * 4) + align16(g.cmax * 2) + align16((kTopkBins + 64) * 4);
  const int comb = align16(kPersistWarps * G * (D + 2) * 4) + align16(G * (D + 2) * 4) +
                   align16(g.A * G * (D + 2) * 4);
  int r = scan;
  if (att > r) r = att;
  if (merge > r) r = merge;
  if (comb > r) r = comb;
  s.total = o + r;
  return s;
}

template <int D, int G>
__global__ void __launch_bounds__(kPersistThreads) persist_fused_kernel(const DecodeParams p,
                                                                        const PersistWs w) {
  using S = PersistShape<D>;
  constexpr int NT = kPersistThreads;
  constexpr int NW = kPersistWarps;
  constexpr int LPR_S = D / 4;     // lanes per centroid row
  constexpr int RPS = 32 / LPR_S;  // centroid rows per warp step
  constexpr int SN = 8 / RPS;      // values per lane per batch of 8 rows
  static_assert(D == 64 || D == 128, "GQA path covers head_dim 64 and 128");

  extern __shared__ __align__(128) unsigned char smem[];
  const PersistGeom gm = w.g;
  const int A = gm.A;
  const PersistSmem Ls = persist_smem_layout(D, G, p.B, gm);
  int* s_prefix = reinterpret_cast<int*>(smem + Ls.prefix);
  uint32_t* s_keys = reinterpret_cast<uint32_t*>(smem + Ls.keys);
  int* s_sel = reinterpret_cast<int*>(smem + Ls.sel);
  int* s_phys = reinterpret_cast<int*>(smem + Ls.phys);
  int* s_misc = reinterpret_cast<int*>(smem + Ls.misc);  // [0] item, [1] flag, [8..] scan
  unsigned char* region = smem + Ls.region;
  const uint32_t region_u32 = smem_u32(region);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // ---- schedule: exclusive prefix of scan items over the requests, in request order
  {
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
    if (tid == 0) s_misc[0] = atomicAdd(w.ctr + 0, 1);
    __syncthreads();
  }
  const int scan_items = s_prefix[p.B];
  const int total_items = scan_items + w.units * A;

  for (;;) {
    const int t = s_misc[0];
    __syncthreads();  // every thread has read the item before the next claim is stored
    if (t >= total_items) break;
    // claim the next item now; its number is only stored (and waited for) at the end
    int next = 0;
    if (tid == 0) next = atomicAdd(w.ctr + 0, 1);

    if (t < scan_items) {
      // ---------------------------------------------------------------- scan item
      int lo = 0, hi = p.B - 1;  // largest k with prefix[k] <= t: a request with items
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_prefix[mid] <= t) lo = mid; else hi = mid - 1;
      }
      const int b = lo;
      const int r = t - s_prefix[b];
      const int L = p.seq_lens[b];
      const int n = (L + kPage - 1) / kPage;
      const int m = n - p.bos - p.eos;
      const int nch = (m + kChunk - 1) / kChunk;
      const int h = r / nch, c = r - h * nch;
      const int u = b * p.Hkv + h;
      const int32_t* ptrow = p.page_table + (int64_t)b * p.pt_stride;
      const int c0 = c * kChunk;
      const int cnt = min(kChunk, m - c0);
      // fp32 mean of the group's queries for this lane's float4 of the row
      const int sub = lane / LPR_S, ch = lane % LPR_S;
      float4 qv = make_float4(0.f, 0.f, 0.f, 0.f);
      {
        const __nv_bfloat16* q0 = p.q + ((int64_t)b * p.Hq + (int64_t)h * G) * D + ch * 4;
#pragma unroll
        for (int j = 0; j < G; ++j) {
          const uint2 raw = *reinterpret_cast<const uint2*>(q0 + (int64_t)j * D);
          qv.x += bf_lo(raw.x);
          qv.y += bf_hi(raw.x);
          qv.z += bf_lo(raw.y);
          qv.w += bf_hi(raw.y);
        }
        qv.x /= (float)G; qv.y /= (float)G; qv.z /= (float)G; qv.w /= (float)G;
      }
      // warp w: rows w + NW i, i < 64 of the chunk; lane l holds the page ids of rows l and
      // l + 32, then streams the rows in batches of 8 through its kScanRing-slot ring
      const int myrows = (cnt - warp + NW - 1) / NW;
      int pidA = -1, pidB = -1;
      if (lane < myrows) pidA = ptrow[p.bos + c0 + warp + NW * lane];
      if (lane + 32 < myrows) pidB = ptrow[p.bos + c0 + warp + NW * (lane + 32)];
      if (pidA >= p.num_pages || pidA < -1 || pidB >= p.num_pages || pidB < -1 ||
          (lane < myrows && pidA < 0) || (lane + 32 < myrows && pidB < 0)) {
        flag(p.status, VT_DEV_BAD_PAGE);
        if (pidA < 0 || pidA >= p.num_pages) pidA = -1;
        if (pidB < 0 || pidB >= p.num_pages) pidB = -1;
      }
      const uint32_t ring = region_u32 + warp * kScanRing * 8 * S::C_ROW;
      const float* cbase = p.centroids + (int64_t)h * D;
      const int64_t cstride = (int64_t)p.Hkv * D;
      const int batches = (myrows + 7) / 8;
      constexpr int CPRS = S::C_ROW / 16;  // 16-byte chunks per centroid row
      auto issue = [&](int bt) {
        if (bt < batches) {
          const uint32_t dst = ring + (bt % kScanRing) * 8 * S::C_ROW;
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
#pragma unroll
      for (int bt = 0; bt < kScanRing - 1; ++bt) issue(bt);
      for (int bt = 0; bt < batches; ++bt) {
        issue(bt + kScanRing - 1);
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
        if ((ch % (LPR_S / SN)) == 0 && i < myrows)
          s_keys[warp + NW * i] = score_key(pg >= 0 ? v[0] : -INFINITY);
        __syncwarp();  // every lane is done with the slot before it is refilled
      }
      cp_async_wait<0>();
      __syncthreads();  // all scores of the chunk are in s_keys; the rings are free
      // exact top-kc of the chunk, stored in ascending page order
      const int kc = min(gm.kc, cnt);
      const int64_t cb = ((int64_t)u * gm.nch_max + c) * gm.kc;
      uint32_t* ck = w.ckey + cb;
      uint16_t* co = w.coff + cb;
      int* hist = reinterpret_cast<int*>(region);
      block_topk<NT>(s_keys, cnt, kc, hist, hist + kTopkBins, [&](int j, int pos) {
        ck[pos] = s_keys[j];
        co[pos] = (uint16_t)j;
      });
      __threadfence();  // this thread's candidates before the unit counter moves
      __syncthreads();
      if (tid == 0) atomicAdd(w.unit_done + u, 1);
    } else {
      // ---------------------------------------------------------------- attention item
      const int a = t - scan_items;
      const int u = a / A, piece = a - u * A;
      const int b = u / p.Hkv, h = u - b * p.Hkv;
      const int L = p.seq_lens[b];
      const int n = (L + kPage - 1) / kPage;
      const bool valid = L >= 1 && n <= p.pt_stride;
      const bool dense = n <= p.kmax;
      const int nch = chunks_of(L, p.pt_stride, p.topk, p.bos, p.eos, p.kmax);
      const int ns = !valid ? 0 : (dense ? n : p.kmax);
      const int j0 = piece * kPiecePages;
      const int np = max(0, min(ns - j0, kPiecePages));
      const bool write_sel = piece == 0 && p.sel != nullptr;
      int32_t* selrow = write_sel ? p.sel + (int64_t)u * p.kmax : nullptr;
      if (tid == 0 && piece == 0) {
        if (!valid && h == 0) flag(p.status, VT_DEV_BAD_LEN);
        if (p.n_sel) p.n_sel[u] = ns;
      }
      int ok = 1;
      if (nch > 0) {
        // wait until every chunk of u has stored its candidates
        if (tid == 0) {
          if (ld_acquire(w.unit_done + u) < nch) {
            const unsigned long long t0 = global_ns();
            for (;;) {
              __nanosleep(128);
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
        // ---- the logical pages of this piece into s_sel[0, np)
        if (nch > 0) {
          const int m = n - p.bos - p.eos;
          const int kc = gm.kc;
          const int C = (nch - 1) * kc + min(kc, m - (nch - 1) * kChunk);
          uint32_t* keys = reinterpret_cast<uint32_t*>(region);
          uint16_t* offs = reinterpret_cast<uint16_t*>(region + align16(gm.cmax * 4));
          int* hist = reinterpret_cast<int*>(region + align16(gm.cmax * 4) + align16(gm.cmax * 2));
          const int64_t cb = (int64_t)u * gm.nch_max * kc;  // chunks are contiguous
          for (int j = tid; j < C; j += NT) {
            keys[j] = __ldcg(w.ckey + cb + j);
            offs[j] = __ldcg(w.coff + cb + j);
          }
          const int bos = p.bos, topk = p.topk;
          for (int q = tid; q < np; q += NT) {  // reserved pages of the piece
            const int pos = j0 + q;
            if (pos < bos) s_sel[q] = pos;
            else if (pos >= bos + topk) s_sel[q] = n - p.eos + (pos - bos - topk);
          }
          if (write_sel) {
            for (int j = tid; j < bos; j += NT) selrow[j] = j;
            for (int j = tid; j < p.eos; j += NT) selrow[bos + topk + j] = n - p.eos + j;
          }
          __syncthreads();
          // candidate j of chunk j / kc sits at offset offs[j] of it; candidates are in
          // ascending page order, so block_topk's ties (lowest position) go to the lowest page
          block_topk<NT>(keys, C, topk, hist, hist + kTopkBins, [&](int j, int pos) {
            const int lp = bos + (j / kc) * kChunk + offs[j];
            const int q = bos + pos - j0;
            if (q >= 0 && q < kPiecePages) s_sel[q] = lp;
            if (write_sel) selrow[bos + pos] = lp;
          });
        } else {
          // dense (every page, in order) or, with topk == 0, the reserved pages alone
          const bool resv = valid && !dense;
          auto page_at = [&](int pos) {
            return (!resv || pos < p.bos) ? pos : n - p.eos + (pos - p.bos);
          };
          for (int q = tid; q < np; q += NT) s_sel[q] = page_at(j0 + q);
          if (write_sel)
            for (int j = tid; j < p.kmax; j += NT) selrow[j] = j < ns ? page_at(j) : -1;
        }
        __syncthreads();
        const int32_t* ptrow = p.page_table + (int64_t)b * p.pt_stride;
        if (tid < np) {
          int pg = ptrow[s_sel[tid]];
          if (pg < 0 || pg >= p.num_pages) {
            flag(p.status, VT_DEV_BAD_PAGE);
            pg = -1;
          }
          s_phys[tid] = pg;
        }
        __syncthreads();
        // ---- warp w: pages w + NW i (i < 4) of the piece through a two-slot ring
        const int last_valid = L - kPage * (n - 1);
        const uint32_t ring = region_u32 + warp * 2 * S::SLOT;
        auto rows_of = [&](int j) {
          return s_phys[j] < 0 ? 0 : (s_sel[j] == n - 1 ? last_valid : kPage);
        };
        const int npw = (np - warp + NW - 1) / NW;
        auto issue = [&](int i) {
          if (i < npw) {
            const int j = warp + NW * i;
            const int64_t pg = s_phys[j] < 0 ? 0 : s_phys[j];
            stage_page<D>(ring + (i & 1) * S::SLOT, p.k_pool + pg * p.sk_p + (int64_t)h * p.sk_h,
                          p.v_pool + pg * p.sv_p + (int64_t)h * p.sv_h, p.sk_t, p.sv_t,
                          rows_of(j), p.k_pool, lane);
          }
          cp_async_commit();
        };
        issue(0);
        WarpAttention<D, G> att;
        const int64_t orow = (int64_t)b * p.Hq + (int64_t)h * G;
        att.init(p.q + orow * D, lane);
        for (int i = 0; i < npw; ++i) {
          issue(i + 1);
          cp_async_wait<1>();
          __syncwarp();
          att.page(ring + (i & 1) * S::SLOT, rows_of(warp + NW * i), p.qscale);
          __syncwarp();
        }
        cp_async_wait<0>();
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
          float* dst = w.part + ((int64_t)u * A + piece) * G * (D + 2);
          for (int i = tid; i < G * (D + 2); i += NT) dst[i] = s_cp[i];
          __threadfence();
          __syncthreads();
          if (tid == 0) {
            const int done = atomicAdd(w.att_cnt + u, 1);
            const int last = (done == A - 1);
            if (last) {  // every piece of u has waited and stored: reset u's counters
              w.att_cnt[u] = 0;
              w.unit_done[u] = 0;
              __threadfence();
            }
            s_misc[1] = last;
          }
          __syncthreads();
          fin = s_misc[1];
          if (fin) {
            const float* src = w.part + (int64_t)u * A * G * (D + 2);
            for (int i = tid; i < A * G * (D + 2); i += NT) s_all[i] = __ldcg(src + i);
            __syncthreads();
            merge_partials<G, D>(s_all, A, s_cp, tid, NT);
            __syncthreads();
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
    if (tid == 0) s_misc[0] = next;
    __syncthreads();
  }

  // leave: the last CTA out resets the queue for the next launch
  if (tid == 0) {
    __threadfence();
    const int out = atomicAdd(w.ctr + 1, 1);
    if (out == (int)gridDim.x - 1) {
      w.ctr[0] = 0;
      __threadfence();
      w.ctr[1] = 0;
    }
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
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kPersistThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  kern<<<sm_count * per_sm, kPersistThreads, smem, stream>>>(p, w);
  return cudaGetLastError();
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
                                 int sm_count, cudaStream_t s) {
  const PersistWsLayout L = persist_ws_layout(p, G, D, unit_cap);
  unsigned char* base = static_cast<unsigned char*>(ws);
  PersistWs w;
  w.ctr = reinterpret_cast<int32_t*>(base + L.ctr);
  w.unit_done = reinterpret_cast<int32_t*>(base + L.unit_done);
  w.att_cnt = reinterpret_cast<int32_t*>(base + L.att_cnt);
  w.ckey = reinterpret_cast<uint32_t*>(base + L.ckey);
  w.coff = reinterpret_cast<uint16_t*>(base + L.coff);
  w.part = reinterpret_cast<float*>(base + L.part);
  w.g = persist_geom(p.pt_stride, p.topk, p.bos, p.eos, p.kmax);
  w.units = p.B * p.Hkv;
  if (D == 64) return dispatch_persist_g<64>(p, w, G, sm_count, s);
  if (D == 128) return dispatch_persist_g<128>(p, w, G, sm_count, s);
  return cudaErrorInvalidValue;
}

}  // namespace vt
