// fused_mla_persistent.cu -- the fused query side for the MLA latent form (one shared latent
// KV head, K row = [latent 512 ; rope 64] bf16, V = the latent part of the same row, 16 or 32
// absorbed query heads of 576 dims) on persistent CTAs that pull work items from a queue.
//
// Sources: "Vortex: Efficient and Programmable Sparse Attention Serving for AI Agents"
// (rndamp.com), "Speedups that scale to 229B parameters" (rope-aware block sparse attention for
// the MLA-based GLM-4.7-Flash on B200) and "A dual-stage programmable abstraction" (workload
// planner, kernel fusion); the thread on digg.com, part [4/6] (MLA's shared latent); the flow
// itself as in the vortex_torch README "Quick Example".  Rope-aware scoring
// q_lat . c_lat + q_rope . c_rope is one dot product over the 576-dim row (the page mean is
// linear in each part).
//
// One CTA of 8 warps per SM (two K tiles, Q, P and the round's scores: ~208 KB of shared
// memory; 256 columns of tensor memory held for the whole launch).
// Items:
//   build items  -- (vt_sparse_decode_step only) the centroid of one page filled at this step;
//   scan items   -- (request, chunk of kMlaChunk candidate pages): each warp streams its rows
//                   of fp32 centroids (2304 B each) through a cp.async ring and dots them with
//                   the fp32 mean of the request's query heads; the CTA keeps the chunk's exact
//                   top-k (key, offset, page id) and counts the chunk done;
//   attention    -- (request, piece of the selected pages): waits until every chunk of the
//   items           request is counted, merges the chunks' candidates with the same exact
//                   top-k, then takes the piece's pages in rounds of kMpRound on the fifth-
//                   generation tensor cores: S^T = K Q^T (M = 64 tokens, N = G heads) and
//                   O^T += V^T P^T (M = 128 output dims, N = G) with both accumulators in
//                   tensor memory, the operands in 128-byte swizzled shared memory (V^T is the
//                   K tile read MN-major), an online softmax between them, and one K tile
//                   landing while the other round computes.  With several pieces, the earlier
//                   ones take whole rounds and publish fp32 partials with one bulk copy each;
//                   the last piece folds them in and writes the request's rows.
// The same kernel, instantiated per mode, serves the select-only call (scan items, then one
// merge item per request that writes its selection) and the decode-only call (attention items
// only, each reading and checking its request's selection).
// Queue, claims and counters work as in the GQA persistent kernel (fused_persistent.cu).
#include "centroid_chunk.cuh"
#include "decode_params.cuh"
#include "topk.cuh"
#include "umma.cuh"

namespace vt {

constexpr int kMpThreads = 256;
constexpr int kMpWarps = kMpThreads / 32;
constexpr int kMpD = 576;
constexpr int kMpDv = 512;
constexpr int kMlaChunk = 256;     // candidate pages per scan item (32 per warp)
constexpr int kMpScanRows = 2;     // centroid rows per ring slot
constexpr int kMpScanSlots = 5;    // ring slots per warp (4 landing while one is used)
constexpr int kMpPiece = 32;       // selected pages per attention item (target)
constexpr int kMpRound = 4;        // pages of a piece staged and computed together (64 tokens)
constexpr int kMpKtBytes = (kMpD / 64) * kMpRound * kPage * 128;  // one round's K tile (72 KB)
constexpr int kMpOcol = 64;        // tensor-memory column of O^T (S^T buffers take [0, 2G))
constexpr int kMpTmemCols = 256;   // tensor-memory columns a CTA holds: 2 G + 4 G <= 192
constexpr int kMpSelCap = kMpPiece + kMpRound;  // most pages of one piece (the last one)
constexpr float kLazyRescale = 8.0f;  // base-2 growth of a head's maximum that moves its reference
constexpr int kMpMaxB = 2048;      // requests the persistent path takes

// ---- sizes derived from the call ----------------------------------------------------------

struct MpGeom {
  int max_cand;  // middle (candidate) pages of a full page-table row, >= 1
  int nch_max;   // chunks of such a row
  int kc;        // candidates a chunk keeps: min(topk, kMlaChunk)
  int cmax;      // candidates one request merges at most
  int A, pp;     // attention pieces per request, pages of each but the last (which takes the rest)
};

__host__ __device__ inline MpGeom mp_geom(int64_t pt_stride, int topk, int bos, int eos, int kmax) {
  MpGeom g;
  const int64_t mc = pt_stride - bos - eos;
  g.max_cand = mc > 1 ? (int)mc : 1;
  g.nch_max = (g.max_cand + kMlaChunk - 1) / kMlaChunk;
  g.kc = topk < kMlaChunk ? (topk > 0 ? topk : 1) : kMlaChunk;
  const int64_t c = (int64_t)g.nch_max * g.kc;
  g.cmax = c < g.max_cand ? (int)c : g.max_cand;
  g.A = (kmax + kMpPiece - 1) / kMpPiece;
  g.pp = (kmax + g.A - 1) / g.A;
  // the pieces before the last take whole rounds, so that they publish their partials about a
  // round before the last piece (which merges them) finishes its own pages
  if (g.A > 1) {
    const int pr = (g.pp / kMpRound) * kMpRound;
    if (pr >= kMpRound && kmax - (g.A - 1) * pr <= kMpSelCap) g.pp = pr;
  }
  return g;
}

// scan items of one request: none when nothing is ranked, else one per chunk of candidates
__host__ __device__ inline int mp_chunks(int L, int64_t pt_stride, int topk, int bos, int eos,
                                         int kmax) {
  const int n = (L + kPage - 1) / kPage;
  if (L < 1 || n > pt_stride || n <= kmax || topk < 1) return 0;
  return (n - bos - eos + kMlaChunk - 1) / kMlaChunk;
}

struct MpWs {
  uint32_t* ctr;       // [2]: claims ever made (mod 2^32), the count when this launch began
  int32_t* unit_done;  // [B]: chunks of the request whose candidates are stored
  int32_t* att_cnt;    // [B]: attention pieces of the request done
  uint32_t* ckey;      // [B][nch_max][kc]: ordered score keys of each chunk's top-k
  uint16_t* coff;      // [B][nch_max][kc]: their offsets in the chunk, ascending
  int32_t* cpid;       // [B][nch_max][kc]: their page ids (-1 where out of range)
  float* part;         // [B][A][G][Dv+4]: attention partials (acc; base-2 max, sums, pad)
  MpGeom g;
};

struct MpWsLayout {
  size_t ctr, unit_done, att_cnt, ckey, coff, cpid, part, total;
};

static inline size_t mp_align256(size_t x) { return (x + 255) & ~(size_t)255; }

static MpWsLayout mp_ws_layout(const DecodeParams& p, int G, int64_t unit_cap) {
  const MpGeom g = mp_geom(p.pt_stride, p.topk, p.bos, p.eos, p.kmax);
  const size_t U = (size_t)p.B;
  const size_t cap = unit_cap > (int64_t)U ? (size_t)unit_cap : U;
  const size_t cand = U * g.nch_max * g.kc;
  MpWsLayout L;
  size_t o = 0;
  L.ctr = o;       o += mp_align256(2 * sizeof(uint32_t));
  L.unit_done = o; o += mp_align256(cap * sizeof(int32_t));
  L.att_cnt = o;   o += mp_align256(cap * sizeof(int32_t));
  L.ckey = o;      o += mp_align256(cand * sizeof(uint32_t));
  L.coff = o;      o += mp_align256(cand * sizeof(uint16_t));
  L.cpid = o;      o += mp_align256(cand * sizeof(int32_t));
  L.part = o;      o += mp_align256(U * g.A * G * (kMpDv + 4) * sizeof(float));
  L.total = o;
  return L;
}

// ---- shared memory -------------------------------------------------------------------------

struct MpSmem {
  int prefix, keys, pids, qm, sel, phys, ml, misc, tc, region;  // region: one phase at a time
  int q, kt, pb, sc, fac, mm;                                   // region offsets (attention)
  int total;  // including 1 KB to align the base to the 1024-byte swizzle atoms
};

__host__ __device__ inline MpSmem mp_smem_layout(int G, int B, const MpGeom& g) {
  MpSmem s;
  int o = 0;
  s.prefix = o; o += align16((B + 1) * 4);
  s.keys = o;   o += align16(kMlaChunk * 4);
  s.pids = o;   o += align16(kMlaChunk * 4);
  s.qm = o;     o += align16(kMpD * 4);
  s.sel = o;    o += align16(kMpSelCap * 4);
  s.phys = o;   o += align16(kMpSelCap * 4);
  s.ml = o;     o += align16(G * 4 * 4);
  s.misc = o;   o += align16(64 * 4);
  s.tc = o;     o += 64;  // four mbarriers, the tensor-memory address
  o = (o + 1023) & ~1023;
  s.region = o;
  // scan: per-warp rings of centroid rows from offset 0 (the chunk top-k scratch reuses warp
  // 0's ring)
  const int scan = kMpWarps * kMpScanSlots * kMpScanRows * kMpD * 4;
  // merge of the request's candidates: keys, logical pages, page ids, top-k scratch
  const int merge_small = 3 * 2 * kMpThreads * 4 + SmallTopk<kMpThreads>::BYTES;
  const int merge_big = align16(g.cmax * 4) + align16(g.cmax * 2) + align16((kTopkBins + 64) * 4);
  const int merge = merge_small > merge_big ? merge_small : merge_big;
  // attention: two buffers of a round's K tiles (first: the merge scratch above is dead once
  // they load), Q (prefetched while the merge runs), two P buffers, the round's scores,
  // rescale factors, the merge's per-head factors; the swizzled operands on 1024-byte bounds
  const int RT = kMpRound * kPage;
  int a = 0;
  s.kt = a; a += 2 * kMpKtBytes;
  s.q = a;  a += (kMpD / 64) * G * 128;
  s.pb = a; a += 2 * G * 128;
  s.sc = a; a += G * RT * 4;
  s.fac = a; a += align16(G * 4);
  s.mm = a; a += align16(G * 8 * 4);
  int r = scan;
  if (merge > r) r = merge;
  if (a > r) r = a;
  s.total = o + r + 1024;
  return s;
}


__device__ __forceinline__ int mp_ld_acquire(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Bounded wait (thread 0) until *ctr >= target; false (and VT_DEV_TIMEOUT) if it gave up.
__device__ __forceinline__ bool mp_wait_at_least(const int32_t* ctr, int target, int32_t* status) {
  if (mp_ld_acquire(ctr) >= target) return true;
  const unsigned long long t0 = global_ns();
  for (;;) {
    __nanosleep(128);
    if (mp_ld_acquire(ctr) >= target) return true;
    if (global_ns() - t0 > kWaitNs) {
      flag(status, kDevTimeout);
      return false;
    }
  }
}

// MODE: kFused, kSelect or kDecode (a template argument, so that the fused launch carries none
// of the other modes' code)
template <int G, int MODE>
__global__ void __launch_bounds__(kMpThreads, 1) persist_mla_kernel(const DecodeParams p,
                                                                    const MpWs w) {
  constexpr int NT = kMpThreads;
  constexpr int NW = kMpWarps;
  constexpr int D = kMpD;
  constexpr int DV = kMpDv;
  constexpr int CH4 = D / 4;  // float4 per centroid row
  constexpr int RB = D * 4;   // bytes of a centroid row
  constexpr int RT = kMpRound * kPage;  // tokens of a round
  static_assert(G == 16 || G == 32, "MLA path covers 16 or 32 query heads");
  static_assert(kMlaChunk <= 32 * kMpWarps, "one page id per lane: at most 32 rows per warp");
  static_assert(RT == 64, "S^T is one M = 64 tile per round: four warps of 16 tokens");
  static_assert(kMpWarps == 8 && DV == 512, "O^T: eight warps hold 2 of its 4 blocks each");
  static_assert(kMpOcol >= 2 * G && kMpOcol + 4 * G <= kMpTmemCols, "tensor-memory columns");
  static_assert(SmallTopk<NT>::BYTES <= kMpScanSlots * kMpScanRows * RB,
                "the chunk top-k scratch fits in warp 0's ring");
  // S^T: M = 64 tokens x N = G heads, both operands K-major; O^T: M = 128 dims x N = G heads,
  // A (V^T) MN-major, B (P) K-major
  constexpr uint32_t kIdescS = umma::idesc_bf16(64, G, false, false);
  constexpr uint32_t kIdescO = umma::idesc_bf16(128, G, true, false);

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // the swizzle atoms need 1024-byte alignment in the shared window
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const MpGeom gm = w.g;
  const MpSmem Ls = mp_smem_layout(G, p.B, gm);
  int* s_prefix = reinterpret_cast<int*>(smem + Ls.prefix);
  uint32_t* s_keys = reinterpret_cast<uint32_t*>(smem + Ls.keys);
  int* s_pids = reinterpret_cast<int*>(smem + Ls.pids);
  float* s_qm = reinterpret_cast<float*>(smem + Ls.qm);
  int* s_sel = reinterpret_cast<int*>(smem + Ls.sel);
  int* s_phys = reinterpret_cast<int*>(smem + Ls.phys);
  float* s_ml = reinterpret_cast<float*>(smem + Ls.ml);
  int* s_misc = reinterpret_cast<int*>(smem + Ls.misc);  // [0] item, [1] flag, [8..] scratch
  unsigned char* region = smem + Ls.region;
  const uint32_t region_u32 = smem_u32(region);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // programmatic dependent launch: nothing global is touched before the previous kernel ends
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

  // tensor memory for the whole launch (warp 0), and the mbarriers: [0], [1] S^T of even and
  // odd rounds, [2] O^T, [3] a partial's bulk load.  Each completion is waited on exactly
  // once, by every thread, so the phase bits below stay in step.
  const uint32_t bars_a = smem_u32(smem + Ls.tc);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + Ls.tc + 32);
  if (warp == 0) umma::tmem_alloc(smem_u32(s_tmem), kMpTmemCols);
  if (tid == 0) {
    umma::mbar_init(bars_a, 1);
    umma::mbar_init(bars_a + 8, 1);
    umma::mbar_init(bars_a + 16, 1);
    umma::mbar_init(bars_a + 24, 1);
    umma::mbar_fence_init();
  }
  umma::fence_before_sync();
  __syncthreads();
  umma::fence_after_sync();
  const uint32_t tm = *s_tmem;
  uint32_t phases = 0u;  // bit i: the parity of mbarrier i's next completion
  // bounded wait for the next completion of mbarrier `which`
  auto bar_wait = [&](int which) {
    const uint32_t bar = bars_a + 8 * which, ph = (phases >> which) & 1u;
    if (!umma::mbar_try_wait(bar, ph)) {
      const unsigned long long t0 = global_ns();
      while (!umma::mbar_try_wait(bar, ph)) {
        if (global_ns() - t0 > kWaitNs) {
          flag(p.status, kDevTimeout);
          break;
        }
      }
    }
    phases ^= 1u << which;
  };

  uint32_t qbase = 0;  // thread 0: the claim count when this launch began
  // items are numbered from -n_fill: the build items of the pages filled at this step first
  auto claim = [&]() { return (int)(atomicAdd(w.ctr + 0, 1u) - qbase) - p.n_fill; };

  // ---- schedule: exclusive prefix of scan items over the requests
  {
    int first = 0;
    if (tid == 0) {
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];\n" : "=r"(qbase) : "l"(w.ctr + 1) : "memory");
      first = claim();
    }
    const int per = (p.B + NT - 1) / NT;
    const int i0 = min(p.B, tid * per), i1 = min(p.B, i0 + per);
    int run = 0;
    for (int i = i0; i < i1; ++i) {
      const int c = MODE == kDecode ? 0
                                      : mp_chunks(p.seq_lens[i], p.pt_stride, p.topk, p.bos, p.eos, p.kmax);
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
  // Queue order: block b holds the scan chunks of request b followed by the attention pieces
  // of request b - lag, and the pieces of the last lag requests come at the end.  The
  // attention (tensor-core bound here) then overlaps the scans (HBM bound) of later requests,
  // and a request's chunks are about five rounds of CTAs ahead of its pieces (measured on the
  // 64-request latent workload with eight-page pieces and 224-page chunks: 1 round 107.2 us,
  // 2 rounds 95.6, 3 rounds 93.9, 5 rounds 93.1, 8 rounds 93.2, every scan first 93.4; with
  // 17-page pieces and 256-page chunks 2 / 3 / 5 rounds gave 84.0 / 75.0 / 75.1 us).  Every
  // wait is still for items earlier in the queue.
  const int scan_items = s_prefix[p.B];
  const int A = MODE == kSelect ? 1 : gm.A;  // items per request after its scans
  const int avg = (scan_items + p.B - 1) / p.B;
  const int lag = min(p.B, 5 * ((int)gridDim.x / (avg + A) + 1));  // ~5 rounds of CTAs
  const int total_items = scan_items + p.B * A;
  auto block_start = [&](int b) { return s_prefix[b] + A * max(0, b - lag); };

  // item t: (scan, request, chunk) or (attention, request, piece)
  auto decode = [&](int t, bool& is_scan, int& ib, int& ic) {
    is_scan = false;
    if (t >= block_start(p.B)) {
      const int r = t - block_start(p.B);
      ib = (p.B - lag) + r / A;
      ic = r % A;
    } else {
      int lo = 0, hi = p.B - 1;  // the block holding t
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (block_start(mid) <= t) lo = mid; else hi = mid - 1;
      }
      const int r = t - block_start(lo), nc = s_prefix[lo + 1] - s_prefix[lo];
      is_scan = r < nc;
      ib = is_scan ? lo : lo - lag;
      ic = is_scan ? r : r - nc;
    }
  };
  // A scan item whose successor is a scan item loads the successor's page ids while its own
  // top-k runs (pre_t, pre_pid), and consecutive chunks of one request keep its query mean in
  // shared memory (qm_b): a chunk then starts streaming one round trip after it is taken.
  int pre_t = -1, pre_pid = -1, qm_b = -1;
  int32_t* pending = nullptr;  // thread 0: a counter to bump after the item's closing barrier
  for (;;) {
    const int t = s_misc[0];
    __syncthreads();
    if (t >= total_items) {
      if (tid == 0 && t == total_items + (int)gridDim.x - 1)
        w.ctr[1] = qbase + (uint32_t)(p.n_fill + total_items) + gridDim.x;
      break;
    }
    int next = -1;
    if (t < 0) {
      // ---------------------------------------------------------------- build item
      // the centroid of one page filled at this step, which no score of this step reads (the
      // page is its request's reserved last page)
      const int64_t pg = p.fill_pages[t + p.n_fill];
      if (pg < 0 || pg >= p.num_pages) {
        if (tid == 0) flag(p.status, VT_DEV_BAD_PAGE);
      } else {
        for (int idx = tid; idx < D / 8; idx += NT)
          build_centroid_chunk(p.k_pool, pg, 0, idx, p.sk_p, p.sk_t, p.sk_h, 1, D, p.cent_out);
      }
      __syncthreads();
      if (tid == 0) s_misc[0] = claim();
      __syncthreads();
      continue;
    }

    bool is_scan;
    int ib, ic;
    decode(t, is_scan, ib, ic);
    if (is_scan) {
      // ---------------------------------------------------------------- scan item
      const int b = ib, c = ic;
      const int L = p.seq_lens[b];
      const int n = (L + kPage - 1) / kPage;
      const int m = n - p.bos - p.eos;
      const int c0 = c * kMlaChunk, cnt = min(kMlaChunk, m - c0);
      const int32_t* ptrow = p.page_table + (int64_t)b * p.pt_stride;
      // warp w: rows w + NW i (i < 32) of the chunk; lane i holds the page id of row i
      const int myrows = (cnt - warp + NW - 1) / NW;
      int pid = -1;
      if (lane < myrows) {
        pid = pre_t == t ? pre_pid : ptrow[p.bos + c0 + warp + NW * lane];
        if (pid < 0 || pid >= p.num_pages) {
          flag(p.status, VT_DEV_BAD_PAGE);
          pid = -1;
        }
        s_pids[warp + NW * lane] = pid;
      }
      // fp32 mean of the request's G query heads: three groups of 72 threads each load every
      // third row (one round of independent 16-byte loads), then sum through shared memory
      const __nv_bfloat16* qb = p.q + (int64_t)b * p.Hq * D;
      if (qm_b != b) {  // (uniform: every thread has seen the same items)
        qm_b = b;
        constexpr int NC8 = D / 8;  // 16-byte chunks per query row
        float* s_part = reinterpret_cast<float*>(region);  // [3][D], in warp 0..2's rings, before use
        const int grp = tid / NC8, c8 = tid - grp * NC8;
        if (grp < 3) {
          float a8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          constexpr int RPG = (G + 2) / 3;
          uint4 raw[RPG];
#pragma unroll
          for (int k = 0; k < RPG; ++k) {
            const int j = grp + 3 * k;
            raw[k] = j < G ? *reinterpret_cast<const uint4*>(qb + (int64_t)j * D + c8 * 8)
                           : make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
          for (int k = 0; k < RPG; ++k) {
            a8[0] += bf_lo(raw[k].x); a8[1] += bf_hi(raw[k].x);
            a8[2] += bf_lo(raw[k].y); a8[3] += bf_hi(raw[k].y);
            a8[4] += bf_lo(raw[k].z); a8[5] += bf_hi(raw[k].z);
            a8[6] += bf_lo(raw[k].w); a8[7] += bf_hi(raw[k].w);
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) s_part[grp * D + c8 * 8 + e] = a8[e];
        }
        __syncthreads();
        for (int d = tid; d < D; d += NT)
          s_qm[d] = ((s_part[d] + s_part[D + d]) + s_part[2 * D + d]) / (float)G;
      }
      __syncthreads();  // the group mean is in shared memory
      float4 qv[5];
#pragma unroll
      for (int i = 0; i < 5; ++i) {
        const int cc = lane + 32 * i;
        qv[i] = cc < CH4 ? reinterpret_cast<const float4*>(s_qm)[cc] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      const uint32_t ring = region_u32 + warp * kMpScanSlots * kMpScanRows * RB;
      const int nb = (myrows + kMpScanRows - 1) / kMpScanRows;
      auto issue = [&](int bt) {
        if (bt < nb) {
          const uint32_t dst = ring + (bt % kMpScanSlots) * kMpScanRows * RB;
#pragma unroll
          for (int rr = 0; rr < kMpScanRows; ++rr) {
            const int i = bt * kMpScanRows + rr;  // uniform, < 28
            const int pg = __shfl_sync(kFull, pid, i & 31);
            if (i < myrows && pg >= 0) {
              const float* crow = p.centroids + (int64_t)pg * D;
              for (int cc = lane; cc < CH4; cc += 32) cp_async16(dst + rr * RB + cc * 16, crow + cc * 4, 16);
            }
          }
        }
        cp_async_commit();
      };
      uint32_t klo = 0xffffffffu, khi = 0u;
#pragma unroll
      for (int bt = 0; bt < kMpScanSlots - 1; ++bt) issue(bt);
      for (int bt = 0; bt < nb; ++bt) {
        issue(bt + kMpScanSlots - 1);
        cp_async_wait<kMpScanSlots - 1>();
        __syncwarp();
        const uint32_t src = ring + (bt % kMpScanSlots) * kMpScanRows * RB;
#pragma unroll
        for (int rr = 0; rr < kMpScanRows; ++rr) {
          float d = 0.0f;
#pragma unroll
          for (int i = 0; i < 5; ++i) {
            const int cc = lane + 32 * i;
            if (cc < CH4) {
              float4 cv;
              asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];\n"
                           : "=f"(cv.x), "=f"(cv.y), "=f"(cv.z), "=f"(cv.w)
                           : "r"(src + rr * RB + cc * 16));
              d = fmaf(cv.x, qv[i].x, d);
              d = fmaf(cv.y, qv[i].y, d);
              d = fmaf(cv.z, qv[i].z, d);
              d = fmaf(cv.w, qv[i].w, d);
            }
          }
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) d += __shfl_xor_sync(kFull, d, o);
          const int i = bt * kMpScanRows + rr;
          const int pg = __shfl_sync(kFull, pid, i & 31);
          if (lane == 0 && i < myrows) {
            const uint32_t key = score_key(pg >= 0 ? d : -INFINITY);
            s_keys[warp + NW * i] = key;
            klo = min(klo, key);
            khi = max(khi, key);
          }
        }
        __syncwarp();  // every lane is done with the slot before it is refilled
      }
      cp_async_wait<0>();
      if (tid == 0) {
        next = claim();
        s_misc[2] = next;
      }
      if (lane == 0) {
        s_misc[16 + warp] = (int)klo;
        s_misc[16 + NW + warp] = (int)khi;
      }
      unsigned char* tk = region;  // warp 0's ring, which only warp 0 has used
      if (warp == 0)
        for (int i = lane; i < SmallTopk<NT>::HIST / 4; i += 32)
          reinterpret_cast<int4*>(tk)[i] = make_int4(0, 0, 0, 0);
      __syncthreads();  // every score of the chunk is in s_keys; the rings are free
      {  // a scan item next: its page ids are loaded now and land while this chunk's top-k runs
        const int t2 = s_misc[2];
        pre_t = -1;
        bool sc2 = false;
        int b2 = 0, c2 = 0;
        if (t2 >= 0 && t2 < total_items) decode(t2, sc2, b2, c2);
        if (sc2) {
          const int n2 = (p.seq_lens[b2] + kPage - 1) / kPage;
          const int c02 = c2 * kMlaChunk, cnt2 = min(kMlaChunk, n2 - p.bos - p.eos - c02);
          const int myrows2 = (cnt2 - warp + NW - 1) / NW;
          pre_pid = lane < myrows2
                        ? p.page_table[(int64_t)b2 * p.pt_stride + p.bos + c02 + warp + NW * lane]
                        : -1;
          pre_t = t2;
        }
      }
      klo = 0xffffffffu;
      khi = 0u;
#pragma unroll
      for (int k = 0; k < NW; ++k) {
        klo = min(klo, (uint32_t)s_misc[16 + k]);
        khi = max(khi, (uint32_t)s_misc[16 + NW + k]);
      }
      const int kc = min(gm.kc, cnt);
      const int64_t cb = ((int64_t)b * gm.nch_max + c) * gm.kc;
      uint32_t* ck = w.ckey + cb;
      uint16_t* co = w.coff + cb;
      int32_t* cp = w.cpid + cb;
      small_topk<NT>(s_keys, cnt, kc, klo, khi, tk, [&](int j, int pos) {
        ck[pos] = s_keys[j];
        co[pos] = (uint16_t)j;
        cp[pos] = s_pids[j];
      });
      pending = w.unit_done + b;
    } else {
      // ---------------------------------------------------------------- attention item
      // (select-only calls: the request's merge item, which writes its selection and stops;
      // decode-only calls: the selection is an input)
      constexpr bool dec = MODE == kDecode, selm = MODE == kSelect;
      const int b = ib, piece = ic;
      const int Ab = A, ppb = gm.pp;
      const int L = p.seq_lens[b];
      const int n = (L + kPage - 1) / kPage;
      const bool valid = L >= 1 && n <= p.pt_stride;
      const bool dense = n <= p.kmax;
      const int nch = dec ? 0 : mp_chunks(L, p.pt_stride, p.topk, p.bos, p.eos, p.kmax);
      int ns = !valid ? 0 : (dense ? n : p.kmax);
      if (dec) {
        // every piece checks the request's whole row, so that a bad entry anywhere zeroes all
        // of the request's outputs
        const int nsi = valid ? p.n_sel[b] : 0;
        int bad = valid && (nsi < 0 || nsi > p.kmax);
        if (!bad)
          for (int j = tid; j < nsi; j += NT) {
            const int v = p.sel[(int64_t)b * p.kmax + j];
            bad |= v < 0 || v >= n;
          }
        bad = __syncthreads_or(bad);
        if (bad && tid == 0 && piece == 0) flag(p.status, VT_DEV_BAD_SEL);
        ns = bad ? 0 : nsi;
      }
      const int j0 = piece * ppb;
      const int np = selm ? 0 : (piece == Ab - 1 ? max(0, ns - j0) : max(0, min(ns - j0, ppb)));
      const bool write_sel = piece == 0 && p.sel != nullptr && !dec;
      int32_t* selrow = write_sel ? p.sel + (int64_t)b * p.kmax : nullptr;
      const int64_t orow = (int64_t)b * p.Hq;
      const int32_t* ptrow = p.page_table + (int64_t)b * p.pt_stride;
      if (tid == 0 && piece == 0) {
        if (!valid) flag(p.status, VT_DEV_BAD_LEN);
        if (p.n_sel && !dec) p.n_sel[b] = ns;
      }
      // Q (G x 576) for the attention below, fetched while the wait and the merge run (its slot
      // lies past every merge scratch of the small path)
      const int m_c = n - p.bos - p.eos;
      const int C_c = nch > 0 ? (nch - 1) * gm.kc + min(gm.kc, m_c - (nch - 1) * kMlaChunk) : 0;
      const bool q_early = !selm && C_c <= 2 * NT;
      const uint32_t q_a = smem_u32(region + Ls.q);  // [atom][G rows][128 B], swizzled K-major
      auto stage_q = [&]() {
        for (int i = tid; i < G * (D / 8); i += NT) {
          const int g = i / (D / 8), c8 = i - g * (D / 8);
          cp_async16(q_a + (c8 >> 3) * (G * 128) + umma::sw128_off(g, c8 & 7),
                     p.q + (orow + g) * D + c8 * 8, 16);
        }
        cp_async_commit();
      };
      if (q_early) stage_q();
      auto phys_of = [&](int lp) {
        int pg = ptrow[lp];
        if (pg < 0 || pg >= p.num_pages) {
          flag(p.status, VT_DEV_BAD_PAGE);
          pg = -1;
        }
        return pg;
      };
      if (nch > 0) {
        // the piece's reserved pages need no score: warp 1 loads their page ids while thread 0
        // waits for the request's chunks below
        const int bos = p.bos, topk = p.topk;
        for (int q = tid - 32; q < np; q += NT) {
          const int pos = j0 + q;
          if (q >= 0 && (pos < bos || pos >= bos + topk)) {
            const int lp = pos < bos ? pos : n - p.eos + (pos - bos - topk);
            s_sel[q] = lp;
            s_phys[q] = phys_of(lp);
          }
        }
      }
      int ok = 1;
      if (nch > 0) {  // every chunk of the request has stored its candidates
        if (tid == 0) s_misc[1] = mp_wait_at_least(w.unit_done + b, nch, p.status) ? 1 : 0;
        __syncthreads();
        ok = s_misc[1];
      }
      if (ok) {
        // ---- the logical pages of this piece into s_sel[0, np), their page ids into s_phys
        bool have_phys = false;
        if (nch > 0) {
          const int m = n - p.bos - p.eos;
          const int kc = gm.kc;
          const int C = (nch - 1) * kc + min(kc, m - (nch - 1) * kMlaChunk);
          const int64_t cb = (int64_t)b * gm.nch_max * kc;  // chunks are contiguous
          const int bos = p.bos, topk = p.topk;  // (the reserved pages are in s_sel already)
          if (write_sel) {
            for (int j = tid; j < bos; j += NT) selrow[j] = j;
            for (int j = tid; j < p.eos; j += NT) selrow[bos + topk + j] = n - p.eos + j;
          }
          // candidate j of chunk j / kc sits at offset coff[j] of it; candidates are in
          // ascending page order, so ties (lowest position) go to the lowest page
          if (C <= 2 * NT) {
            uint32_t* keys = reinterpret_cast<uint32_t*>(region);
            int* lps = reinterpret_cast<int*>(region + 2 * NT * 4);
            int* pids = reinterpret_cast<int*>(region + 4 * NT * 4);
            unsigned char* tk = region + 6 * NT * 4;
            for (int i = tid; i < SmallTopk<NT>::HIST / 4; i += NT)
              reinterpret_cast<int4*>(tk)[i] = make_int4(0, 0, 0, 0);
            uint32_t klo = 0xffffffffu, khi = 0u;
            for (int j = tid; j < C; j += NT) {
              const uint32_t key = __ldcg(w.ckey + cb + j);
              keys[j] = key;
              lps[j] = bos + (j / kc) * kMlaChunk + __ldcg(w.coff + cb + j);
              pids[j] = __ldcg(w.cpid + cb + j);
              klo = min(klo, key);
              khi = max(khi, key);
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
            small_topk<NT>(keys, C, topk, klo, khi, tk, [&](int j, int pos) {
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
            });
            have_phys = true;
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
              const int lp = bos + (j / kc) * kMlaChunk + offs[j];
              const int q = bos + pos - j0;
              if (q >= 0 && q < np) s_sel[q] = lp;
              if (write_sel) selrow[bos + pos] = lp;
            });
          }
        } else {
          // dense (every page, in order) or, with topk == 0, the reserved pages alone
          const bool resv = valid && !dense;
          auto page_at = [&](int pos) {
            return (!resv || pos < p.bos) ? pos : n - p.eos + (pos - p.bos);
          };
          for (int q = tid; q < np; q += NT)
            s_sel[q] = dec ? p.sel[(int64_t)b * p.kmax + j0 + q] : page_at(j0 + q);
          if (write_sel)
            for (int j = tid; j < p.kmax; j += NT) selrow[j] = j < ns ? page_at(j) : -1;
        }
        __syncthreads();
        if (!have_phys) {
          if (tid < np) s_phys[tid] = phys_of(s_sel[tid]);
          __syncthreads();
        }
        if (selm) {
          // select-only: the request's selection is written; its chunk counter goes back to 0
          if (tid == 0 && nch > 0) w.unit_done[b] = 0;
        } else {
          // ---- the piece's pages in rounds of kMpRound pages (RT = 64 tokens) on the tensor cores.
          // A round's K tile lands (zero rows past the valid tokens) in 128-byte swizzled K-major
          // order in one of two buffers; per round
          //   S^T = K Q^T      M = 64 tokens, N = G heads, K = 576, into tensor memory;
          //   the softmax of each head against its reference maximum, through a shared-memory
          //                    transpose of S^T (a group of NT / G threads per head); P in bf16,
          //                    heads x tokens, as the next MMA's K-major operand;
          //   O^T += V^T P^T   M = 128 output dims per block (four blocks), N = G, K = the round's
          //                    tokens; V^T is the latent part of the same K tile, read MN-major;
          //                    O^T stays in tensor memory for the whole piece.
          // A head's reference maximum moves only when a round's maximum exceeds it by more than
          // kLazyRescale (base 2), and O^T is then rescaled in tensor memory; P stays below 2^8.
          // The tensor core runs round r's MMAs while round r + 1's tile lands in the other buffer.
          unsigned char* kt = region + Ls.kt;
          const uint32_t kt_a = smem_u32(kt), pb_a = smem_u32(region + Ls.pb);
          float* s_sc = reinterpret_cast<float*>(region + Ls.sc);    // [G][RT] scores of the round
          float* s_fac = reinterpret_cast<float*>(region + Ls.fac);  // [G] rescale factors
          const int last_valid = L - kPage * (n - 1);
          if (!q_early) stage_q();
          const int nr = (np + kMpRound - 1) / kMpRound;
          auto row_ok = [&](int j, int tt) {  // token tt of the piece's j-th page is attended
            return j < np && s_phys[j] >= 0 && (s_sel[j] != n - 1 || tt < last_valid);
          };
          // staging: thread t copies rows t / 8 and t / 8 + 32 of the round, 16-byte chunk t % 8
          // of each of the nine 128-byte atoms (eight threads read 128 contiguous bytes of a row)
          static_assert(NT == 4 * RT, "eight threads per row, two rows per thread");
          const int st_c = tid & 7;
          auto stage_round = [&](int r) {  // every thread commits one group per call
            if (r < nr) {
              const uint32_t buf = kt_a + (r & 1) * kMpKtBytes;
  #pragma unroll
              for (int h2 = 0; h2 < 2; ++h2) {
                const int row = (tid >> 3) + 32 * h2;
                const int j = r * kMpRound + row / kPage, tt = row % kPage;
                const bool ok_row = row_ok(j, tt);
                const __nv_bfloat16* src =
                    ok_row ? p.k_pool + (int64_t)s_phys[j] * p.sk_p + (int64_t)tt * p.sk_t + st_c * 8
                           : p.k_pool;
                const uint32_t dst = buf + umma::sw128_off(row, st_c);
  #pragma unroll
                for (int kb = 0; kb < D / 64; ++kb)
                  cp_async16(dst + kb * (RT * 128), src + (ok_row ? kb * 64 : 0), ok_row ? 16 : 0);
              }
            }
            cp_async_commit();
          };
          constexpr int TPH = NT / G;   // softmax threads per head
          constexpr int TPT = RT / TPH; // tokens per softmax thread
          const int sh = tid / TPH, spart = tid % TPH;  // this thread's head and token group
          // the head's reference maximum, the sum of its bf16 weights (as the MMA reads them: O's
          // normaliser) and the sum of the same weights unrounded (for the lse: with a reference
          // below the maximum, the largest weight is not a power of two and its rounding would
          // reach the lse)
          float M_run = -INFINITY, L_run = 0.0f, Le_run = 0.0f;
          stage_round(0);
          stage_round(1);
          for (int r = 0; r < nr; ++r) {
            // round r has landed (and Q with it): S^T(r) on the tensor core
            if (r == 0) cp_async_wait<1>(); else cp_async_wait<0>();
            umma::fence_async_smem();
            __syncthreads();
            if (warp == 0) {
              umma::fence_after_sync();
              const uint32_t ka = kt_a + (r & 1) * kMpKtBytes;
              const uint32_t d = tm + (uint32_t)((r & 1) * G);
  #pragma unroll
              for (int ks = 0; ks < D / 16; ++ks)
                umma::mma_bf16(d, umma::sdesc_sw128(ka + (ks >> 2) * (RT * 128) + (ks & 3) * 32, 16, 1024),
                               umma::sdesc_sw128(q_a + (ks >> 2) * (G * 128) + (ks & 3) * 32, 16, 1024),
                               kIdescS, ks > 0 ? 1u : 0u);
              umma::commit(bars_a + 8 * (r & 1));
            }
            if (r >= 1) {
              // O^T(r - 1) has completed (its commit is waited on once), so the buffer it read
              // takes round r + 1
              bar_wait(2);
              if (r + 1 < nr) stage_round(r + 1);
            }
            bar_wait(r & 1);
            umma::fence_after_sync();
            if (warp < 4) {  // token 16 w + lane (lane < 16) sits in lane 32 w + lane
              uint32_t v[G / 16][16];
  #pragma unroll
              for (int c = 0; c < G / 16; ++c)
                umma::tmem_ld16(tm + ((uint32_t)(32 * warp) << 16) + (uint32_t)((r & 1) * G + 16 * c), v[c]);
              umma::fence_before_sync();
              if (lane < 16) {
                const bool ok = row_ok(r * kMpRound + warp, lane);
                const int t = 16 * warp + lane;
  #pragma unroll
                for (int h = 0; h < G; ++h)
                  s_sc[h * RT + t] = ok ? __uint_as_float(v[h >> 4][h & 15]) * p.qscale : -INFINITY;
              }
            }
            __syncthreads();
            // softmax of head sh over tokens [TPT spart, TPT spart + TPT) of the round
            int need = 0;
            {
              float sv[TPT];
  #pragma unroll
              for (int i = 0; i < TPT; i += 4) {
                const float4 f4 = *reinterpret_cast<const float4*>(s_sc + sh * RT + spart * TPT + i);
                sv[i] = f4.x; sv[i + 1] = f4.y; sv[i + 2] = f4.z; sv[i + 3] = f4.w;
              }
              float mr = sv[0];
  #pragma unroll
              for (int i = 1; i < TPT; ++i) mr = fmaxf(mr, sv[i]);
  #pragma unroll
              for (int o = 1; o < TPH; o <<= 1) mr = fmaxf(mr, __shfl_xor_sync(kFull, mr, o));
              const float Mn = mr > M_run + kLazyRescale ? mr : M_run;
              const float fac = Mn == M_run ? 1.0f : (M_run == -INFINITY ? 0.0f : exp2f(M_run - Mn));
              float ls = 0.0f, le = 0.0f;
              uint32_t pk[TPT / 2];
  #pragma unroll
              for (int i = 0; i < TPT; i += 2) {
                const float e0 = sv[i] == -INFINITY ? 0.0f : exp2f(sv[i] - Mn);
                const float e1 = sv[i + 1] == -INFINITY ? 0.0f : exp2f(sv[i + 1] - Mn);
                const __nv_bfloat16 p0 = __float2bfloat16(e0), p1 = __float2bfloat16(e1);
                ls += __bfloat162float(p0) + __bfloat162float(p1);  // the weights the MMA reads
                le += e0 + e1;
                pk[i / 2] = (uint32_t)__bfloat16_as_ushort(p0) | ((uint32_t)__bfloat16_as_ushort(p1) << 16);
              }
  #pragma unroll
              for (int o = 1; o < TPH; o <<= 1) {
                ls += __shfl_xor_sync(kFull, ls, o);
                le += __shfl_xor_sync(kFull, le, o);
              }
              L_run = fmaf(L_run, fac, ls);
              Le_run = fmaf(Le_run, fac, le);
              M_run = Mn;
              unsigned char* prow = region + Ls.pb + (r & 1) * (G * 128);
              if constexpr (TPT == 8) {
                *reinterpret_cast<uint4*>(prow + umma::sw128_off(sh, spart)) =
                    make_uint4(pk[0], pk[1], pk[2], pk[3]);
              } else {
                *reinterpret_cast<uint2*>(prow + umma::sw128_off(sh, spart >> 1) + (spart & 1) * 8) =
                    make_uint2(pk[0], pk[1]);
              }
              if (spart == 0) s_fac[sh] = fac;
              need = (r > 0 && fac != 1.0f) ? 1 : 0;
            }
            umma::fence_async_smem();  // P is read by the tensor core
            if (__syncthreads_or(need)) {
              // O^T *= fac per head (column); O^T(r - 1) has completed.  Warp w rescales blocks
              // 2 (w / 4) and 2 (w / 4) + 1 in its lane quarter.
              const int sp = warp & 3, bh = warp >> 2;
  #pragma unroll
              for (int bi = 0; bi < 2; ++bi)
  #pragma unroll
                for (int c = 0; c < G / 16; ++c) {
                  const uint32_t ta = tm + ((uint32_t)(32 * sp) << 16) +
                                      (uint32_t)(kMpOcol + G * (2 * bh + bi) + 16 * c);
                  uint32_t v[16];
                  umma::tmem_ld16(ta, v);
  #pragma unroll
                  for (int j = 0; j < 16; ++j)
                    v[j] = __float_as_uint(__uint_as_float(v[j]) * s_fac[16 * c + j]);
                  umma::tmem_st16(ta, v);
                }
              umma::fence_before_sync();
              __syncthreads();
            }
            if (warp == 0) {  // O^T += V^T P^T over the round's pages (16 tokens each)
              umma::fence_after_sync();
              const int pr = min(kMpRound, np - r * kMpRound);
              const uint32_t ka = kt_a + (r & 1) * kMpKtBytes, pa = pb_a + (r & 1) * (G * 128);
  #pragma unroll
              for (int i = 0; i < DV / 128; ++i)
  #pragma unroll
                for (int ks = 0; ks < kMpRound; ++ks)
                  if (ks < pr)
                    umma::mma_bf16(tm + (uint32_t)(kMpOcol + G * i),
                                   umma::sdesc_sw128(ka + 2 * i * (RT * 128) + ks * 2048, RT * 128, 1024),
                                   umma::sdesc_sw128(pa + ks * 32, 16, 1024), kIdescO,
                                   (r > 0 || ks > 0) ? 1u : 0u);
              umma::commit(bars_a + 16);
            }
          }
          cp_async_wait<0>();
          if (nr > 0) {
            bar_wait(2);
            umma::fence_after_sync();
          }
          if (spart == 0) {
            s_ml[4 * sh] = M_run;
            s_ml[4 * sh + 1] = L_run;
            s_ml[4 * sh + 2] = Le_run;
          }
          // this thread's outputs: dims 128 (2 (w / 4) + bi) + 32 (w % 4) + lane, every head
          const int sp = warp & 3, bh = warp >> 2;
          float o[2][G];
          if (nr > 0) {
  #pragma unroll
            for (int bi = 0; bi < 2; ++bi)
  #pragma unroll
              for (int c = 0; c < G / 16; ++c) {
                uint32_t v[16];
                umma::tmem_ld16(tm + ((uint32_t)(32 * sp) << 16) +
                                    (uint32_t)(kMpOcol + G * (2 * bh + bi) + 16 * c), v);
  #pragma unroll
                for (int j = 0; j < 16; ++j) o[bi][16 * c + j] = __uint_as_float(v[j]);
              }
          } else {
  #pragma unroll
            for (int bi = 0; bi < 2; ++bi)
  #pragma unroll
              for (int h = 0; h < G; ++h) o[bi][h] = 0.0f;
          }
          umma::fence_before_sync();
          __syncthreads();  // s_ml is complete
          auto dim_of = [&](int bi) { return 128 * (2 * bh + bi) + 32 * sp + lane; };
          // Results leave through shared memory (the K buffers are free now) and one bulk copy:
          // the output rows of this request ([G][DV] bf16, contiguous), or a piece's partial
          // ([G][DV + 4] fp32: unnormalised O, reference maximum, the two sums, pad).
          constexpr int PR = DV + 4;
          constexpr uint32_t kPartBytes = G * PR * 4;
          float* tile = reinterpret_cast<float*>(region);
          const uint32_t tile_a = smem_u32(region);
          auto store_out = [&](auto&& scale_of) {  // scale_of(h): the head's 1 / L
            __nv_bfloat16* dst = p.out + orow * DV;
            if ((reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
              __nv_bfloat16* ot = reinterpret_cast<__nv_bfloat16*>(region);
  #pragma unroll
              for (int h = 0; h < G; ++h) {
                const float inv = scale_of(h);
  #pragma unroll
                for (int bi = 0; bi < 2; ++bi) ot[h * DV + dim_of(bi)] = __float2bfloat16(o[bi][h] * inv);
              }
              umma::fence_async_smem();
              __syncthreads();
              if (tid == 0) {  // the item's closing barrier waits for thread 0, so for the read
                umma::bulk_s2g(dst, tile_a, G * DV * 2);
                umma::bulk_wait_read();
              }
            } else {
  #pragma unroll
              for (int h = 0; h < G; ++h) {
                const float inv = scale_of(h);
  #pragma unroll
                for (int bi = 0; bi < 2; ++bi) dst[h * DV + dim_of(bi)] = __float2bfloat16(o[bi][h] * inv);
              }
            }
          };
          if (Ab == 1) {
            store_out([&](int h) { return s_ml[4 * h + 1] > 0.0f ? 1.0f / s_ml[4 * h + 1] : 0.0f; });
            if (spart == 0 && p.lse)
              p.lse[orow + sh] = Le_run > 0.0f ? (M_run + log2f(Le_run)) * kLn2 : -INFINITY;
            if (tid == 0 && nch > 0) w.unit_done[b] = 0;
          } else if (piece < Ab - 1) {
            // publish this piece's partial and move on: the request's last piece merges them
  #pragma unroll
            for (int h = 0; h < G; ++h)
  #pragma unroll
              for (int bi = 0; bi < 2; ++bi) tile[h * PR + dim_of(bi)] = o[bi][h];
            if (spart == 0) {
              tile[sh * PR + DV] = M_run;
              tile[sh * PR + DV + 1] = L_run;
              tile[sh * PR + DV + 2] = Le_run;
              tile[sh * PR + DV + 3] = 0.0f;
            }
            umma::fence_async_smem();
            __syncthreads();
            if (tid == 0) {  // complete before the count that publishes it (after the item)
              umma::bulk_s2g(w.part + ((int64_t)b * A + piece) * G * PR, tile_a, kPartBytes);
              umma::bulk_wait_done();
            }
            pending = w.att_cnt + b;
          } else {
            // the last piece: wait for the other Ab - 1 partials (claimed before this item, and
            // they never wait on a later one), then fold them in one at a time: each lands in
            // shared memory with one bulk copy, and the running maximum and sum move with it
            if (tid == 0) s_misc[1] = mp_wait_at_least(w.att_cnt + b, Ab - 1, p.status) ? 1 : 0;
            // per head: [0] maximum, [1] [2] the two sums, [3] [4] the factors of this step, [5] 1/L
            float* s_mm = reinterpret_cast<float*>(region + Ls.mm);  // [G][8]
            for (int g = tid; g < G; g += NT) {
              s_mm[8 * g] = s_ml[4 * g];
              s_mm[8 * g + 1] = s_ml[4 * g + 1];
              s_mm[8 * g + 2] = s_ml[4 * g + 2];
            }
            __syncthreads();
            if (s_misc[1]) {
              const float* src = w.part + (int64_t)b * A * G * PR;
              for (int q = 0; q < Ab - 1; ++q) {
                if (tid == 0) {
                  umma::fence_async_global();
                  umma::mbar_expect_tx(bars_a + 24, kPartBytes);
                  umma::bulk_g2s(tile_a, src + (int64_t)q * G * PR, kPartBytes, bars_a + 24);
                }
                bar_wait(3);
                for (int g = tid; g < G; g += NT) {
                  const float mq = tile[g * PR + DV];
                  const float M = s_mm[8 * g], Mn = fmaxf(M, mq);
                  const float fo = M == -INFINITY ? 0.0f : exp2f(M - Mn);
                  const float fq = mq == -INFINITY ? 0.0f : exp2f(mq - Mn);
                  s_mm[8 * g] = Mn;
                  s_mm[8 * g + 1] = fmaf(s_mm[8 * g + 1], fo, tile[g * PR + DV + 1] * fq);
                  s_mm[8 * g + 2] = fmaf(s_mm[8 * g + 2], fo, tile[g * PR + DV + 2] * fq);
                  s_mm[8 * g + 3] = fo;
                  s_mm[8 * g + 4] = fq;
                }
                __syncthreads();
  #pragma unroll
                for (int h = 0; h < G; ++h) {
                  const float fo = s_mm[8 * h + 3], fq = s_mm[8 * h + 4];
  #pragma unroll
                  for (int bi = 0; bi < 2; ++bi)
                    o[bi][h] = fmaf(tile[h * PR + dim_of(bi)], fq, o[bi][h] * fo);
                }
                __syncthreads();  // the tile is free for the next partial (or the output)
              }
              for (int g = tid; g < G; g += NT) {
                const float M = s_mm[8 * g], Lsum = s_mm[8 * g + 1], Le = s_mm[8 * g + 2];
                s_mm[8 * g + 5] = Lsum > 0.0f ? 1.0f / Lsum : 0.0f;
                if (p.lse) p.lse[orow + g] = Le > 0.0f ? (M + log2f(Le)) * kLn2 : -INFINITY;
              }
              __syncthreads();
              store_out([&](int h) { return s_mm[8 * h + 5]; });
              if (tid == 0) {  // every piece is past its waits: reset the request's counters
                w.att_cnt[b] = 0;
                w.unit_done[b] = 0;
              }
            }
          }
        }
      }
    }
    if (tid == 0) s_misc[0] = next >= 0 ? next : claim();
    __syncthreads();
    if (tid == 0 && pending != nullptr) {
      // the barrier above ordered every thread's stores of the item before this fence
      __threadfence();
      atomicAdd(pending, 1);
      pending = nullptr;
    }
  }
  // every MMA of this launch has completed (each attention item waits for its last one)
  umma::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    umma::fence_after_sync();
    umma::tmem_dealloc(tm, kMpTmemCols);
  }
}


// ---- host side ----------------------------------------------------------------------------

size_t mla_persist_workspace_bytes(const DecodeParams& p, int G, int64_t unit_cap) {
  return mp_ws_layout(p, G, unit_cap).total;
}

int mla_persist_smem_bytes(const DecodeParams& p, int G) {
  return mp_smem_layout(G, p.B, mp_geom(p.pt_stride, p.topk, p.bos, p.eos, p.kmax)).total;
}

int mla_persist_max_batch() { return kMpMaxB; }

template <int G, int MODE>
static cudaError_t launch_mla_persist_t(const DecodeParams& p, const MpWs& w, int sm_count,
                                        cudaStream_t stream) {
  auto kern = persist_mla_kernel<G, MODE>;
  const int smem = mp_smem_layout(G, p.B, w.g).total;
  static std::atomic<int> optin[64];
  cudaError_t e = ensure_smem_optin(kern, smem, false, optin);
  if (e != cudaSuccess) return e;
  static std::atomic<long long> occ[64];
  int per_sm = 0;
  e = blocks_per_sm(kern, kMpThreads, smem, occ, &per_sm);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sm_count * per_sm);
  cfg.blockDim = dim3(kMpThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p, w);
}

// The MLA call (fused, select-only or decode-only, by `mode`) on `ws`
// (mla_persist_workspace_bytes() bytes for the same unit_cap, counters zero): as many CTAs as
// fit on the sm_count SMs at once.
cudaError_t launch_mla_persist(const DecodeParams& p, int G, void* ws, int64_t unit_cap,
                               int sm_count, cudaStream_t s, int mode) {
  const MpWsLayout L = mp_ws_layout(p, G, unit_cap);
  unsigned char* base = static_cast<unsigned char*>(ws);
  MpWs w;
  w.ctr = reinterpret_cast<uint32_t*>(base + L.ctr);
  w.unit_done = reinterpret_cast<int32_t*>(base + L.unit_done);
  w.att_cnt = reinterpret_cast<int32_t*>(base + L.att_cnt);
  w.ckey = reinterpret_cast<uint32_t*>(base + L.ckey);
  w.coff = reinterpret_cast<uint16_t*>(base + L.coff);
  w.cpid = reinterpret_cast<int32_t*>(base + L.cpid);
  w.part = reinterpret_cast<float*>(base + L.part);
  w.g = mp_geom(p.pt_stride, p.topk, p.bos, p.eos, p.kmax);
  if (mode != kFused && mode != kSelect && mode != kDecode) return cudaErrorInvalidValue;
  if (G == 16)
    return mode == kFused    ? launch_mla_persist_t<16, kFused>(p, w, sm_count, s)
           : mode == kSelect ? launch_mla_persist_t<16, kSelect>(p, w, sm_count, s)
                             : launch_mla_persist_t<16, kDecode>(p, w, sm_count, s);
  if (G == 32)
    return mode == kFused    ? launch_mla_persist_t<32, kFused>(p, w, sm_count, s)
           : mode == kSelect ? launch_mla_persist_t<32, kSelect>(p, w, sm_count, s)
                             : launch_mla_persist_t<32, kDecode>(p, w, sm_count, s);
  return cudaErrorInvalidValue;
}

}  // namespace vt
