// decode_gqa.cu -- query side of block top-k sparse decode for GQA heads (head_dim 64/128,
// group G <= 8 query heads per KV head): group-mean query, GeMV against the page centroids,
// exact top-k with the reserved first/last pages, exact softmax attention over the selected
// pages.
//
// Sources: "Vortex: A Flexible and Efficient Sparse Attention Framework" (vortex_torch
// README), "Quick Example" (forward_indexer: q.mean -> GeMV -> topK) and "Using Your Sparse
// Attention with SGLang" (page size 16, vortex_topk_val, reserved bos/eos pages); "Vortex:
// Efficient and Programmable Sparse Attention Serving for AI Agents", "A dual-stage
// programmable abstraction" (query-dependent scoring, top-k block selection, attention over
// the paged layout; kernel fusion).
//
// One thread-block cluster of C CTAs (4 warps each) serves one (request, KV head) unit:
//   1. score (CUDA cores): CTA r scores a contiguous 1/C of the middle pages.  Each warp
//      streams fp32 centroid rows through the page table with 16-byte loads, one batch of 8
//      rows in flight while the previous batch is reduced (exchange reduction: 9 shuffles
//      for 8 rows); the GEMV has one query row, so it stays on the FMA pipe;
//   2. select: after one cluster barrier every CTA reads all the unit's scores over DSMEM and
//      runs the same exact top-k (so no CTA waits for another); ties go to the lower page;
//   3. attend (tensor cores): CTA r takes 1/C of the selected pages and each warp a quarter
//      of those, page by page.  A warp stages its next page's K and V rows into its own
//      shared-memory slot with 16-byte cp.async copies (rows past the end of the request are
//      zero-filled) while it computes on the current one:
//        S = Q K^T   (m16n8k16, bf16 -> fp32; the G query rows padded to 16, K from
//                     ldmatrix), scaled and masked, online softmax per query head,
//        O += P V    (P straight from the S fragments, V through ldmatrix.trans).
//      With only G <= 8 useful rows the MMA is mostly padding, but it replaces ~400 CUDA-core
//      instructions per page (bf16 unpacking, G FMAs per element, reductions) by ~75, and
//      this phase is limited by instruction issue, not by FLOPs;
//   4. the warps' and then the C CTAs' (max, sum, acc) partials are merged, the latter over
//      DSMEM, each CTA writing 1/C of the unit's G x D outputs (and lse).
// A request with n <= topk+bos+eos pages skips 1-2 and attends to every page.
#include "decode_params.cuh"
#include "gqa_attend.cuh"
#include "topk.cuh"

namespace vt {

constexpr int kGqaThreads = 128;
constexpr int kGqaWarps = kGqaThreads / 32;
constexpr int kGqaSlots = 3;       // page slots per warp: one computing, two landing
constexpr int kScanSlots = 6;      // centroid batches (8 rows) per warp: five landing

template <int D>
struct GqaShape : PageTile<D> {
  static constexpr int C_ROW = D * 4;           // bytes of one fp32 centroid row
  static constexpr int SCAN_SLOT = 8 * C_ROW;   // one batch: 8 centroid rows
  static constexpr int WARP_RING = (kGqaSlots * PageTile<D>::SLOT > kScanSlots * SCAN_SLOT)
                                       ? kGqaSlots * PageTile<D>::SLOT : kScanSlots * SCAN_SLOT;
};

__host__ __device__ inline GqaSmem gqa_smem_layout(int D, int G, int cand_cap, int key_cap,
                                                   int kmax) {
  GqaSmem s;
  int o = 0;
  s.score = o; o += align16(cand_cap * 4);  // read by cluster peers until the end
  s.sel = o;   o += align16(kmax * 4);
  s.phys = o;  o += align16(kmax * 4);
  s.qm = o;    o += align16(D * 4);         // live during the scan
  s.cpage = o; o += align16(cand_cap * 4);  // live during the scan
  o = (o + 127) & ~127;
  const int base = o;  // one region, three successive uses:
  // selection (after the scan has drained its ring)
  int a = base;
  s.key = a;   a += align16(key_cap * 4);
  s.misc = a;  a += align16((kTopkBins + 64) * 4);
  // streaming phases: per-warp rings (centroid batches, then K/V page tiles)
  s.ring = base;
  const int att = kGqaSlots * 2 * kPage * (D + 8) * 2, scn = kScanSlots * 8 * D * 4;
  const int ring_end = base + kGqaWarps * (att > scn ? att : scn);
  // combine phase (after the slots are drained)
  int c = base;
  s.warp = c;  c += align16(kGqaWarps * G * (D + 2) * 4);
  s.cta = c;   c += align16(G * (D + 2) * 4);
  int end = a > ring_end ? a : ring_end;
  s.total = end > c ? end : c;
  return s;
}

template <int D, int G, int MODE>
__global__ void __launch_bounds__(kGqaThreads) gqa_decode_kernel(const DecodeParams p) {
  using S = GqaShape<D>;
  constexpr int NT = kGqaThreads;
  constexpr int NW = kGqaWarps;
  constexpr int LPR_S = D / 4;     // lanes per centroid row: one float4 each
  constexpr int RPS = 32 / LPR_S;  // centroid rows per warp step
  constexpr int SN = 8 / RPS;      // values per lane per batch of 8 rows
  static_assert(D == 64 || D == 128, "GQA path covers head_dim 64 and 128");
  static_assert(G >= 1 && G <= 8, "GQA path covers groups of 1..8 query heads");

  extern __shared__ __align__(128) unsigned char smem[];
  const GqaSmem Ls = gqa_smem_layout(D, G, p.cand_cap, p.key_cap, p.kmax);
  float* s_score = reinterpret_cast<float*>(smem + Ls.score);
  int* s_sel = reinterpret_cast<int*>(smem + Ls.sel);
  int* s_phys = reinterpret_cast<int*>(smem + Ls.phys);

  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int slot = blockIdx.x / C;
  const int bslot = slot / p.Hkv;
  const int h = slot - bslot * p.Hkv;
  const int b = p.order ? p.order[bslot] : bslot;
  const bool b_ok = b >= 0 && b < p.B;
  const int seq = b_ok ? p.seq_lens[b] : 0;
  const int n = (seq + kPage - 1) / kPage;
  const int unit = b * p.Hkv + h;
  const int64_t orow = ((int64_t)b * p.Hq + (int64_t)h * G);  // first output row of the unit

  auto zero_unit = [&]() {  // skipped unit: defined, recognisable outputs
    if (rank != 0) return;
    if (MODE != kSelect) {
      for (int i = tid; i < G * D; i += NT) p.out[orow * D + i] = __float2bfloat16(0.0f);
      if (p.lse)
        for (int g = tid; g < G; g += NT) p.lse[orow + g] = -INFINITY;
    }
    if (MODE != kDecode && p.sel) {
      for (int j = tid; j < p.kmax; j += NT) p.sel[(int64_t)unit * p.kmax + j] = -1;
      if (tid == 0) p.n_sel[unit] = 0;
    }
  };

  if (!b_ok || seq < 1 || n > p.pt_stride) {
    if (rank == 0 && tid == 0) flag(p.status, b_ok ? VT_DEV_BAD_LEN : kDevBadOrder);
    if (b_ok) zero_unit();
    return;  // uniform over the cluster: every CTA sees the same request
  }
  const int32_t* ptrow = p.page_table + (int64_t)b * p.pt_stride;

  int ns;  // number of selected pages
  if (MODE == kDecode) {
    ns = p.n_sel[unit];
    int bad = (ns < 0 || ns > p.kmax);
    if (!bad)
      for (int j = tid; j < ns; j += NT) {
        const int v = p.sel[(int64_t)unit * p.kmax + j];
        s_sel[j] = v;
        bad |= (v < 0 || v >= n);
      }
    if (__syncthreads_or(bad)) {
      if (rank == 0 && tid == 0) flag(p.status, VT_DEV_BAD_SEL);
      zero_unit();
      return;
    }
  } else if (n <= p.kmax) {  // dense rule: every page
    ns = n;
    for (int j = tid; j < n; j += NT) s_sel[j] = j;
    __syncthreads();
  } else {
    float* s_qm = reinterpret_cast<float*>(smem + Ls.qm);
    int* s_cpage = reinterpret_cast<int*>(smem + Ls.cpage);
    uint32_t* s_key = reinterpret_cast<uint32_t*>(smem + Ls.key);
    int* s_hist = reinterpret_cast<int*>(smem + Ls.misc);
    int* s_small = s_hist + kTopkBins;
    ns = p.kmax;
    const int m = n - p.bos - p.eos;
    const int per = (m + C - 1) / C;
    const int c0 = min(m, rank * per);
    const int cnt = min(m, c0 + per) - c0;
    // 1a. page ids of this CTA's candidates, and the fp32 mean of the group's queries
    int badp = 0;
    for (int i = tid; i < cnt; i += NT) {
      int pg = ptrow[p.bos + c0 + i];
      if (pg < 0 || pg >= p.num_pages) {
        pg = -1;
        badp = 1;
      }
      s_cpage[i] = pg;
    }
    for (int d = tid; d < D; d += NT) {
      float s = 0.0f;
#pragma unroll
      for (int j = 0; j < G; ++j) s += __bfloat162float(p.q[(orow + j) * D + d]);
      s_qm[d] = s / (float)G;
    }
    if (__syncthreads_or(badp) && tid == 0) flag(p.status, VT_DEV_BAD_PAGE);

    // 1b. scores.  Warp w owns rows w, w+NW, ... of this CTA's candidates, in batches of 8;
    //     it keeps kScanSlots-1 batches landing in its own ring (16-byte cp.async, L2 only)
    //     while it reduces the oldest one.  The queries' mean stays in registers.
    float* s_score_w = s_score;
    const int sub = lane / LPR_S, ch = lane % LPR_S;
    const float4 qv = reinterpret_cast<const float4*>(s_qm)[ch];
    const float* cbase = p.centroids + (int64_t)h * D;
    const int64_t cstride = (int64_t)p.Hkv * D;
    const int myrows = (cnt - warp + NW - 1) / NW;   // rows warp + NW*i, i < myrows
    const int batches = (myrows + 7) / 8;
    const uint32_t wring = smem_u32(smem + Ls.ring) + warp * S::WARP_RING;
    auto issue_scan = [&](int bt) {  // 8 rows x (C_ROW / 16) chunks, spread over the lanes
      if (bt < batches) {
        constexpr int CPRS = S::C_ROW / 16;
        const uint32_t dst = wring + (bt % kScanSlots) * S::SCAN_SLOT;
#pragma unroll
        for (int c = lane; c < 8 * CPRS; c += 32) {
          const int t = c / CPRS, kk = c % CPRS;
          const int i = bt * 8 + t;
          const int pg = i < myrows ? s_cpage[warp + NW * i] : -1;
          if (pg >= 0) cp_async16(dst + t * S::C_ROW + kk * 16, cbase + (int64_t)pg * cstride + kk * 4, 16);
        }
      }
      cp_async_commit();
    };
#pragma unroll
    for (int bt = 0; bt < kScanSlots - 1; ++bt) issue_scan(bt);
    for (int bt = 0; bt < batches; ++bt) {
      issue_scan(bt + kScanSlots - 1);
      cp_async_wait<kScanSlots - 1>();
      __syncwarp();  // batch bt is in this warp's ring for every lane
      const uint32_t src = wring + (bt % kScanSlots) * S::SCAN_SLOT;
      float v[SN];
#pragma unroll
      for (int q = 0; q < SN; ++q) {
        const int t = q * RPS + sub;  // row of the batch this lane works on
        float4 c;
        asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];\n"
                     : "=f"(c.x), "=f"(c.y), "=f"(c.z), "=f"(c.w)
                     : "r"(src + t * S::C_ROW + ch * 16));
        float d = c.x * qv.x;
        d = fmaf(c.y, qv.y, d);
        d = fmaf(c.z, qv.z, d);
        v[q] = fmaf(c.w, qv.w, d);
      }
      exchange_reduce<SN, LPR_S>(v, lane);
      const int i = bt * 8 + exchange_index<SN, LPR_S>(lane) * RPS + sub;
      if ((ch % (LPR_S / SN)) == 0 && i < myrows) {
        const int row = warp + NW * i;
        s_score_w[row] = s_cpage[row] >= 0 ? v[0] : -INFINITY;
      }
      __syncwarp();  // every lane is done with the slot before it is refilled
    }
    cp_async_wait<0>();
    __syncthreads();  // the ring is free again (keys of the selection may overlap it)
    cluster.sync();  // #1: every CTA's scores are visible cluster-wide

    // 2. every CTA selects from all the unit's scores (same input -> same result)
    for (int j = tid; j < m; j += NT) {
      const int r = j / per;
      s_key[j] = score_key(cluster.map_shared_rank(s_score, r)[j - r * per]);
    }
    for (int j = tid; j < p.bos; j += NT) s_sel[j] = j;
    for (int j = tid; j < p.eos; j += NT) s_sel[p.bos + p.topk + j] = n - p.eos + j;
    __syncthreads();
    const int bos = p.bos, topk = p.topk;
    auto put = [&](int j, int pos) {
      if (pos < topk) s_sel[bos + pos] = bos + j;  // exactly topk are emitted; guard anyway
    };
    if (p.approx) {
      const int start = (int)(splitmix64(p.seed + (uint64_t)unit) % (uint64_t)m);
      approx_topk<NT>(s_key, m, topk, start, s_hist, s_small, put);
    } else {
      block_topk<NT>(s_key, m, topk, s_hist, s_small, put);
    }
  }
  if (MODE != kDecode && rank == 0 && p.sel) {
    for (int j = tid; j < p.kmax; j += NT)
      p.sel[(int64_t)unit * p.kmax + j] = j < ns ? s_sel[j] : -1;
    if (tid == 0) p.n_sel[unit] = ns;
  }
  if (MODE == kSelect) {
    if (n > p.kmax) cluster.sync();  // peers may still be reading this CTA's scores
    return;
  }

  // 3. attention over this CTA's share of the selected pages, one page per warp at a time
  {
    int badp = 0;
    for (int j = tid; j < ns; j += NT) {
      int pg = ptrow[s_sel[j]];
      if (pg < 0 || pg >= p.num_pages) {
        pg = -1;
        badp = 1;
      }
      s_phys[j] = pg;
    }
    if (__syncthreads_or(badp) && rank == 0 && tid == 0) flag(p.status, VT_DEV_BAD_PAGE);
  }
  const int j0 = (rank * ns) / C, j1 = ((rank + 1) * ns) / C;
  const int last_valid = seq - kPage * (n - 1);
  const int npw = (j1 - j0 - warp + NW - 1) / NW;  // pages of this warp: j0 + warp + NW i
  const uint32_t ring = smem_u32(smem + Ls.ring) + warp * S::WARP_RING;

  // one page (16 K rows and 16 V rows of head h) into slot i % kGqaSlots; rows past the end
  // of the request (or of an unusable page) are zero-filled instead of read
  auto rows_of = [&](int j) { return s_phys[j] < 0 ? 0 : (s_sel[j] == n - 1 ? last_valid : kPage); };
  auto issue = [&](int i) {
    if (i < npw) {
      const int j = j0 + warp + NW * i;
      const int64_t pg = s_phys[j] < 0 ? 0 : s_phys[j];
      stage_page<D>(ring + (i % kGqaSlots) * S::SLOT, p.k_pool + pg * p.sk_p + (int64_t)h * p.sk_h,
                    p.v_pool + pg * p.sv_p + (int64_t)h * p.sv_h, p.sk_t, p.sv_t, rows_of(j),
                    p.k_pool, lane);
    }
    cp_async_commit();
  };
#pragma unroll
  for (int i = 0; i < kGqaSlots - 1; ++i) issue(i);
  WarpAttention<D, G> att;
  att.init(p.q + orow * D, lane);
  for (int i = 0; i < npw; ++i) {
    issue(i + kGqaSlots - 1);
    cp_async_wait<kGqaSlots - 1>();
    __syncwarp();  // page i is in this warp's slot for every lane
    att.page(ring + (i % kGqaSlots) * S::SLOT, rows_of(j0 + warp + NW * i), p.qscale);
    __syncwarp();  // every lane is done with slot i before a later issue refills it
  }
  cp_async_wait<0>();
  __syncthreads();  // all warps are out of their slots: the combine area may reuse them

  float* s_warp = reinterpret_cast<float*>(smem + Ls.warp);  // [NW][G][D+2]: acc, m, l
  float* s_cta = reinterpret_cast<float*>(smem + Ls.cta);    // [G][D+2]
  att.store(s_warp + warp * G * (D + 2), lane);
  __syncthreads();
  merge_partials<G, D>(s_warp, NW, s_cta, tid, NT);
  cluster.sync();  // #2: every CTA's partial is visible (and every score has been read)

  // 4. each CTA finalises a 1/C slice of the unit's G x D outputs
  {
    const int total = G * D;
    const int per = (total + C - 1) / C;
    const int i1 = min(total, (rank + 1) * per);
    for (int idx = rank * per + tid; idx < i1; idx += NT) {
      const int gg = idx / D, d = idx - gg * D;
      float M = -INFINITY;
      for (int r = 0; r < C; ++r)
        M = fmaxf(M, cluster.map_shared_rank(s_cta, r)[gg * (D + 2) + D]);
      float A = 0.0f, Lsum = 0.0f;
      for (int r = 0; r < C; ++r) {
        const float* pc = cluster.map_shared_rank(s_cta, r) + gg * (D + 2);
        const float mr = pc[D];
        const float f = (mr == -INFINITY) ? 0.0f : exp2f(mr - M);
        A = fmaf(pc[d], f, A);
        Lsum = fmaf(pc[D + 1], f, Lsum);
      }
      p.out[(orow + gg) * D + d] = __float2bfloat16(Lsum > 0.0f ? A / Lsum : 0.0f);
      if (d == 0 && p.lse) p.lse[orow + gg] = Lsum > 0.0f ? (M + log2f(Lsum)) * kLn2 : -INFINITY;
    }
  }
  cluster.sync();  // #3: peers may still be reading this CTA's partial
}

// ---------------------------------------------------------------------------------------
// host-side launch
// ---------------------------------------------------------------------------------------

template <int D, int G, int MODE>
static cudaError_t launch_gqa_t(const DecodeParams& p, int C, cudaStream_t stream) {
  auto kern = gqa_decode_kernel<D, G, MODE>;
  const GqaSmem L = gqa_smem_layout(D, G, p.cand_cap, p.key_cap, p.kmax);
  static std::atomic<int> optin[64];
  cudaError_t e = ensure_smem_optin(kern, L.total, C > 8, optin);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((int64_t)C * p.B * p.Hkv), 1, 1);
  cfg.blockDim = dim3(kGqaThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)L.total;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int D, int MODE>
static cudaError_t dispatch_g(const DecodeParams& p, int G, int C, cudaStream_t s) {
  switch (G) {
    case 1: return launch_gqa_t<D, 1, MODE>(p, C, s);
    case 2: return launch_gqa_t<D, 2, MODE>(p, C, s);
    case 3: return launch_gqa_t<D, 3, MODE>(p, C, s);
    case 4: return launch_gqa_t<D, 4, MODE>(p, C, s);
    case 5: return launch_gqa_t<D, 5, MODE>(p, C, s);
    case 6: return launch_gqa_t<D, 6, MODE>(p, C, s);
    case 7: return launch_gqa_t<D, 7, MODE>(p, C, s);
    case 8: return launch_gqa_t<D, 8, MODE>(p, C, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int MODE>
static cudaError_t dispatch_d(const DecodeParams& p, int D, int G, int C, cudaStream_t s) {
  if (D == 64) return dispatch_g<64, MODE>(p, G, C, s);
  if (D == 128) return dispatch_g<128, MODE>(p, G, C, s);
  return cudaErrorInvalidValue;
}

int gqa_smem_bytes(int D, int G, int cand_cap, int key_cap, int kmax) {
  return gqa_smem_layout(D, G, cand_cap, key_cap, kmax).total;
}

cudaError_t launch_gqa_decode(const DecodeParams& p, int mode, int D, int G, int C,
                              cudaStream_t s) {
  switch (mode) {
    case kSelect: return dispatch_d<kSelect>(p, D, G, C, s);
    case kDecode: return dispatch_d<kDecode>(p, D, G, C, s);
    case kFused: return dispatch_d<kFused>(p, D, G, C, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace vt
