// decode_fma.cu -- query side of block top-k sparse decode on CUDA cores (head_dim 64/128,
// GQA group G <= 8): group-mean query, GeMV against the page centroids, exact top-k with the
// reserved first/last pages, and exact softmax attention over the selected pages.
//
// Sources: "Vortex: A Flexible and Efficient Sparse Attention Framework" (vortex_torch
// README), "Quick Example" (forward_indexer: q.mean -> GeMV -> topK) and "Using Your Sparse
// Attention with SGLang" (page size 16, vortex_topk_val, reserved bos/eos pages); "Vortex:
// Efficient and Programmable Sparse Attention Serving for AI Agents", "A dual-stage
// programmable abstraction" (query-dependent scoring, top-k block selection, attention over
// the paged layout; kernel fusion).
//
// One thread-block cluster of C CTAs serves one (request, KV head) unit:
//   1. every CTA scores a contiguous 1/C of the middle pages: it loads their page-table
//      entries, then streams their fp32 centroid rows (one float4 per lane, several rows in
//      flight per warp) and dots them with the fp32 group mean of the unit's G query heads;
//   2. rank 0 gathers all scores over DSMEM and runs an exact radix select (8-bit digits,
//      ties -> lower logical page), then adds the reserved pages; the others copy the
//      ascending selection from rank 0 over DSMEM;
//   3. CTA r attends to its 1/C of the selected pages: LPR lanes share one 16-byte slice of
//      a K/V row each, every stream of LPR lanes walks its own tokens with an online softmax
//      (base-2 exponent, fp32), streams merge by shuffles, warps through shared memory;
//   4. the C partial (max, sum, acc) triples are combined over DSMEM, each CTA producing
//      1/C of the unit's G x Dv outputs (and lse).
// A request with n <= topk+bos+eos pages skips 1-2 and attends to every page.  The tensor
// cores are not used: with G <= 8 query rows per KV head there is no MMA-sized tile.
#include "decode_params.cuh"

namespace vt {

constexpr int kFmaThreads = 128;

template <int D, int G, int MODE>
__global__ void __launch_bounds__(kFmaThreads) fma_decode_kernel(const DecodeParams p) {
  constexpr int NT = kFmaThreads;
  constexpr int NW = NT / 32;
  constexpr int LPR = D / 8;        // lanes per K/V row: 8 bf16 (16 bytes) each
  constexpr int RPW = 32 / LPR;     // rows a warp covers per step
  constexpr int NS = NW * RPW;      // independent token streams in a CTA
  constexpr int LPR_S = D / 4;      // lanes per fp32 centroid row: one float4 each
  constexpr int RPW_S = 32 / LPR_S;
  constexpr int U = (G <= 4) ? 4 : 2;  // tokens per stream per step (loads in flight)
  constexpr int US = 8;                // centroid rows per lane group per step
  static_assert(D == 64 || D == 128, "CUDA-core path covers head_dim 64 and 128");

  extern __shared__ __align__(16) unsigned char smem[];
  const FmaSmem Ls = fma_smem_layout(D, G, NW, p.cand_cap, p.key_cap, p.kmax);
  float* s_qm = reinterpret_cast<float*>(smem + Ls.qm);
  int* s_cpage = reinterpret_cast<int*>(smem + Ls.cpage);
  float* s_score = reinterpret_cast<float*>(smem + Ls.score);
  uint32_t* s_key = reinterpret_cast<uint32_t*>(smem + Ls.key);
  int* s_sel = reinterpret_cast<int*>(smem + Ls.sel);
  int* s_phys = reinterpret_cast<int*>(smem + Ls.phys);
  float* s_warp = reinterpret_cast<float*>(smem + Ls.warp);  // [NW][G][D+2]: acc, m, l
  float* s_cta = reinterpret_cast<float*>(smem + Ls.cta);    // [G][D+2]
  int* s_misc = reinterpret_cast<int*>(smem + Ls.misc);
  int* s_hist = s_misc;         // 256
  int* s_info = s_misc + 256;   // 4
  int* s_scan = s_misc + 264;   // 32

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
  } else {
    if (n <= p.kmax) {  // dense rule: every page
      ns = n;
      for (int j = tid; j < n; j += NT) s_sel[j] = j;
    } else {
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
      // 1b. scores: qm . centroid, LPR_S lanes per row, US rows per lane group in flight
      {
        const int sub = lane / LPR_S, ch = lane % LPR_S;
        const float4 qv = reinterpret_cast<const float4*>(s_qm)[ch];
        const float* cbase = p.centroids + (int64_t)h * D + ch * 4;
        const int64_t cstride = (int64_t)p.Hkv * D;
        constexpr int STEP = NW * RPW_S;
        for (int r0 = warp * RPW_S + sub; r0 - sub < cnt; r0 += STEP * US) {
          float4 c[US];
#pragma unroll
          for (int u = 0; u < US; ++u) {
            const int r = r0 + u * STEP;
            const int pg = (r < cnt) ? s_cpage[r] : -1;
            c[u] = (pg >= 0) ? ld_stream_f4(cbase + (int64_t)pg * cstride)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int u = 0; u < US; ++u) {
            float d = c[u].x * qv.x;
            d = fmaf(c[u].y, qv.y, d);
            d = fmaf(c[u].z, qv.z, d);
            d = fmaf(c[u].w, qv.w, d);
#pragma unroll
            for (int o = LPR_S / 2; o >= 1; o >>= 1) d += __shfl_xor_sync(kFull, d, o);
            const int r = r0 + u * STEP;
            if (ch == 0 && r < cnt) s_score[r] = (s_cpage[r] >= 0) ? d : -INFINITY;
          }
        }
      }
      cluster.sync();  // #1: every CTA's scores are visible cluster-wide
      if (rank == 0) {
        for (int j = tid; j < m; j += NT) {
          const int r = j / per;
          const float* ps = cluster.map_shared_rank(s_score, r);
          s_key[j] = score_key(ps[j - r * per]);
        }
        for (int j = tid; j < p.bos; j += NT) s_sel[j] = j;
        for (int j = tid; j < p.eos; j += NT) s_sel[p.bos + p.topk + j] = n - p.eos + j;
        __syncthreads();
        if (p.topk > 0) {
          uint32_t prefix, mask;
          int need;
          bool take_all;
          radix_select<NT>(s_key, m, p.topk, s_hist, s_info, prefix, mask, need, take_all);
          const int bos = p.bos, topk = p.topk;
          emit_topk<NT>(s_key, m, prefix, mask, need, take_all, s_scan, [&](int j, int pos) {
            if (pos < topk) s_sel[bos + pos] = bos + j;  // exactly topk emitted; guard anyway
          });
        }
      }
      cluster.sync();  // #2: the selection in rank 0 is complete; peers' scores are dead
      if (rank != 0) {
        const int* r0sel = cluster.map_shared_rank(s_sel, 0);
        for (int j = tid; j < ns; j += NT) s_sel[j] = r0sel[j];
      }
    }
    __syncthreads();
    if (rank == 0 && (MODE == kSelect || p.sel)) {
      for (int j = tid; j < p.kmax; j += NT)
        p.sel[(int64_t)unit * p.kmax + j] = j < ns ? s_sel[j] : -1;
      if (tid == 0) p.n_sel[unit] = ns;
    }
    if (MODE == kSelect) return;
  }

  // 3. attention over this CTA's share of the selected pages
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
  const int ntok = (j1 - j0) * kPage;
  const int last_valid = seq - kPage * (n - 1);
  const int stream = warp * RPW + lane / LPR;
  const int ch = lane % LPR;

  float qr[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint4 raw = *reinterpret_cast<const uint4*>(p.q + (orow + g) * D + ch * 8);
    unpack8(raw, qr[g]);
#pragma unroll
    for (int i = 0; i < 8; ++i) qr[g][i] *= p.qscale;
  }
  float m[G], l[G], acc[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[g][i] = 0.0f;
  }
  const __nv_bfloat16* kb = p.k_pool + (int64_t)h * p.sk_h + ch * 8;
  const __nv_bfloat16* vb = p.v_pool + (int64_t)h * p.sv_h + ch * 8;

  // the loop bound is uniform over the warp (shuffles below), each lane offsets by its stream
  for (int base = warp * RPW; base < ntok; base += NS * U) {
    const int t0 = base + (stream - warp * RPW);
    uint4 kr[U], vr[U];
    bool ok[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int tau = t0 + u * NS;
      ok[u] = false;
      if (tau < ntok) {
        const int j = j0 + (tau >> 4), t = tau & 15;
        const int pg = s_phys[j];
        ok[u] = pg >= 0 && (s_sel[j] != n - 1 || t < last_valid);
        if (ok[u]) {
          kr[u] = ld_stream_u4(kb + (int64_t)pg * p.sk_p + (int64_t)t * p.sk_t);
          vr[u] = ld_stream_u4(vb + (int64_t)pg * p.sv_p + (int64_t)t * p.sv_t);
        }
      }
      if (!ok[u]) kr[u] = vr[u] = make_uint4(0, 0, 0, 0);
    }
    float s[U][G];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float kf[8];
      unpack8(kr[u], kf);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float d = qr[g][0] * kf[0];
#pragma unroll
        for (int i = 1; i < 8; ++i) d = fmaf(qr[g][i], kf[i], d);
        s[u][g] = d;
      }
    }
#pragma unroll
    for (int o = LPR / 2; o >= 1; o >>= 1)
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int g = 0; g < G; ++g) s[u][g] += __shfl_xor_sync(kFull, s[u][g], o);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float mx = m[g];
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (ok[u]) mx = fmaxf(mx, s[u][g]);
      if (mx != -INFINITY && mx != m[g]) {
        const float corr = exp2f(m[g] - mx);
        l[g] *= corr;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[g][i] *= corr;
        m[g] = mx;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (!ok[u]) continue;
      float vf[8];
      unpack8(vr[u], vf);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float pr = exp2f(s[u][g] - m[g]);
        l[g] += pr;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[g][i] = fmaf(pr, vf[i], acc[g][i]);
      }
    }
  }

  // merge the RPW streams of each warp (lanes LPR apart hold the same dims)
#pragma unroll
  for (int o = LPR; o < 32; o <<= 1) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float mo = __shfl_xor_sync(kFull, m[g], o);
      const float lo = __shfl_xor_sync(kFull, l[g], o);
      float M, fa, fb;
      merge_scale(m[g], mo, M, fa, fb);
      l[g] = l[g] * fa + lo * fb;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float ao = __shfl_xor_sync(kFull, acc[g][i], o);
        acc[g][i] = acc[g][i] * fa + ao * fb;
      }
      m[g] = M;
    }
  }
  if (lane < LPR) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float* w = s_warp + (warp * G + g) * (D + 2);
#pragma unroll
      for (int i = 0; i < 8; ++i) w[ch * 8 + i] = acc[g][i];
      if (lane == 0) {
        w[D] = m[g];
        w[D + 1] = l[g];
      }
    }
  }
  __syncthreads();
  for (int idx = tid; idx < G * D; idx += NT) {
    const int g = idx / D, d = idx - g * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, s_warp[(w * G + g) * (D + 2) + D]);
    float A = 0.0f, Lsum = 0.0f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float* pw = s_warp + (w * G + g) * (D + 2);
      const float f = (pw[D] == -INFINITY) ? 0.0f : exp2f(pw[D] - M);
      A = fmaf(pw[d], f, A);
      Lsum = fmaf(pw[D + 1], f, Lsum);
    }
    s_cta[g * (D + 2) + d] = A;
    if (d == 0) {
      s_cta[g * (D + 2) + D] = M;
      s_cta[g * (D + 2) + D + 1] = Lsum;
    }
  }
  cluster.sync();  // #3: every CTA's partial is visible cluster-wide

  // 4. each CTA finalises a 1/C slice of the unit's G x D outputs
  {
    const int total = G * D;
    const int per = (total + C - 1) / C;
    const int i1 = min(total, (rank + 1) * per);
    for (int idx = rank * per + tid; idx < i1; idx += NT) {
      const int g = idx / D, d = idx - g * D;
      float M = -INFINITY;
      for (int r = 0; r < C; ++r)
        M = fmaxf(M, cluster.map_shared_rank(s_cta, r)[g * (D + 2) + D]);
      float A = 0.0f, Lsum = 0.0f;
      for (int r = 0; r < C; ++r) {
        const float* pc = cluster.map_shared_rank(s_cta, r) + g * (D + 2);
        const float mr = pc[D];
        const float f = (mr == -INFINITY) ? 0.0f : exp2f(mr - M);
        A = fmaf(pc[d], f, A);
        Lsum = fmaf(pc[D + 1], f, Lsum);
      }
      p.out[(orow + g) * D + d] = __float2bfloat16(Lsum > 0.0f ? A / Lsum : 0.0f);
      if (d == 0 && p.lse) p.lse[orow + g] = Lsum > 0.0f ? (M + log2f(Lsum)) * kLn2 : -INFINITY;
    }
  }
  cluster.sync();  // #4: peers may still be reading this CTA's partial
}

// ---------------------------------------------------------------------------------------
// host-side launch
// ---------------------------------------------------------------------------------------

template <int D, int G, int MODE>
static cudaError_t launch_fma_t(const DecodeParams& p, int C, cudaStream_t stream) {
  auto kern = fma_decode_kernel<D, G, MODE>;
  const FmaSmem L = fma_smem_layout(D, G, kFmaThreads / 32, p.cand_cap, p.key_cap, p.kmax);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
  if (e != cudaSuccess) return e;
  if (C > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((int64_t)C * p.B * p.Hkv), 1, 1);
  cfg.blockDim = dim3(kFmaThreads, 1, 1);
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
    case 1: return launch_fma_t<D, 1, MODE>(p, C, s);
    case 2: return launch_fma_t<D, 2, MODE>(p, C, s);
    case 3: return launch_fma_t<D, 3, MODE>(p, C, s);
    case 4: return launch_fma_t<D, 4, MODE>(p, C, s);
    case 5: return launch_fma_t<D, 5, MODE>(p, C, s);
    case 6: return launch_fma_t<D, 6, MODE>(p, C, s);
    case 7: return launch_fma_t<D, 7, MODE>(p, C, s);
    case 8: return launch_fma_t<D, 8, MODE>(p, C, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int MODE>
static cudaError_t dispatch_d(const DecodeParams& p, int D, int G, int C, cudaStream_t s) {
  if (D == 64) return dispatch_g<64, MODE>(p, G, C, s);
  if (D == 128) return dispatch_g<128, MODE>(p, G, C, s);
  return cudaErrorInvalidValue;
}

int fma_smem_bytes(int D, int G, int cand_cap, int key_cap, int kmax) {
  return fma_smem_layout(D, G, kFmaThreads / 32, cand_cap, key_cap, kmax).total;
}

cudaError_t launch_fma_decode(const DecodeParams& p, int mode, int D, int G, int C,
                              cudaStream_t s) {
  switch (mode) {
    case kSelect: return dispatch_d<kSelect>(p, D, G, C, s);
    case kDecode: return dispatch_d<kDecode>(p, D, G, C, s);
    case kFused: return dispatch_d<kFused>(p, D, G, C, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace vt
