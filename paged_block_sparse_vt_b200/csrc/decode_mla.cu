// decode_mla.cu -- block top-k sparse decode for the MLA latent form: one shared latent KV
// head per token (K row = [latent 512 ; rope 64] bf16, V = the latent part of the same row),
// 16 or 32 absorbed query heads of 576 dims.
//
// Sources: "Vortex: Efficient and Programmable Sparse Attention Serving for AI Agents"
// (rndamp.com), section "Speedups that scale to 229B parameters" (a rope-aware block sparse
// attention for the MLA-based GLM-4.7-Flash) and the thread on digg.com, part [4/6] (MLA
// squeezes the KV cache into one shared latent; a rope-aware block sparse attention was
// written for it); the flow itself as in the vortex_torch README "Quick Example".
// Rope-aware scoring q_lat . c_lat + q_rope . c_rope equals one dot product over the
// 576-dim row because the page mean is linear in each part.
//
// Same cluster-per-request structure as the CUDA-core path (score -> DSMEM top-k ->
// attention -> DSMEM combine), but with G >= 16 query heads sharing every K/V row the
// attention is a real contraction and runs on the tensor cores (mma.sync m16n8k16 bf16 ->
// fp32):
//   S^T[tokens x heads] = K_tile[tokens x 576] . Q^T   (one warp per page of 16 tokens)
//   P = softmax over the CTA's tokens (fp32, base 2), rounded to bf16
//   O[heads x 512]     = P[heads x tokens] . V_tile   (each warp owns 64 output dims)
// The CTA's K tiles are copied once into shared memory (cp.async, zero-filled past the end
// of the request) and serve as both the K operand and, through a transposed ldmatrix, the
// V operand.
#include "decode_params.cuh"
#include "topk.cuh"

namespace vt {

constexpr int kMlaThreads = 256;
constexpr int kMlaD = 576;
constexpr int kMlaDv = 512;
constexpr int kMlaRow = kMlaD + 8;  // smem row stride (elements): 1168 B, ldmatrix conflict-free
constexpr int kMlaMaxPages = 8;     // pages one CTA attends to (one warp per page)
constexpr int kMlaScanRows = 2;     // centroid rows per ring slot (2 x 2304 B)
constexpr int kMlaScanSlots = 4;    // ring slots per warp: 3 batches landing while one is used
constexpr int kMlaRingBytes = (kMlaThreads / 32) * kMlaScanSlots * kMlaScanRows * kMlaD * 4;

struct MlaSmem {
  int sel, phys, misc;               // persistent
  int qm, cpage, score, key, ring;   // selection phase
  int q, kt, st, pm, ml;             // attention phase (aliases the selection phase)
  int total;
};

__host__ __device__ inline MlaSmem mla_smem_layout(int G, int cand_cap, int key_cap, int kmax,
                                                   int ppc) {
  MlaSmem s;
  int o = 0;
  s.sel = o;  o += align16(kmax * 4);
  s.phys = o; o += align16(kmax * 4);
  s.misc = o; o += align16((kTopkBins + 64) * 4);
  const int base = o;
  int a = base;  // selection phase
  s.qm = a;    a += align16(kMlaD * 4);
  s.cpage = a; a += align16(cand_cap * 4);
  s.score = a; a += align16(cand_cap * 4);
  s.key = a;   a += align16(key_cap * 4);
  s.ring = a;  a += kMlaRingBytes;  // per-warp cp.async rings of centroid rows
  int b = base;  // attention phase
  const int T = ppc * kPage;
  s.q = b;  b += align16(G * kMlaRow * 2);
  s.kt = b;
  const int kt_bytes = T * kMlaRow * 2;
  const int o_bytes = G * (kMlaDv + 2) * 4;  // CTA partial (aliases the K tiles)
  b += align16(kt_bytes > o_bytes ? kt_bytes : o_bytes);
  s.st = b; b += align16(T * (G + 1) * 4);
  s.pm = b; b += align16(G * (T + 8) * 2);
  s.ml = b; b += align16(G * 2 * 4);
  s.total = a > b ? a : b;
  return s;
}

template <int G, int MODE>
__global__ void __launch_bounds__(kMlaThreads, 1) mla_decode_kernel(const DecodeParams p) {
  constexpr int NT = kMlaThreads;
  constexpr int NW = NT / 32;
  constexpr int D = kMlaD, DV = kMlaDv;
  constexpr int CH = D / 4;  // float4 per centroid row (144)
  static_assert(G == 16 || G == 32, "MLA path: 16 or 32 query heads");

  extern __shared__ __align__(16) unsigned char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ppc = (p.kmax + C - 1) / C;
  const MlaSmem Ls = mla_smem_layout(G, p.cand_cap, p.key_cap, p.kmax, ppc);
  int* s_sel = reinterpret_cast<int*>(smem + Ls.sel);
  int* s_phys = reinterpret_cast<int*>(smem + Ls.phys);
  int* s_hist = reinterpret_cast<int*>(smem + Ls.misc);  // kTopkBins
  int* s_small = s_hist + kTopkBins;                      // 64

  const int bslot = blockIdx.x / C;  // Hkv == 1: one unit per request
  const int b = p.order ? p.order[bslot] : bslot;
  const bool b_ok = b >= 0 && b < p.B;
  const int seq = b_ok ? p.seq_lens[b] : 0;
  const int n = (seq + kPage - 1) / kPage;
  const int unit = b;
  const int64_t orow = (int64_t)b * p.Hq;

  auto zero_unit = [&]() {
    if (rank != 0) return;
    if (MODE != kSelect) {
      for (int i = tid; i < G * DV; i += NT) p.out[orow * DV + i] = __float2bfloat16(0.0f);
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
    return;
  }
  const int32_t* ptrow = p.page_table + (int64_t)b * p.pt_stride;

  int ns;
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
    if (n <= p.kmax) {
      ns = n;
      for (int j = tid; j < n; j += NT) s_sel[j] = j;
    } else {
      ns = p.kmax;
      float* s_qm = reinterpret_cast<float*>(smem + Ls.qm);
      int* s_cpage = reinterpret_cast<int*>(smem + Ls.cpage);
      float* s_score = reinterpret_cast<float*>(smem + Ls.score);
      uint32_t* s_key = reinterpret_cast<uint32_t*>(smem + Ls.key);
      const int m = n - p.bos - p.eos;
      const int per = (m + C - 1) / C;
      const int c0 = min(m, rank * per);
      const int cnt = min(m, c0 + per) - c0;
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
        for (int j = 0; j < G; ++j) s += __bfloat162float(p.q[(orow + j) * D + d]);
        s_qm[d] = s / (float)G;
      }
      if (__syncthreads_or(badp) && tid == 0) flag(p.status, VT_DEV_BAD_PAGE);
      {
        // Warp w scores rows w + NW i of the CTA's candidates: the fp32 centroid rows stream
        // through the warp's ring of kMlaScanSlots slots of kMlaScanRows rows (cp.async, three
        // slots landing while one is used); float4 chunk c = lane + 32 i of a row (i < 5, the
        // 5th only for lanes < 16) is dotted with the same chunk of the group mean.
        float4 qv[5];
#pragma unroll
        for (int i = 0; i < 5; ++i) {
          const int c = lane + 32 * i;
          qv[i] = c < CH ? reinterpret_cast<const float4*>(s_qm)[c] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        constexpr int RB = D * 4;  // bytes of a centroid row
        const uint32_t ring = smem_u32(smem + Ls.ring) + warp * kMlaScanSlots * kMlaScanRows * RB;
        const int myrows = (cnt - warp + NW - 1) / NW;
        const int nb = (myrows + kMlaScanRows - 1) / kMlaScanRows;
        auto issue = [&](int bt) {
          if (bt < nb) {
            const uint32_t dst = ring + (bt % kMlaScanSlots) * kMlaScanRows * RB;
#pragma unroll
            for (int rr = 0; rr < kMlaScanRows; ++rr) {
              const int i = bt * kMlaScanRows + rr;
              const int pg = i < myrows ? s_cpage[warp + NW * i] : -1;
              if (pg >= 0) {
                const float* row = p.centroids + (int64_t)pg * D;
                for (int c = lane; c < CH; c += 32) cp_async16(dst + rr * RB + c * 16, row + 4 * c, 16);
              }
            }
          }
          cp_async_commit();
        };
#pragma unroll
        for (int bt = 0; bt < kMlaScanSlots - 1; ++bt) issue(bt);
        for (int bt = 0; bt < nb; ++bt) {
          issue(bt + kMlaScanSlots - 1);
          cp_async_wait<kMlaScanSlots - 1>();
          __syncwarp();
          const uint32_t src = ring + (bt % kMlaScanSlots) * kMlaScanRows * RB;
#pragma unroll
          for (int rr = 0; rr < kMlaScanRows; ++rr) {
            float d = 0.0f;
#pragma unroll
            for (int i = 0; i < 5; ++i) {
              const int c = lane + 32 * i;
              if (c < CH) {
                float4 cv;
                asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];\n"
                             : "=f"(cv.x), "=f"(cv.y), "=f"(cv.z), "=f"(cv.w)
                             : "r"(src + rr * RB + c * 16));
                d = fmaf(cv.x, qv[i].x, d);
                d = fmaf(cv.y, qv[i].y, d);
                d = fmaf(cv.z, qv[i].z, d);
                d = fmaf(cv.w, qv[i].w, d);
              }
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) d += __shfl_xor_sync(kFull, d, o);
            const int i = bt * kMlaScanRows + rr;
            if (lane == 0 && i < myrows) {
              const int r = warp + NW * i;
              s_score[r] = (s_cpage[r] >= 0) ? d : -INFINITY;
            }
          }
          __syncwarp();  // every lane is done with the slot before it is refilled
        }
        cp_async_wait<0>();
      }
      cluster.sync();  // #1
      if (rank == 0) {
        for (int j = tid; j < m; j += NT) {
          const int r = j / per;
          const float* ps = cluster.map_shared_rank(s_score, r);
          s_key[j] = score_key(ps[j - r * per]);
        }
        for (int j = tid; j < p.bos; j += NT) s_sel[j] = j;
        for (int j = tid; j < p.eos; j += NT) s_sel[p.bos + p.topk + j] = n - p.eos + j;
        __syncthreads();
        const int bos = p.bos, topk = p.topk;
        auto put = [&](int j, int pos) {
          if (pos < topk) s_sel[bos + pos] = bos + j;  // exactly topk are emitted
        };
        if (p.approx) {
          const int start = (int)(splitmix64(p.seed + (uint64_t)unit) % (uint64_t)m);
          approx_topk<NT>(s_key, m, topk, start, s_hist, s_small, put);
        } else {
          block_topk<NT>(s_key, m, topk, s_hist, s_small, put);
        }
      }
      cluster.sync();  // #2
      // Only the attending modes need the selection in every CTA.  In kSelect mode rank 0
      // returns right after writing it out, so nobody may touch its shared memory here.
      if (MODE != kSelect && rank != 0) {
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

  // ---- attention on the tensor cores ----------------------------------------------------
  __nv_bfloat16* s_q = reinterpret_cast<__nv_bfloat16*>(smem + Ls.q);
  __nv_bfloat16* s_kt = reinterpret_cast<__nv_bfloat16*>(smem + Ls.kt);
  float* s_o = reinterpret_cast<float*>(smem + Ls.kt);  // after P.V: CTA partial [G][DV+2]
  float* s_st = reinterpret_cast<float*>(smem + Ls.st);  // [T][G+1] scaled scores
  __nv_bfloat16* s_pm = reinterpret_cast<__nv_bfloat16*>(smem + Ls.pm);  // [G][T+8]
  float* s_ml = reinterpret_cast<float*>(smem + Ls.ml);  // [G][2]
  const int j0 = (rank * ns) / C, j1 = ((rank + 1) * ns) / C;
  const int np = j1 - j0;  // pages of this CTA (<= ppc)
  const int T = ppc * kPage;
  const int PST = T + 8;
  const int last_valid = seq - kPage * (n - 1);
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
  // stage Q (G x 576) and the K tiles of this CTA's pages (zero rows past the valid tokens)
  for (int i = tid; i < G * (D / 8); i += NT) {
    const int g = i / (D / 8), c = i - g * (D / 8);
    cp_async16(smem_u32(s_q + g * kMlaRow + c * 8), p.q + (orow + g) * D + c * 8, 16);
  }
  for (int i = tid; i < np * kPage * (D / 8); i += NT) {
    const int row = i / (D / 8), c = i - row * (D / 8);
    const int jj = row >> 4, t = row & 15;
    const int pg = s_phys[j0 + jj];
    const bool valid = pg >= 0 && (s_sel[j0 + jj] != n - 1 || t < last_valid);
    const __nv_bfloat16* src =
        valid ? p.k_pool + (int64_t)pg * p.sk_p + (int64_t)t * p.sk_t + c * 8 : p.k_pool;
    cp_async16(smem_u32(s_kt + row * kMlaRow + c * 8), src, valid ? 16 : 0);
  }
  cp_async_commit();
  cp_async_wait_all();
  __syncthreads();

  // S^T = K Q^T: warp w owns page w (16 tokens) x all G heads
  if (warp < np) {
    float acc[G / 8][4];
#pragma unroll
    for (int nt = 0; nt < G / 8; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[nt][i] = 0.0f;
    const uint32_t a_base =
        smem_u32(s_kt + (warp * 16 + (lane & 15)) * kMlaRow + (lane >> 4) * 8);
    const uint32_t b_base =
        smem_u32(s_q + ((lane & 7) + ((lane >> 4) << 3)) * kMlaRow + ((lane >> 3) & 1) * 8);
#pragma unroll 4
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(a_base + ks * 32, a0, a1, a2, a3);
#pragma unroll
      for (int n2 = 0; n2 < G / 16; ++n2) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(b_base + n2 * 16 * kMlaRow * 2 + ks * 32, b0, b1, b2, b3);
        mma_16816(acc[2 * n2], a0, a1, a2, a3, b0, b1);
        mma_16816(acc[2 * n2 + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    const int r = warp * 16 + (lane >> 2);
#pragma unroll
    for (int nt = 0; nt < G / 8; ++nt) {
      const int c = nt * 8 + 2 * (lane & 3);
      s_st[r * (G + 1) + c] = acc[nt][0] * p.qscale;
      s_st[r * (G + 1) + c + 1] = acc[nt][1] * p.qscale;
      s_st[(r + 8) * (G + 1) + c] = acc[nt][2] * p.qscale;
      s_st[(r + 8) * (G + 1) + c + 1] = acc[nt][3] * p.qscale;
    }
  }
  __syncthreads();

  // softmax over this CTA's tokens, per head (warp w: heads w, w+NW, ...)
  for (int g = warp; g < G; g += NW) {
    float mx = -INFINITY;
    for (int t = lane; t < np * kPage; t += 32) {
      const int jj = t >> 4, tt = t & 15;
      const bool valid = s_phys[j0 + jj] >= 0 && (s_sel[j0 + jj] != n - 1 || tt < last_valid);
      if (valid) mx = fmaxf(mx, s_st[t * (G + 1) + g]);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
    float sum = 0.0f;
    for (int t = lane; t < T; t += 32) {
      const int jj = t >> 4, tt = t & 15;
      const bool valid = t < np * kPage && s_phys[j0 + jj] >= 0 &&
                         (s_sel[j0 + jj] != n - 1 || tt < last_valid);
      __nv_bfloat16 pb = __float2bfloat16(0.0f);
      if (valid && mx != -INFINITY) {
        pb = __float2bfloat16(exp2f(s_st[t * (G + 1) + g] - mx));
        sum += __bfloat162float(pb);  // normalise by the weights actually used
      }
      s_pm[g * PST + t] = pb;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);
    if (lane == 0) {
      s_ml[2 * g] = mx;
      s_ml[2 * g + 1] = sum;
    }
  }
  __syncthreads();

  // O = P V: warp w owns output dims [64 w, 64 w + 64) for all G heads
  float oacc[G / 16][8][4];
#pragma unroll
  for (int mt = 0; mt < G / 16; ++mt)
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) oacc[mt][nt][i] = 0.0f;
  {
    const uint32_t pa_base = smem_u32(s_pm + (lane & 15) * PST + (lane >> 4) * 8);
    const uint32_t vb_base = smem_u32(s_kt + ((lane & 7) + ((lane >> 3) & 1) * 8) * kMlaRow +
                                      warp * 64 + (lane >> 4) * 8);
    for (int ks = 0; ks < np; ++ks) {  // 16 tokens per step
      uint32_t a[G / 16][4];
#pragma unroll
      for (int mt = 0; mt < G / 16; ++mt)
        ldsm_x4(pa_base + (mt * 16 * PST + ks * 16) * 2, a[mt][0], a[mt][1], a[mt][2], a[mt][3]);
#pragma unroll
      for (int n2 = 0; n2 < 4; ++n2) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vb_base + (ks * 16 * kMlaRow + n2 * 16) * 2, b0, b1, b2, b3);
#pragma unroll
        for (int mt = 0; mt < G / 16; ++mt) {
          mma_16816(oacc[mt][2 * n2], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b0, b1);
          mma_16816(oacc[mt][2 * n2 + 1], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b2, b3);
        }
      }
    }
  }
  __syncthreads();  // K tiles are dead: s_o aliases them
#pragma unroll
  for (int mt = 0; mt < G / 16; ++mt)
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const int g = mt * 16 + (lane >> 2);
      const int d = warp * 64 + nt * 8 + 2 * (lane & 3);
      s_o[g * (DV + 2) + d] = oacc[mt][nt][0];
      s_o[g * (DV + 2) + d + 1] = oacc[mt][nt][1];
      s_o[(g + 8) * (DV + 2) + d] = oacc[mt][nt][2];
      s_o[(g + 8) * (DV + 2) + d + 1] = oacc[mt][nt][3];
    }
  for (int g = tid; g < G; g += NT) {
    s_o[g * (DV + 2) + DV] = s_ml[2 * g];
    s_o[g * (DV + 2) + DV + 1] = s_ml[2 * g + 1];
  }
  cluster.sync();  // #3

  {
    const int total = G * DV;
    const int per = (total + C - 1) / C;
    const int i1 = min(total, (rank + 1) * per);
    for (int idx = rank * per + tid; idx < i1; idx += NT) {
      const int g = idx / DV, d = idx - g * DV;
      float M = -INFINITY;
      for (int r = 0; r < C; ++r)
        M = fmaxf(M, cluster.map_shared_rank(s_o, r)[g * (DV + 2) + DV]);
      float A = 0.0f, Lsum = 0.0f;
      for (int r = 0; r < C; ++r) {
        const float* pc = cluster.map_shared_rank(s_o, r) + g * (DV + 2);
        const float mr = pc[DV];
        const float f = (mr == -INFINITY) ? 0.0f : exp2f(mr - M);
        A = fmaf(pc[d], f, A);
        Lsum = fmaf(pc[DV + 1], f, Lsum);
      }
      p.out[(orow + g) * DV + d] = __float2bfloat16(Lsum > 0.0f ? A / Lsum : 0.0f);
      if (d == 0 && p.lse) p.lse[orow + g] = Lsum > 0.0f ? (M + log2f(Lsum)) * kLn2 : -INFINITY;
    }
  }
  cluster.sync();  // #4
}

template <int G, int MODE>
static cudaError_t launch_mla_t(const DecodeParams& p, int C, cudaStream_t stream) {
  auto kern = mla_decode_kernel<G, MODE>;
  const int ppc = (p.kmax + C - 1) / C;
  const MlaSmem L = mla_smem_layout(G, p.cand_cap, p.key_cap, p.kmax, ppc);
  static std::atomic<int> optin[64];
  cudaError_t e = ensure_smem_optin(kern, L.total, C > 8, optin);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((int64_t)C * p.B), 1, 1);
  cfg.blockDim = dim3(kMlaThreads, 1, 1);
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

template <int MODE>
static cudaError_t dispatch_mla_g(const DecodeParams& p, int G, int C, cudaStream_t s) {
  if (G == 16) return launch_mla_t<16, MODE>(p, C, s);
  if (G == 32) return launch_mla_t<32, MODE>(p, C, s);
  return cudaErrorInvalidValue;
}

int mla_max_pages_per_cta() { return kMlaMaxPages; }

int mla_smem_bytes(int G, int cand_cap, int key_cap, int kmax, int ppc) {
  return mla_smem_layout(G, cand_cap, key_cap, kmax, ppc).total;
}

cudaError_t launch_mla_decode(const DecodeParams& p, int mode, int G, int C, cudaStream_t s) {
  switch (mode) {
    case kSelect: return dispatch_mla_g<kSelect>(p, G, C, s);
    case kDecode: return dispatch_mla_g<kDecode>(p, G, C, s);
    case kFused: return dispatch_mla_g<kFused>(p, G, C, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace vt
