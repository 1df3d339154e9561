// gqa_attend.cuh -- one warp's exact softmax attention over 16-token pages for GQA heads
// (head_dim 64/128, G <= 8 query heads sharing one KV head), on the tensor cores.
//
// "Performs the actual attention" over the selected blocks through the paged layout
// (rndamp.com article, "A dual-stage programmable abstraction").  Per page of 16 tokens:
//   S = Q K^T   mma.sync m16n8k16 (bf16 -> fp32); the G query rows are padded to 16 (rows
//               >= G are zero), K enters through ldmatrix from a shared-memory tile;
//   online softmax per query head in base 2 (running max m, running sum l), probabilities
//               rounded once to bf16 so that the MMA and the sum use the same values;
//   O += P V    P straight from the S accumulators (their layout is the A-operand layout),
//               V through ldmatrix.trans.
// With G <= 8 useful rows the MMA is mostly padding, but one page costs ~75 warp
// instructions instead of ~400 on the FMA pipe (bf16 unpacking, G FMAs per element and
// shuffle reductions), and this work is bound by instruction issue, not by FLOPs.
#pragma once

#include "common.cuh"

namespace vt {

// Shared-memory tile of one page: 16 rows of D bf16, row stride D + 8 elements so that the
// eight rows an ldmatrix phase touches fall into distinct bank groups.
template <int D>
struct PageTile {
  static constexpr int ROW = D + 8;             // elements
  static constexpr int TILE = kPage * ROW * 2;  // bytes of one K or V tile
  static constexpr int SLOT = 2 * TILE;         // K tile, then V tile
  static constexpr int KS = D / 16;             // k-steps of S = Q K^T
  static constexpr int NT = D / 8;              // n-tiles of O = P V
  static constexpr int CPR = D / 8;             // 16-byte chunks per row
};

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const uint32_t l = (uint32_t)__bfloat16_as_ushort(__float2bfloat16(lo));
  const uint32_t h = (uint32_t)__bfloat16_as_ushort(__float2bfloat16(hi));
  return l | (h << 16);
}
__device__ __forceinline__ float bf16_round(float x) {
  return __bfloat162float(__float2bfloat16(x));
}

// Stage one page (K rows and V rows of one KV head) into a slot with 16-byte cp.async; rows
// r >= vr are zero-filled instead of read.  kp / vp point at row 0 of the page for that head
// (ignored when vr == 0); zsrc is any valid global address.  The caller commits the group.
template <int D>
__device__ __forceinline__ void stage_page(uint32_t slot, const __nv_bfloat16* kp,
                                           const __nv_bfloat16* vp, int64_t sk_t,
                                           int64_t sv_t, int vr, const void* zsrc, int lane) {
  using T = PageTile<D>;
  constexpr int RPI = 32 / T::CPR;  // rows per warp instruction
#pragma unroll
  for (int t = 0; t < kPage / RPI; ++t) {
    const int row = t * RPI + lane / T::CPR, k = lane % T::CPR;
    const bool ok = row < vr;
    const uint32_t o = (row * T::ROW + k * 8) * 2;
    cp_async16(slot + o, ok ? (const void*)(kp + (int64_t)row * sk_t + k * 8) : zsrc, ok ? 16 : 0);
    cp_async16(slot + T::TILE + o, ok ? (const void*)(vp + (int64_t)row * sv_t + k * 8) : zsrc,
               ok ? 16 : 0);
  }
}

template <int D, int G>
struct WarpAttention {
  using T = PageTile<D>;
  uint32_t qa0[T::KS], qa2[T::KS];  // Q as the A operand: row g = lane / 4, k = 2 (lane % 4)
  float o[T::NT][4];                // O accumulators: row g, dims t*8 + 2 (lane % 4) + {0, 1}
  float mrun, lrun;                 // running max (base 2) and this lane's partial sum
  int g, qd;
  uint32_t koff, voff;

  // q_rows: the G query rows of the unit (bf16 [G][D], 4-byte aligned)
  __device__ __forceinline__ void init(const __nv_bfloat16* q_rows, int lane) {
    g = lane >> 2;
    qd = 2 * (lane & 3);
#pragma unroll
    for (int ks = 0; ks < T::KS; ++ks) {
      if (g < G) {
        const __nv_bfloat16* qr = q_rows + (int64_t)g * D + ks * 16 + qd;
        qa0[ks] = *reinterpret_cast<const uint32_t*>(qr);
        qa2[ks] = *reinterpret_cast<const uint32_t*>(qr + 8);
      } else {
        qa0[ks] = qa2[ks] = 0u;
      }
    }
#pragma unroll
    for (int t = 0; t < T::NT; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.0f;
    mrun = -INFINITY;
    lrun = 0.0f;
    koff = (((lane & 7) + ((lane >> 4) << 3)) * T::ROW + ((lane >> 3) & 1) * 8) * 2;
    voff = (((lane & 7) + ((lane >> 3) & 1) * 8) * T::ROW + (lane >> 4) * 8) * 2;
  }

  // Attend to one staged page with vr valid tokens; qscale = sm_scale * log2(e).
  __device__ __forceinline__ void page(uint32_t slot, int vr, float qscale) {
    const uint32_t kt = slot, vt = slot + T::TILE;
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < T::KS; ++ks) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4(kt + koff + ks * 32, b0, b1, b2, b3);
      mma_16816(s0, qa0[ks], 0u, qa2[ks], 0u, b0, b1);
      mma_16816(s1, qa0[ks], 0u, qa2[ks], 0u, b2, b3);
    }
    // this lane holds head g at tokens qd, qd+1 (s0) and 8+qd, 9+qd (s1)
    const bool live = g < G;
    const float z0 = (live && qd < vr) ? s0[0] * qscale : -INFINITY;
    const float z1 = (live && qd + 1 < vr) ? s0[1] * qscale : -INFINITY;
    const float z2 = (live && qd + 8 < vr) ? s1[0] * qscale : -INFINITY;
    const float z3 = (live && qd + 9 < vr) ? s1[1] * qscale : -INFINITY;
    float mx = fmaxf(fmaxf(z0, z1), fmaxf(z2, z3));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
    const float mnew = fmaxf(mrun, mx);
    const float corr = (mnew == -INFINITY) ? 1.0f : exp2f(mrun - mnew);
    const float p0 = z0 == -INFINITY ? 0.0f : bf16_round(exp2f(z0 - mnew));
    const float p1 = z1 == -INFINITY ? 0.0f : bf16_round(exp2f(z1 - mnew));
    const float p2 = z2 == -INFINITY ? 0.0f : bf16_round(exp2f(z2 - mnew));
    const float p3 = z3 == -INFINITY ? 0.0f : bf16_round(exp2f(z3 - mnew));
    lrun = lrun * corr + ((p0 + p1) + (p2 + p3));
    mrun = mnew;
#pragma unroll
    for (int t = 0; t < T::NT; ++t) {
      o[t][0] *= corr;
      o[t][1] *= corr;
    }
    const uint32_t pa0 = pack_bf16(p0, p1), pa2 = pack_bf16(p2, p3);
#pragma unroll
    for (int n2 = 0; n2 < T::NT / 2; ++n2) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(vt + voff + n2 * 32, b0, b1, b2, b3);
      mma_16816(o[2 * n2], pa0, 0u, pa2, 0u, b0, b1);
      mma_16816(o[2 * n2 + 1], pa0, 0u, pa2, 0u, b2, b3);
    }
  }

  // Sum the partial sums of the four lanes that share a head, then write this warp's
  // partial (acc[D], m, l) for each of its G heads to w[G][D + 2].
  __device__ __forceinline__ void store(float* w, int lane) {
    lrun += __shfl_xor_sync(kFull, lrun, 1);
    lrun += __shfl_xor_sync(kFull, lrun, 2);
    if (g < G) {
      float* r = w + g * (D + 2);
#pragma unroll
      for (int t = 0; t < T::NT; ++t) {
        r[t * 8 + qd] = o[t][0];
        r[t * 8 + qd + 1] = o[t][1];
      }
      if ((lane & 3) == 0) {
        r[D] = mrun;
        r[D + 1] = lrun;
      }
    }
  }
};

// Merge NP partials part[i][G][D+2] (acc, max, sum; base-2 max) into dst[G][D+2] with the
// threads of a block (any count); partials with max -inf are empty.
template <int G, int D>
__device__ __forceinline__ void merge_partials(const float* part, int np, float* dst, int tid,
                                               int nthreads) {
  for (int idx = tid; idx < G * D; idx += nthreads) {
    const int gg = idx / D, d = idx - gg * D;
    float M = -INFINITY;
    for (int w = 0; w < np; ++w) M = fmaxf(M, part[(w * G + gg) * (D + 2) + D]);
    float A = 0.0f, L = 0.0f;
    for (int w = 0; w < np; ++w) {
      const float* pw = part + (w * G + gg) * (D + 2);
      const float f = (pw[D] == -INFINITY) ? 0.0f : exp2f(pw[D] - M);
      A = fmaf(pw[d], f, A);
      L = fmaf(pw[D + 1], f, L);
    }
    dst[gg * (D + 2) + d] = A;
    if (d == 0) {
      dst[gg * (D + 2) + D] = M;
      dst[gg * (D + 2) + D + 1] = L;
    }
  }
}

}  // namespace vt
