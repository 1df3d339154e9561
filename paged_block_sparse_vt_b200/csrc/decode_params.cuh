// decode_params.cuh -- launch parameters shared by the query-side kernels.
#pragma once

#include "common.cuh"

namespace vt {

enum Mode : int { kSelect = 1, kDecode = 2, kFused = 3 };

struct DecodeParams {
  // paged K/V (strides in elements)
  const __nv_bfloat16* k_pool;
  const __nv_bfloat16* v_pool;
  int64_t num_pages;
  int Hkv;
  int64_t sk_p, sk_t, sk_h;
  int64_t sv_p, sv_t, sv_h;
  // batch
  int B, Hq;
  const __nv_bfloat16* q;
  const int32_t* page_table;
  int64_t pt_stride;
  const int32_t* seq_lens;
  const float* centroids;
  int topk, bos, eos, kmax;
  float qscale;  // sm_scale * log2(e): scores are kept in base-2 units
  const int32_t* order;
  int32_t* status;
  // selection: written by kSelect / kFused (may be null in kFused), read by kDecode
  int32_t* sel;
  int32_t* n_sel;
  // attention outputs
  __nv_bfloat16* out;
  float* lse;
  // per-CTA capacities sizing the shared-memory carve-up
  int cand_cap;  // candidates scored by one CTA
  int key_cap;   // candidates of one unit (rank 0 selects over all of them)
};

__host__ __device__ inline int align16(int x) { return (x + 15) & ~15; }

// Shared-memory carve-up of the CUDA-core decode kernel (byte offsets).
struct FmaSmem {
  int qm, cpage, score, key, sel, phys, warp, cta, misc, total;
};

__host__ __device__ inline FmaSmem fma_smem_layout(int D, int G, int NW, int cand_cap, int key_cap,
                                                   int kmax) {
  FmaSmem s;
  int o = 0;
  s.qm = o;    o += align16(D * 4);
  s.cpage = o; o += align16(cand_cap * 4);
  s.score = o; o += align16(cand_cap * 4);
  s.key = o;   o += align16(key_cap * 4);
  s.sel = o;   o += align16(kmax * 4);
  s.phys = o;  o += align16(kmax * 4);
  s.warp = o;  o += align16(NW * G * (D + 2) * 4);
  s.cta = o;   o += align16(G * (D + 2) * 4);
  s.misc = o;  o += align16(320 * 4);
  s.total = o;
  return s;
}

}  // namespace vt
