// centroid_chunk.cuh -- one (page, KV head, 8-dim chunk) of the cache-side centroid build
// (CMean over the 16 tokens of a finished page: "Vortex: A Flexible and Efficient Sparse
// Attention Framework", README "Quick Example", forward_cache), shared by the standalone
// build kernel and the fused decode step that builds the pages filled at this step.
//
// All 16 token loads are issued before use; the sum is accumulated in fp64, where 16 bf16
// values add exactly for any realistic exponent spread, so the fp32 centroid is the exact
// mean rounded once -- the same bits whichever kernel computes it.
#pragma once

#include "common.cuh"

namespace vt {

__device__ __forceinline__ void build_centroid_chunk(const __nv_bfloat16* __restrict__ k_pool,
                                                     int64_t p, int h, int c, int64_t sk_p,
                                                     int64_t sk_t, int64_t sk_h,
                                                     int num_kv_heads, int head_dim,
                                                     float* __restrict__ centroids) {
  const __nv_bfloat16* base = k_pool + p * sk_p + (int64_t)h * sk_h + (int64_t)c * 8;
  uint4 r[kPage];
#pragma unroll
  for (int t = 0; t < kPage; ++t) r[t] = ld_stream_u4(base + (int64_t)t * sk_t);
  double acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.0;
#pragma unroll
  for (int t = 0; t < kPage; ++t) {
    float f[8];
    unpack8(r[t], f);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] += (double)f[i];
  }
  float o[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = __double2float_rn(acc[i] * (1.0 / kPage));
  float4* dst = reinterpret_cast<float4*>(centroids + (p * num_kv_heads + h) * head_dim + c * 8);
  dst[0] = make_float4(o[0], o[1], o[2], o[3]);
  dst[1] = make_float4(o[4], o[5], o[6], o[7]);
}

}  // namespace vt
