// centroids.cu -- cache-side centroid build (CMean over the tokens of a finished page).
//
// Source: "Vortex: A Flexible and Efficient Sparse Attention Framework" (vortex_torch
// README), "Quick Example": forward_cache runs CMean(dim=1) over cache["k"] into
// cache["centroids"] when a page is finished; create_cache declares one (1, head_dim)
// centroid per page.
//
// Pure HBM stream: each thread owns 8 consecutive dims (one 16-byte load per token) of one
// (page, KV head) and issues all 16 token loads before using them.  Consecutive threads
// cover consecutive 16-byte chunks, so a warp reads whole 256-byte head rows.  The sum is
// accumulated in fp64, where 16 bf16 values add exactly for any realistic exponent spread,
// so the fp32 centroid is the exact mean rounded once -- independent of summation order.
#include "common.cuh"

namespace vt {

__global__ void __launch_bounds__(256) build_centroids_kernel(
    const __nv_bfloat16* __restrict__ k_pool, int64_t num_pages, int num_kv_heads, int head_dim,
    int64_t sk_p, int64_t sk_t, int64_t sk_h, const int32_t* __restrict__ pages, int n_pages,
    float* __restrict__ centroids, int32_t* status) {
  // Launched as a programmatic dependent of the previous kernel on the stream (which may read
  // the centroids): nothing is read or written before that kernel has completed.  The next
  // kernel may be placed at once and waits the same way.
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  const int chunks = head_dim >> 3;
  const int64_t per_page = (int64_t)num_kv_heads * chunks;
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= (int64_t)n_pages * per_page) return;
  const int pi = (int)(gid / per_page);
  const int rem = (int)(gid - (int64_t)pi * per_page);
  const int h = rem / chunks;
  const int c = rem - h * chunks;
  const int64_t p = pages[pi];
  if (p < 0 || p >= num_pages) {
    if (rem == 0) flag(status, VT_DEV_BAD_PAGE);
    return;
  }
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

cudaError_t launch_build_centroids(const vt_paged_kv& kv, const int32_t* pages, int n_pages,
                                   float* centroids, int32_t* status, cudaStream_t stream) {
  const int64_t threads = (int64_t)n_pages * kv.num_kv_heads * (kv.head_dim / 8);
  if (threads == 0) return cudaSuccess;
  const int nt = 256;
  const int64_t blocks = (threads + nt - 1) / nt;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(nt);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, build_centroids_kernel,
                            static_cast<const __nv_bfloat16*>(kv.k_pool), kv.num_pages,
                            kv.num_kv_heads, kv.head_dim, kv.sk_p, kv.sk_t, kv.sk_h, pages,
                            n_pages, centroids, status);
}

}  // namespace vt
