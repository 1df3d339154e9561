// centroids.cu -- cache-side centroid build (CMean over the tokens of a finished page).
//
// Source: "Vortex: A Flexible and Efficient Sparse Attention Framework" (vortex_torch
// README), "Quick Example": forward_cache runs CMean(dim=1) over cache["k"] into
// cache["centroids"] when a page is finished; create_cache declares one (1, head_dim)
// centroid per page.
//
// Pure HBM stream: each thread owns 8 consecutive dims (one 16-byte load per token) of one
// (page, KV head) (build_centroid_chunk).  Consecutive threads cover consecutive 16-byte
// chunks, so a warp reads whole 256-byte head rows.
#include "centroid_chunk.cuh"

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
  build_centroid_chunk(k_pool, p, h, c, sk_p, sk_t, sk_h, num_kv_heads, head_dim, centroids);
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
