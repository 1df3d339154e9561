// plan.cu -- workload planner: request visiting order, longest first.
//
// Source: "Vortex: Efficient and Programmable Sparse Attention Serving for AI Agents"
// (rndamp.com), "A dual-stage programmable abstraction": a workload planner balances GPU
// scheduling across a heterogeneous batch.  Here the plan is the order in which the decode
// kernels hand requests to thread-block clusters: requests with more pages (longer centroid
// scans) are issued first so that short ones fill in behind them.
#include "common.cuh"

namespace vt {

__global__ void __launch_bounds__(1024) plan_kernel(const int32_t* __restrict__ seq_lens, int B,
                                                    int32_t* __restrict__ order) {
  extern __shared__ uint16_t s_n[];  // page count per request (saturating at 65535)
  for (int i = threadIdx.x; i < B; i += blockDim.x) {
    const int L = seq_lens[i];
    const int n = L < 1 ? 0 : (L + kPage - 1) / kPage;
    s_n[i] = (uint16_t)min(n, 65535);
  }
  __syncthreads();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < B; i += gridDim.x * blockDim.x) {
    const int ni = s_n[i];
    int rank = 0;
    for (int j = 0; j < B; ++j) {
      const int nj = s_n[j];
      rank += (nj > ni) | ((nj == ni) & (j < i));
    }
    order[rank] = i;  // ranks form a permutation of [0, B)
  }
}

cudaError_t launch_plan(const int32_t* seq_lens, int B, int32_t* order, cudaStream_t s) {
  const int nt = 1024;
  const int blocks = (B + nt - 1) / nt;
  const int smem = B * (int)sizeof(uint16_t);
  cudaError_t e = cudaFuncSetAttribute(plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       smem);
  if (e != cudaSuccess) return e;
  plan_kernel<<<blocks, nt, smem, s>>>(seq_lens, B, order);
  return cudaGetLastError();
}

}  // namespace vt
