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
  // the fused step's centroid build of the pages filled at this step (before its scans;
  // never pages that this step scores): page ids, their count, the centroid cache written
  const int32_t* fill_pages;
  int n_fill;
  float* cent_out;
  // the indexer's lossy mode (select only): one radix pass, a seeded start in the last bin
  int approx;
  unsigned long long seed;
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

// Shared-memory carve-up of the GQA decode kernel (byte offsets).
struct GqaSmem {
  int score, sel, phys, qm, cpage, key, misc, ring, warp, cta, total;
};

}  // namespace vt

#include <atomic>

namespace vt {

// cudaFuncSetAttribute once per (kernel, device) and size: the shared-memory opt-in only
// ever grows, so a later call asking for no more than what was set makes no runtime call
// (which also keeps repeated launches cheap on the host and safe inside stream capture).
// `cache` is a per-kernel array indexed by device: bytes * 2 + (non-portable cluster bit).
template <typename Kernel>
inline cudaError_t ensure_smem_optin(Kernel kern, int bytes, bool nonportable_cluster,
                                     std::atomic<int>* cache) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::atomic<int>& slot = cache[dev & 63];
  const int have = slot.load(std::memory_order_acquire);
  if (have != 0 && (have >> 1) >= bytes && (!nonportable_cluster || (have & 1))) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  if (nonportable_cluster) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  const int hb = have >> 1;
  slot.store(((hb > bytes ? hb : bytes) << 1) | (have & 1) | (nonportable_cluster ? 1 : 0),
             std::memory_order_release);
  return cudaSuccess;
}

// CTAs of kern per SM at this block size and dynamic shared memory, cached per device for
// the last size asked for (the occupancy query otherwise costs host time on every call).
template <typename Kernel>
inline cudaError_t blocks_per_sm(Kernel kern, int threads, int bytes, std::atomic<long long>* cache,
                                 int* per_sm) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::atomic<long long>& slot = cache[dev & 63];
  const long long have = slot.load(std::memory_order_acquire);
  if (have != 0 && (int)(have >> 32) == bytes) {
    *per_sm = (int)(have & 0xffffffffLL);
    return cudaSuccess;
  }
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(per_sm, kern, threads, bytes);
  if (e != cudaSuccess) return e;
  slot.store(((long long)bytes << 32) | (long long)(unsigned)*per_sm, std::memory_order_release);
  return cudaSuccess;
}

}  // namespace vt
