// topk.cuh -- exact block-wide top-k over 32-bit ordered score keys, and warp exchange
// reductions.
//
// Top-k ("topK" in the vortex_torch README "Quick Example"; the rndamp.com article's
// "A dual-stage programmable abstraction" selects the top-k blocks) is exact here: the
// selected set is the k largest keys, ties at the threshold going to the lowest indices.
//
// Method (one block of NT threads, keys in shared memory):
//   1. min and max of the keys;
//   2. one histogram of 1024 bins linear in the score between the two (a monotone map, so
//      every key in a higher bin is strictly larger);
//   3. the bin B holding the k-th largest key: everything above B is selected; if B holds
//      exactly the keys still needed they are all selected -- the common case, because the
//      top of the distribution is sparse;
//   4. otherwise 8-bit radix passes, most significant digit first, over the members of B
//      only, ending either when a digit class holds exactly the keys still needed or with
//      a single key value whose lowest-index members are taken;
//   5. selected indices are emitted in ascending order with their output position: every
//      warp counts its contiguous range by ballots, one barrier, then emits.
#pragma once

#include "common.cuh"

namespace vt {

constexpr int kTopkBins = 1024;

// Inverse of score_key: the fp32 score an ordered key came from.
__device__ __forceinline__ float key_score(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// Scratch in shared memory: hist[kTopkBins] ints, small[64] ints.
template <int NT, typename Emit>
__device__ void block_topk(const uint32_t* keys, int m, int k, int* hist, int* small, Emit emit) {
  constexpr int NW = NT / 32;
  static_assert(NW <= 8, "small[] holds per-warp counts of at most 8 warps");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (k <= 0) return;
  if (k >= m) {  // everything is selected
    for (int j = tid; j < m; j += NT) emit(j, j);
    __syncthreads();
    return;
  }
  // 1. range of the keys
  uint32_t lo = 0xffffffffu, hi = 0u;
  for (int j = tid; j < m; j += NT) {
    const uint32_t key = keys[j];
    lo = min(lo, key);
    hi = max(hi, key);
  }
  lo = __reduce_min_sync(kFull, lo);
  hi = __reduce_max_sync(kFull, hi);
  if (lane == 0) {
    small[warp] = (int)lo;
    small[NW + warp] = (int)hi;
  }
  for (int i = tid; i < kTopkBins; i += NT) hist[i] = 0;
  __syncthreads();
  lo = 0xffffffffu;
  hi = 0u;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    lo = min(lo, (uint32_t)small[w]);
    hi = max(hi, (uint32_t)small[NW + w]);
  }
  // Bins linear in the score between the smallest and the largest one (scores near the
  // top are then spread over many bins); when the range is not finite, bins of width 2^sh
  // in key space.  Either map is monotone in the key.
  const float flo = key_score(lo), fhi = key_score(hi);
  const float width = fhi - flo;
  const float inv0 = (float)kTopkBins / width;
  const bool linear = isfinite(flo) && isfinite(fhi) && width > 0.0f && isfinite(inv0);
  const float inv = linear ? inv0 : 0.0f;
  const int bits = 32 - __clz(hi - lo);
  const int sh = bits > 10 ? bits - 10 : 0;
  auto bin_of = [&](uint32_t key) -> int {
    if (linear) {
      const float x = (key_score(key) - flo) * inv;
      return x >= (float)(kTopkBins - 1) ? kTopkBins - 1 : (int)x;  // x >= 0 by construction
    }
    return (int)((key - lo) >> sh);
  };
  // 2. histogram
  for (int j = tid; j < m; j += NT) atomicAdd(&hist[bin_of(keys[j])], 1);
  __syncthreads();
  // 3. the bin holding the k-th largest key (warp 0: 32 bins per lane, top bins in lane 31)
  if (warp == 0) {
    constexpr int BPL = kTopkBins / 32;
    int tot = 0;
#pragma unroll
    for (int i = 0; i < BPL; ++i) tot += hist[lane * BPL + i];
    int incl = tot;  // sum over lanes >= lane
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_down_sync(kFull, incl, o);
      if (lane + o < 32) incl += y;
    }
    const int above_lane = incl - tot;
    if (above_lane < k && k <= incl) {
      int acc = above_lane;
      for (int i = BPL - 1; i >= 0; --i) {
        const int c = hist[lane * BPL + i];
        if (acc + c >= k) {
          small[40] = lane * BPL + i;
          small[41] = acc;
          small[42] = c;
          break;
        }
        acc += c;
      }
    }
  }
  __syncthreads();
  const int B = small[40];
  int need = k - small[41];
  const int cntB = small[42];
  // 4. refine inside bin B when it holds more keys than are still needed (8-bit radix over
  //    the keys of B, most significant digit first)
  uint32_t prefix = 0u, mask = 0u;
  bool take_all = (cntB == need);
  if (!take_all) {
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
      __syncthreads();
      for (int i = tid; i < 256; i += NT) hist[i] = 0;
      __syncthreads();
      for (int j = tid; j < m; j += NT) {
        const uint32_t key = keys[j];
        if (bin_of(key) == B && (key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
      }
      __syncthreads();
      if (warp == 0) {
        int cnt[8], tot = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          cnt[i] = hist[8 * lane + i];
          tot += cnt[i];
        }
        int incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_down_sync(kFull, incl, o);
          if (lane + o < 32) incl += y;
        }
        const int above_lane = incl - tot;
        if (above_lane < need && need <= incl) {
          int acc = above_lane;
#pragma unroll
          for (int i = 7; i >= 0; --i) {
            if (acc + cnt[i] >= need) {
              small[44] = 8 * lane + i;
              small[45] = acc;
              small[46] = cnt[i];
              break;
            }
            acc += cnt[i];
          }
        }
      }
      __syncthreads();
      const int d = small[44], above = small[45], cnt_d = small[46];
      prefix |= (uint32_t)d << shift;
      mask |= 0xffu << shift;
      need -= above;
      if (cnt_d == need) {
        take_all = true;
        break;
      }
    }
  }
  // 5. emit in ascending index order.  Class 2 = surely selected, 1 = tie at the threshold
  //    (the lowest-index `need` of them are selected unless take_all).  Each warp walks a
  //    contiguous range in chunks of 32 keys; ballots give positions inside a chunk.
  auto cls = [&](uint32_t key) -> int {
    const int b = bin_of(key);
    if (b > B) return 2;
    if (b < B) return 0;
    if (take_all && mask == 0u) return 2;
    const uint32_t km = key & mask;
    if (km > prefix) return 2;
    if (km < prefix) return 0;
    return take_all ? 2 : 1;
  };
  const int R = ((m + NW * 32 - 1) / (NW * 32)) * 32;  // keys per warp, whole chunks
  const int w0 = min(m, warp * R), w1 = min(m, w0 + R);
  const unsigned lt = (1u << lane) - 1u;
  int c2 = 0, c1 = 0;
  for (int j0 = w0; j0 < w1; j0 += 32) {
    const int j = j0 + lane;
    const int c = j < w1 ? cls(keys[j]) : 0;
    c2 += __popc(__ballot_sync(kFull, c == 2));
    c1 += __popc(__ballot_sync(kFull, c == 1));
  }
  __syncthreads();  // everyone is done with small[] reads above
  if (lane == 0) {
    small[48 + warp] = c2;
    small[56 + warp] = c1;
  }
  __syncthreads();
  int sel_off = 0, tie_off = 0;
  for (int w = 0; w < warp; ++w) {
    const int t1 = small[56 + w];
    const int taken = take_all ? t1 : max(0, min(t1, need - tie_off));
    sel_off += small[48 + w] + taken;
    tie_off += t1;
  }
  for (int j0 = w0; j0 < w1; j0 += 32) {
    const int j = j0 + lane;
    const int c = j < w1 ? cls(keys[j]) : 0;
    const unsigned tb = __ballot_sync(kFull, c == 1);
    const int tie_rank = tie_off + __popc(tb & lt);
    const bool take = (c == 2) || (c == 1 && (take_all || tie_rank < need));
    const unsigned sb = __ballot_sync(kFull, take);
    if (take) emit(j, sel_off + __popc(sb & lt));
    sel_off += __popc(sb);
    tie_off += __popc(tb);
  }
  __syncthreads();
}

// Reduce N per-lane partial sums over aligned groups of L lanes (N <= L, both powers of two)
// with log2(N) exchange steps (each lane keeps half, sends half) and log2(L/N) plain steps:
// N - 1 + log2(L/N) shuffles instead of N log2(L).  On return v[0] holds the group sum of
// value number exchange_index<N, L>(lane).
template <int N, int L>
__device__ __forceinline__ void exchange_reduce(float (&v)[N], int lane) {
  static_assert(N <= L && (N & (N - 1)) == 0 && (L & (L - 1)) == 0, "powers of two, N <= L");
#pragma unroll
  for (int n = N, off = L / 2; n > 1; n >>= 1, off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
      const float send = upper ? v[i] : v[i + n / 2];
      const float keep = upper ? v[i + n / 2] : v[i];
      v[i] = keep + __shfl_xor_sync(kFull, send, off);
    }
  }
#pragma unroll
  for (int off = L / N / 2; off >= 1; off >>= 1) v[0] += __shfl_xor_sync(kFull, v[0], off);
}

template <int N, int L>
__device__ __forceinline__ int exchange_index(int lane) {
  int idx = 0;
#pragma unroll
  for (int n = N, off = L / 2; n > 1; n >>= 1, off >>= 1)
    if (lane & off) idx += n / 2;
  return idx;
}

}  // namespace vt
