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

// NB bins over the keys in [lo, hi]: linear in the score between the smallest and the
// largest one (scores near the top are then spread over many bins); when that range is not
// finite, bins of width 2^sh in key space.  Either map is monotone in the key.
template <int NB>
struct KeyBinsT {
  static constexpr int LOG2 = NB == 1024 ? 10 : (NB == 256 ? 8 : -1);
  static_assert(LOG2 > 0, "1024 or 256 bins");
  float flo, inv;
  uint32_t lo;
  int sh;
  bool linear;
  __device__ __forceinline__ KeyBinsT(uint32_t lo_, uint32_t hi) : lo(lo_) {
    flo = key_score(lo_);
    const float fhi = key_score(hi);
    const float width = fhi - flo;
    const float inv0 = __fdividef((float)NB, width);  // any positive scale is monotone
    linear = isfinite(flo) && isfinite(fhi) && width > 0.0f && isfinite(inv0);
    inv = linear ? inv0 : 0.0f;
    const int bits = 32 - __clz(hi - lo_);
    sh = bits > LOG2 ? bits - LOG2 : 0;
  }
  __device__ __forceinline__ int operator()(uint32_t key) const {
    if (linear) {
      const float x = (key_score(key) - flo) * inv;
      return x >= (float)(NB - 1) ? NB - 1 : (int)x;  // x >= 0 by construction
    }
    return (int)((key - lo) >> sh);
  }
};
using KeyBins = KeyBinsT<kTopkBins>;

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
  const KeyBins bin_of(lo, hi);
  // 2. histogram
  for (int j = tid; j < m; j += NT) atomicAdd(&hist[bin_of(keys[j])], 1);
  __syncthreads();
  // 3. the bin holding the k-th largest key (warp 0: 32 bins per lane, top bins in lane 31)
  if (warp == 0) {
    constexpr int BPL = kTopkBins / 32;
    int tot = 0;
#pragma unroll
    for (int i = 0; i < BPL; ++i) tot += hist[lane * BPL + ((i + lane) & (BPL - 1))];  // no bank conflicts
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

// ---- the lossy mode: one radix pass, then stop --------------------------------------------
// The indexer's early-terminating ("stochastic radix") top-k of the rndamp.com article, "A
// dual-stage programmable abstraction", read as: one histogram pass of 1024 bins linear in
// the fp32 score between the smallest and the largest key (IEEE fp32 steps: (s - lo) * (1024 /
// (hi - lo)), truncated, capped at 1023; one bin when hi == lo or the range is not finite),
// every key in a bin above the k-th key's bin B selected, and no refinement inside B: its
// remaining slots go to B's keys in cyclic index order starting at index `start`.

// SplitMix64's output step (Steele, Lea and Flood 2014): advance by the golden gamma, then
// two xor-shift-multiply rounds.  The counter-based generator of the lossy mode's start.
__host__ __device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Scratch in shared memory: hist[kTopkBins] ints, small[64] ints.  Emits exactly k indices
// (k < m) in ascending order with their positions.
template <int NT, typename Emit>
__device__ void approx_topk(const uint32_t* keys, int m, int k, int start, int* hist, int* small,
                            Emit emit) {
  constexpr int NW = NT / 32;
  static_assert(NW <= 8, "small[] holds per-warp counts of at most 8 warps");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (k <= 0) return;
  if (k >= m) {
    for (int j = tid; j < m; j += NT) emit(j, j);
    __syncthreads();
    return;
  }
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
  const float flo = key_score(lo), width = __fsub_rn(key_score(hi), flo);
  const bool linear = width > 0.0f && isfinite(width);
  const float inv = linear ? __fdiv_rn((float)kTopkBins, width) : 0.0f;
  auto bin_of = [&](uint32_t key) {
    if (!linear) return 0;
    const float x = __fmul_rn(__fsub_rn(key_score(key), flo), inv);
    return x >= (float)(kTopkBins - 1) ? kTopkBins - 1 : (int)x;
  };
  for (int j = tid; j < m; j += NT) atomicAdd(&hist[bin_of(keys[j])], 1);
  __syncthreads();
  if (warp == 0) {  // the bin of the k-th largest key (32 bins per lane, top bins in lane 31)
    constexpr int BPL = kTopkBins / 32;
    int tot = 0;
#pragma unroll
    for (int i = 0; i < BPL; ++i) tot += hist[lane * BPL + ((i + lane) & (BPL - 1))];
    int incl = tot;
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
          break;
        }
        acc += c;
      }
    }
  }
  __syncthreads();
  const int B = small[40];
  const int need = k - small[41];
  // emit in ascending index order: every warp walks a contiguous range in chunks of 32; the
  // members of B are ranked in cyclic order from `start`
  const int R = ((m + NW * 32 - 1) / (NW * 32)) * 32;
  const int w0 = min(m, warp * R), w1 = min(m, w0 + R);
  const unsigned lt = (1u << lane) - 1u;
  int c2 = 0, c1 = 0, c1lo = 0;  // above B; in B; in B with index < start
  for (int j0 = w0; j0 < w1; j0 += 32) {
    const int j = j0 + lane;
    const int b = j < w1 ? bin_of(keys[j]) : -1;
    c2 += __popc(__ballot_sync(kFull, b > B));
    c1 += __popc(__ballot_sync(kFull, b == B));
    c1lo += __popc(__ballot_sync(kFull, b == B && j < start));
  }
  __syncthreads();  // everyone is done with small[] reads above
  if (lane == 0) {
    small[48 + warp] = c2;
    small[56 + warp] = c1;
    small[32 + warp] = c1lo;
  }
  __syncthreads();
  int T1 = 0, L1 = 0, pre2 = 0, pre1 = 0;
  for (int w = 0; w < NW; ++w) {
    T1 += small[56 + w];
    L1 += small[32 + w];
    if (w < warp) {
      pre2 += small[48 + w];
      pre1 += small[56 + w];
    }
  }
  auto taken_tie = [&](int j, int rank_from_0) {  // rank_from_0: members of B below j
    const int cyc = j >= start ? rank_from_0 - L1 : (T1 - L1) + rank_from_0;
    return cyc < need;
  };
  // offsets of this warp's first selected key: every selected key of earlier warps
  int sel_off = pre2;
  {
    // members of B taken among indices < w0: count them from the prefix counts
    // (taken(j) depends only on j's rank among B's members, so count ranks [0, pre1))
    int t = 0;
    // ranks r < pre1 belong to indices < w0; those with index >= start are the ranks >= L1
    const int lo_taken = min(pre1, L1);           // ranks [0, lo_taken): index < start
    // index < start: cyclic rank (T1 - L1) + r, taken when < need
    t += max(0, min(lo_taken, need - (T1 - L1)));
    // index >= start: ranks [L1, pre1): cyclic rank r - L1, taken when < need
    if (pre1 > L1) t += max(0, min(pre1, L1 + need) - L1);
    sel_off += t;
  }
  int rank1 = pre1;
  for (int j0 = w0; j0 < w1; j0 += 32) {
    const int j = j0 + lane;
    const int b = j < w1 ? bin_of(keys[j]) : -1;
    const unsigned tb = __ballot_sync(kFull, b == B);
    const int r1 = rank1 + __popc(tb & lt);
    const bool take = (b > B) || (b == B && taken_tie(j, r1));
    const unsigned sb = __ballot_sync(kFull, take);
    if (take) emit(j, sel_off + __popc(sb & lt));
    sel_off += __popc(sb);
    rank1 += __popc(tb);
  }
  __syncthreads();
}

// Shared-memory scratch of small_topk (16-byte aligned): hist[HIST] ints that are ZERO on
// entry (hist[kSmallBins] counts the members of the threshold bin), list[2 NT] (key, index)
// pairs, cnt[2 NW] ints.
constexpr int kSmallBins = 256;
template <int NT>
struct SmallTopk {
  static constexpr int HIST = kSmallBins + 4;
  static constexpr int LIST = HIST * 4;                 // byte offset of list
  static constexpr int CNT = LIST + 2 * NT * 8;         // byte offset of cnt
  static constexpr int BYTES = CNT + 2 * (NT / 32) * 4;
};

// Exact top-k of m <= 2 NT keys, ties going to the lowest index, with two block barriers
// (three when the bin of the k-th largest key holds more keys than are still needed).
// On entry keys[0, m) and the zeroed histogram are visible to every thread and lo / hi are
// the smallest and the largest of the keys.  Thread t owns keys t and t + NT.  emit(j, pos)
// receives the selected indices with their positions in ascending index order; no barrier
// follows the emits.  Steps: one histogram of kSmallBins bins monotone in the key; every warp
// finds the threshold bin B from it on its own (no barrier); keys above B are selected, and
// the keys of B are all selected when B holds exactly the number still needed, otherwise
// ranked among the members of B (by key, then index).
template <int NT, typename Emit>
__device__ __forceinline__ void small_topk(const uint32_t* keys, int m, int k, uint32_t lo,
                                           uint32_t hi, unsigned char* scratch, Emit emit) {
  constexpr int NW = NT / 32;
  using S = SmallTopk<NT>;
  int* hist = reinterpret_cast<int*>(scratch);
  uint2* list = reinterpret_cast<uint2*>(scratch + S::LIST);
  int* cnt = reinterpret_cast<int*>(scratch + S::CNT);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int j0 = tid, j1 = tid + NT;
  if (k <= 0) return;
  if (k >= m) {  // every key is selected
    if (j0 < m) emit(j0, j0);
    if (j1 < m) emit(j1, j1);
    return;
  }
  const uint32_t k0 = j0 < m ? keys[j0] : 0u, k1 = j1 < m ? keys[j1] : 0u;
  const KeyBinsT<kSmallBins> bins(lo, hi);
  auto bin_of = [&](uint32_t key) { return min(max(bins(key), 0), kSmallBins - 1); };
  const int b0 = j0 < m ? bin_of(k0) : -1, b1 = j1 < m ? bin_of(k1) : -1;
  if (b0 >= 0) atomicAdd(&hist[b0], 1);
  if (b1 >= 0) atomicAdd(&hist[b1], 1);
  __syncthreads();
  // threshold bin, found by every warp.  Lane l totals bins [8 l, 8 l + 8) (two 16-byte
  // loads, the pair's order rotated so that no two lanes of a phase share banks); a suffix scan
  // over the lanes finds the lane src holding the k-th key, and lanes 0..7 then split src's
  // eight bins for a second suffix scan.
  static_assert(kSmallBins == 8 * 32, "eight bins per lane");
  const int4* h4 = reinterpret_cast<const int4*>(hist);
  const int rot = (lane >> 2) & 1;
  const int4 va = h4[2 * lane + rot], vb = h4[2 * lane + (rot ^ 1)];
  const int tot = ((va.x + va.y) + (va.z + va.w)) + ((vb.x + vb.y) + (vb.z + vb.w));
  int incl = tot;  // keys in the bins of lanes >= lane
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_down_sync(kFull, incl, o);
    if (lane + o < 32) incl += y;
  }
  const int src = __ffs(__ballot_sync(kFull, incl - tot < k && k <= incl)) - 1;
  const int above = __shfl_sync(kFull, incl - tot, src);
  const int i8 = lane & 7;
  const int cbin = hist[8 * src + i8];
  int s8 = cbin;  // keys in src's bins >= i8
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {
    const int y = __shfl_down_sync(kFull, s8, o, 8);
    if (i8 + o < 8) s8 += y;
  }
  const int bi = __ffs(__ballot_sync(kFull, lane < 8 && above + s8 - cbin < k && k <= above + s8)) - 1;
  const int B = 8 * src + bi;
  const int cntB = __shfl_sync(kFull, cbin, bi);
  const int need = k - above - __shfl_sync(kFull, s8 - cbin, bi);
  bool s0 = b0 > B, s1 = b1 > B;
  if (cntB == need) {
    s0 |= b0 == B;
    s1 |= b1 == B;
  } else {
    if (b0 == B) list[atomicAdd(&hist[kSmallBins], 1)] = make_uint2(k0, (uint32_t)j0);
    if (b1 == B) list[atomicAdd(&hist[kSmallBins], 1)] = make_uint2(k1, (uint32_t)j1);
    __syncthreads();
    auto ranked_in = [&](uint32_t key, int j) {
      int r = 0;
      for (int i = 0; i < cntB; ++i) {
        const uint2 e = list[i];
        r += (e.x > key) || (e.x == key && (int)e.y < j);
      }
      return r < need;
    };
    if (b0 == B) s0 = ranked_in(k0, j0);
    if (b1 == B) s1 = ranked_in(k1, j1);
  }
  const unsigned bal0 = __ballot_sync(kFull, s0), bal1 = __ballot_sync(kFull, s1);
  if (lane == 0) {
    cnt[warp] = __popc(bal0);
    cnt[NW + warp] = __popc(bal1);
  }
  __syncthreads();
  int off0 = 0, off1 = 0, tot0 = 0;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const int c0 = cnt[w];
    tot0 += c0;
    if (w < warp) {
      off0 += c0;
      off1 += cnt[NW + w];
    }
  }
  const unsigned lt = (1u << lane) - 1u;
  if (s0) emit(j0, off0 + __popc(bal0 & lt));
  if (s1) emit(j1, tot0 + off1 + __popc(bal1 & lt));
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
