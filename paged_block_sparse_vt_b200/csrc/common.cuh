// common.cuh -- device helpers shared by the libvt kernels (sm_100a).
#pragma once

#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/vt.h"

namespace vt {

namespace cg = cooperative_groups;

constexpr int kPage = VT_PAGE_SIZE;
constexpr unsigned kFull = 0xffffffffu;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Extra device status bit: an `order` entry outside [0, B).
constexpr int kDevBadOrder = 8;

// ---- bf16 <-> fp32 -------------------------------------------------------------------
// A bf16 value is the upper half of a binary32: widening is a 16-bit shift.
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ void unpack8(const uint4& r, float (&f)[8]) {
  f[0] = bf_lo(r.x); f[1] = bf_hi(r.x);
  f[2] = bf_lo(r.y); f[3] = bf_hi(r.y);
  f[4] = bf_lo(r.z); f[5] = bf_hi(r.z);
  f[6] = bf_lo(r.w); f[7] = bf_hi(r.w);
}

// ---- global loads ---------------------------------------------------------------------
// 16-byte read-only loads of data touched once per launch: skip L1 allocation.
__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}
__device__ __forceinline__ float4 ld_stream_f4(const void* p) {
  float4 r;
  asm("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
      : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
      : "l"(p));
  return r;
}

// ---- ordering keys for scores ---------------------------------------------------------
// Monotone map fp32 -> uint32 (larger score -> larger key); -0 is folded onto +0 so that
// equal scores compare equal.
__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t u = __float_as_uint(s == 0.0f ? 0.0f : s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---- status ---------------------------------------------------------------------------
__device__ __forceinline__ void flag(int32_t* status, int bits) {
  if (status) atomicOr(status, bits);
}

// ---- block-wide exclusive scan (NT threads, scratch >= NT/32 ints) ---------------------
template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int v, int* scratch) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < NW ? scratch[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(kFull, wi, o);
      if (lane >= o) wi += y;
    }
    if (lane < NW) scratch[lane] = wi - w;
  }
  __syncthreads();
  int res = scratch[warp] + x - v;
  __syncthreads();
  return res;
}

// ---- exact top-k by radix select over 32-bit keys ---------------------------------------
// Finds the k-th largest key (k >= 1, k <= m) of keys[0..m) with 8-bit digits, most
// significant first.  On return: every key whose masked value is > prefix is in the top-k;
// keys whose masked value == prefix are all in it when take_all, else (mask is full) the
// `need` lowest-index ones are.  hist: 256 ints; info: 4 ints (shared).
template <int NT>
__device__ void radix_select(const uint32_t* keys, int m, int k, int* hist, int* info,
                             uint32_t& prefix, uint32_t& mask, int& need, bool& take_all) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  prefix = 0;
  mask = 0;
  need = k;
  take_all = false;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += NT) hist[i] = 0;
    __syncthreads();
    for (int j = tid; j < m; j += NT) {
      const uint32_t key = keys[j];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255], 1);
    }
    __syncthreads();
    if (warp == 0) {
      int cnt[8], tot = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        cnt[i] = hist[8 * lane + i];
        tot += cnt[i];
      }
      int incl = tot;  // sum over lanes >= lane (bins at or above this lane's)
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_down_sync(kFull, incl, o);
        if (lane + o < 32) incl += y;
      }
      const int above_lane = incl - tot;
      if (above_lane < need && need <= incl) {
        int acc = above_lane;
#pragma unroll
        for (int i = 7; i >= 0; --i) {
          if (acc + cnt[i] >= need) {
            info[0] = 8 * lane + i;
            info[1] = acc;
            info[2] = cnt[i];
            break;
          }
          acc += cnt[i];
        }
      }
    }
    __syncthreads();
    const int d = info[0], above = info[1], cnt_d = info[2];
    prefix |= (uint32_t)d << shift;
    mask |= 0xffu << shift;
    need -= above;
    if (cnt_d == need) {
      take_all = true;
      break;
    }
  }
  __syncthreads();
}

// Selected candidates in ascending index order: calls emit(j, position) for each of the k
// selected j (position in [0, k)).  Ties at the threshold go to the lowest indices.
template <int NT, typename Emit>
__device__ void emit_topk(const uint32_t* keys, int m, uint32_t prefix, uint32_t mask, int need,
                          bool take_all, int* scratch, Emit emit) {
  const int tid = threadIdx.x;
  const int per = (m + NT - 1) / NT;
  const int j0 = min(m, tid * per), j1 = min(m, j0 + per);
  int eq = 0;
  for (int j = j0; j < j1; ++j) eq += ((keys[j] & mask) == prefix);
  int eq_rank = block_exclusive_scan<NT>(eq, scratch);
  int cnt = 0;
  {
    int r = eq_rank;
    for (int j = j0; j < j1; ++j) {
      const uint32_t km = keys[j] & mask;
      const bool is_eq = km == prefix;
      cnt += (km > prefix) || (is_eq && (take_all || r < need));
      r += is_eq;
    }
  }
  int pos = block_exclusive_scan<NT>(cnt, scratch);
  int r = eq_rank;
  for (int j = j0; j < j1; ++j) {
    const uint32_t km = keys[j] & mask;
    const bool is_eq = km == prefix;
    if ((km > prefix) || (is_eq && (take_all || r < need))) emit(j, pos++);
    r += is_eq;
  }
}

// ---- online-softmax state merge (base-2 exponent) --------------------------------------
__device__ __forceinline__ void merge_scale(float ma, float mb, float& M, float& fa, float& fb) {
  M = fmaxf(ma, mb);
  fa = (ma == -INFINITY) ? 0.0f : exp2f(ma - M);
  fb = (mb == -INFINITY) ? 0.0f : exp2f(mb - M);
}

}  // namespace vt

namespace vt {

// ---- shared-memory addresses, async copies and warp-level MMA (sm_80+ forms) -----------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte global -> shared copy through L2 only; src_bytes == 0 writes zeros.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D(16x8, fp32) += A(16x16, bf16, row) * B(16x8, bf16, col)
__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

}  // namespace vt
