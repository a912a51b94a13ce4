// Block-wide scans and the exact top-k radix select used by the selection kernels.
#pragma once

#include "common.cuh"

namespace msb {

// Exclusive prefix sum over the block (blockDim.x == NT, NT multiple of 32, <= 1024).
// `tmp` must hold NT/32 + 1 ints of shared memory.  Returns the exclusive prefix of
// `v` and writes the block total to *total.
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* tmp, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  if (lane == 31) tmp[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < NT / 32 ? tmp[lane] : 0u;
    uint32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    if (lane < NT / 32) tmp[lane] = wi - w;
    if (lane == NT / 32 - 1) tmp[NT / 32] = wi;
  }
  __syncthreads();
  uint32_t res = tmp[warp] + inc - v;
  *total = tmp[NT / 32];
  __syncthreads();
  return res;
}

// Exact top-k over non-negative float keys given as their bit patterns (bit
// order == value order for non-negative floats).  Each thread holds up to EPT
// keys of a contiguous index range; `valid` masks entries beyond n.
// Finds the k-th largest key `kth` and `need` = how many keys equal to it are
// taken (the lowest-index ones), by an MSB-first 8-bit radix descent.
// Shared scratch: hist[256], info[4].
template <int NT, int EPT>
__device__ __forceinline__ void radix_kth(const uint32_t (&key)[EPT], uint32_t valid, int k,
                                          uint32_t* hist, uint32_t* info, uint32_t* kth,
                                          uint32_t* need) {
  uint32_t prefix = 0, mask = 0;
  uint32_t kk = (uint32_t)k;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += NT) hist[i] = 0;
    __syncthreads();
#pragma unroll
    for (int m = 0; m < EPT; ++m)
      if (((valid >> m) & 1u) && (key[m] & mask) == prefix) atomicAdd(&hist[(key[m] >> shift) & 255u], 1u);
    __syncthreads();
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      // lane owns digits [8*(31-lane), 8*(31-lane)+8): lane 0 the highest digits
      const int base = 8 * (31 - lane);
      uint32_t c[8], s = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) { c[i] = hist[base + i]; s += c[i]; }
      // inclusive scan over lanes (lane 0 = highest digits)
      uint32_t inc = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint32_t n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
      }
      uint32_t above = inc - s;  // keys with a digit higher than this lane's range
      // the digit D with above(D) < kk <= above(D) + hist[D], scanning down from the top
      bool mine = above < kk && kk <= inc;
      if (mine) {
        uint32_t a = above;
#pragma unroll
        for (int i = 7; i >= 0; --i) {
          if (a < kk && kk <= a + c[i]) { info[0] = (uint32_t)(base + i); info[1] = kk - a; }
          a += c[i];
        }
      }
    }
    __syncthreads();
    prefix |= info[0] << shift;
    mask |= 255u << shift;
    kk = info[1];
    __syncthreads();
  }
  *kth = prefix;
  *need = kk;
}

}  // namespace msb
