// Block-wide scans and the exact top-k radix select used by the selection steps.
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

// Exact top-k over n non-negative float keys held in shared memory as their bit
// patterns (bit order == value order for non-negative floats).  Finds the k-th
// largest key `kth` and `need` = how many keys equal to it are taken (the
// lowest-index ones), by an MSB-first 8-bit radix descent.  Runtime loops keep
// the code small.  Shared scratch: hist[512] (two alternating histograms, so the
// next pass's bins are cleared while this pass counts), info[2].
template <int NT>
__device__ __forceinline__ void radix_kth_smem(const uint32_t* keys, int n, int k, uint32_t* hist2,
                                               uint32_t* info, uint32_t* kth, uint32_t* need) {
  uint32_t prefix = 0, mask = 0;
  uint32_t kk = (uint32_t)k;
  for (int i = threadIdx.x; i < 256; i += NT) hist2[i] = 0;
  __syncthreads();
#pragma unroll 1
  for (int shift = 24, pass = 0; shift >= 0; shift -= 8, ++pass) {
    uint32_t* hist = hist2 + 256 * (pass & 1);
    uint32_t* next = hist2 + 256 * ((pass + 1) & 1);
    for (int i = threadIdx.x; i < 256; i += NT) next[i] = 0;
    // shared-memory atomics handle same-bin contention in hardware
#pragma unroll 1
    for (int j = threadIdx.x; j < n; j += NT) {
      const uint32_t key = keys[j];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      // lane owns digits [8*(31-lane), +8): lane 0 the highest digits
      const int base = 8 * (31 - lane);
      uint32_t c[8], s = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) { c[i] = hist[base + i]; s += c[i]; }
      uint32_t inc = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += t;
      }
      const uint32_t above = inc - s;  // keys with a higher digit than this lane's range
      if (above < kk && kk <= inc) {
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
  }
  __syncthreads();
  *kth = prefix;
  *need = kk;
}

// Exact k-th largest of n <= 4096 non-negative float keys (bit patterns) in shared
// memory, fast path: one counting pass over a 4096-bin histogram of the top 12 key
// bits (hist must be zero on entry; the sign bit is 0), a block scan to find the
// bin holding the k-th key, then the keys of that bin (usually a handful) are
// gathered and ranked.  When that bin holds more than 64 keys (heavy ties) it
// falls back to radix_kth_smem, reusing hist's first 512 words.  scratch: >= 200
// words of shared memory.  Results are identical to radix_kth_smem's.
template <int NT>
__device__ __forceinline__ void hist_kth_smem(const uint32_t* keys, int n, int k, uint32_t* hist,
                                              uint32_t* scratch, uint32_t* kth, uint32_t* need) {
  const int tid = threadIdx.x;
  if (tid == 0) scratch[66] = 0;  // candidate counter
#pragma unroll 1
  for (int j = tid; j < n; j += NT) atomicAdd(&hist[keys[j] >> 19], 1u);
  __syncthreads();
  // thread t owns the 4096/NT bins just below those of thread t-1 (thread 0: the top)
  constexpr int PER = 4096 / NT;
  static_assert(PER % 4 == 0, "bins per thread");
  const int base = 4096 - PER * (tid + 1);
  uint32_t c[PER];
#pragma unroll
  for (int i = 0; i < PER; i += 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(hist + base + i);
    c[i] = v.x; c[i + 1] = v.y; c[i + 2] = v.z; c[i + 3] = v.w;
  }
  uint32_t local = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) local += c[i];
  uint32_t total;
  const uint32_t above = block_excl_scan<NT>(local, scratch, &total);
  if (above < (uint32_t)k && (uint32_t)k <= above + local) {
    uint32_t a = above;
#pragma unroll
    for (int i = PER - 1; i >= 0; --i) {
      if (a < (uint32_t)k && (uint32_t)k <= a + c[i]) {
        scratch[64] = (uint32_t)(base + i);  // the bin
        scratch[65] = (uint32_t)k - a;       // rank of the k-th key inside the bin (1-based)
        scratch[67] = c[i];                  // keys in the bin
      }
      a += c[i];
    }
  }
  __syncthreads();
  const uint32_t bin = scratch[64], rem = scratch[65], cnt = scratch[67];
  if (cnt > 64) {  // rare (heavy ties): exact fallback
    __syncthreads();
    radix_kth_smem<NT>(keys, n, k, hist, scratch + 68, kth, need);
    return;
  }
  // gather the bin's keys (any order) with their indices
  uint32_t* ck = scratch + 72;        // [64]
  uint32_t* ci = scratch + 72 + 64;   // [64]
#pragma unroll 1
  for (int j = tid; j < n; j += NT) {
    const uint32_t key = keys[j];
    if ((key >> 19) == bin) {
      const uint32_t slot = atomicAdd(&scratch[66], 1u);
      ck[slot] = key;
      ci[slot] = (uint32_t)j;
    }
  }
  __syncthreads();
  // rank inside the bin by (key desc, index asc); the k-th has rank rem - 1
  if (tid < (int)cnt) {
    const uint32_t mk = ck[tid], mi = ci[tid];
    uint32_t rank = 0, gt = 0;
#pragma unroll 4
    for (int i = 0; i < (int)cnt; ++i) {
      const uint32_t ok_ = ck[i], oi = ci[i];
      rank += (ok_ > mk) || (ok_ == mk && oi < mi);
      gt += ok_ > mk;
    }
    if (rank == rem - 1) { scratch[68] = mk; scratch[69] = rem - gt; }
  }
  __syncthreads();
  *kth = scratch[68];
  *need = scratch[69];
}

// Given the k-th key and how many of the equal keys to take, write the selected
// indices (ascending) to sel[0..k).  Thread t owns the contiguous index range
// [t*ept, (t+1)*ept).  Returns the number written by the block (== k).
template <int NT>
__device__ __forceinline__ void scatter_topk(const uint32_t* keys, int n, uint32_t kth,
                                             uint32_t need, uint16_t* sel, uint32_t* scan_tmp) {
  const int ept = (n + NT - 1) / NT;
  const int j0 = threadIdx.x * ept, j1 = min(n, j0 + ept);
  uint32_t ngt = 0, neq = 0;
#pragma unroll 1
  for (int j = j0; j < j1; ++j) { ngt += keys[j] > kth; neq += keys[j] == kth; }
  uint32_t tot;
  const uint32_t pre = block_excl_scan<NT>(ngt | (neq << 16), scan_tmp, &tot);
  uint32_t gtb = pre & 0xffffu, eqb = pre >> 16;
#pragma unroll 1
  for (int j = j0; j < j1; ++j) {
    const bool gt = keys[j] > kth, eq = keys[j] == kth;
    if (gt || (eq && eqb < need)) sel[gtb + min(eqb, need)] = (uint16_t)j;
    gtb += gt;
    eqb += eq;
  }
}

}  // namespace msb
