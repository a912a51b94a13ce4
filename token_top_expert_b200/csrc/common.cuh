// Shared device helpers for the sparse-MoE block kernels (sm_100a).
//
// PTX wrappers for mbarriers, 1-D bulk async copies (no multicast), the
// bf16 tensor-core MMA used for sketch scoring, cluster/DSMEM access, and
// the packed-format constants shared by the packer and the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "msb.h"

namespace msb {

// ---------------------------------------------------------------- packed sketch format
// Rows are grouped in tiles of 16 and columns in chunks of 64.  One (tile, chunk)
// is 64 uint32 = 256 bytes, stored as [lane 0..31][h 0..1]: lane = 4*g + c
// (g = 0..7, c = 0..3), h = 0 holds row 16*tile + g, h = 1 row 16*tile + g + 8.
// A word holds 8 element pairs q = 0..7, q = 2*s + p (s = 16-column step 0..3,
// p = 0/1): the pair covers columns 64*chunk + 16*s + 2*c + 8*p and the next one.
// The low element's 2-bit code sits at bits (15-2q, 14-2q) = (sign, magnitude),
// the high element's at bits (31-2q, 30-2q).  T = +1 -> (0,1), -1 -> (1,1), 0 -> (0,0).
// Hence (word << 2q) & 0xC000C000 is the bf16x2 pair (2*T_lo, 2*T_hi): the A
// fragment of mma.m16n8k16 for that step, with no further decoding.
constexpr int kRowTile = 16;
constexpr int kColChunk = 64;
constexpr int kChunkWords = 64;
constexpr uint32_t kSketchMask = 0xC000C000u;

__host__ __device__ inline int pad16(int v) { return (v + 15) & ~15; }
// 32-bit words of a per-channel bitmask over ipad channels
__host__ __device__ inline int mask_words(int ipad) { return (ipad + 31) / 32; }

// ---------------------------------------------------------------- device error word
constexpr uint32_t kErrTimeout = 1u;
constexpr uint32_t kErrNonFinite = 2u;  // router saw NaN/Inf logits (invalid input)
constexpr uint32_t kErrInternal = 4u;   // a kernel's consistency check failed (a selection of
                                        // the wrong size); the offending access was skipped
constexpr uint32_t kSpinLimit = 1u << 22;            // polls before a wait gives up ...
constexpr uint64_t kWaitLimitNs = 2000ull * 1000000;  // ... or 2 s of wall time, whichever first

// ---------------------------------------------------------------- small PTX wrappers
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// arrive (count 1) and add `bytes` to the barrier's expected transaction count
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// As mbar_try_wait, but a thread whose phase is not complete may sleep for up to
// `hint_ns` before the call returns false (it wakes as soon as the phase completes), so
// that a waiting warp takes no issue slots from the warps that work meanwhile.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for phase `parity` of the barrier, bounded by a poll count and by wall time
// (limit_ns).  On expiry sets the sticky error word and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* err,
                                          uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1; i < kSpinLimit; ++i) {
    if (mbar_try_wait_sleep(bar, parity, 2000u)) return true;
    if ((i & 15u) == 0 && globaltimer_ns() - t0 > limit_ns) break;
  }
  atomicOr(err, kErrTimeout);
  return false;
}

// 1-D bulk copy global -> this CTA's shared memory, completion counted on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.  No multicast.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Prefetch `bytes` (multiple of 16, 16-byte aligned) of global memory into L2.
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// D += A*B with A 16x16 bf16 (row), B 16x8 bf16 (col), D 16x8 fp32.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Four 8x8 b16 matrices from shared memory (lane l gives the address of row l % 8 of
// matrix l / 8); register j holds matrix j in the mma fragment layout.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// vector reduction-add of 4 floats into global memory (16-byte aligned)
__device__ __forceinline__ void red_add_v4(float* dst, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(dst), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// 8 bf16 (one uint4) dot 8 bf16, fp32 accumulate
__device__ __forceinline__ float dot8(uint4 a, uint4 b, float acc) {
  acc = fmaf(bf16_lo(a.x), bf16_lo(b.x), acc);
  acc = fmaf(bf16_hi(a.x), bf16_hi(b.x), acc);
  acc = fmaf(bf16_lo(a.y), bf16_lo(b.y), acc);
  acc = fmaf(bf16_hi(a.y), bf16_hi(b.y), acc);
  acc = fmaf(bf16_lo(a.z), bf16_lo(b.z), acc);
  acc = fmaf(bf16_hi(a.z), bf16_hi(b.z), acc);
  acc = fmaf(bf16_lo(a.w), bf16_lo(b.w), acc);
  acc = fmaf(bf16_hi(a.w), bf16_hi(b.w), acc);
  return acc;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float silu(float g) { return g / (1.0f + expf(-g)); }

// ---------------------------------------------------------------- workspace layout
// Fixed header (same offsets for every batch size): error word, counters, y_acc.
struct Workspace {
  uint32_t* err;        // sticky error word
  uint32_t* counters;   // [kCounters] arrival counters (zero between calls)
  float* y_acc;         // [B][d] fp32 output accumulator (zero between calls)
  float* logits;        // [B][E]
  int32_t* ids;         // [B][K]
  float* wts;           // [B][K]
  int32_t* slot_expert; // [E] expert of used slot u (ascending expert order)
  int32_t* slot_off;    // [E+1] first pair of slot u
  int32_t* nused;       // [1]
  int32_t* pair_tok;    // [B*K] token of pair p (pairs sorted by (expert, token))
  float* pair_w;        // [B*K] combine weight of pair p
  int32_t* pair_slot;   // [B*K]
  int32_t* pair_of;     // [B][K] pair index of (token, rank)
  float* scores;        // [B*K][Ipad]
  uint32_t* selmask;    // [B*K][Ipad/32]
  uint16_t* sel;        // [B*K][Ipad]
  int32_t* selcnt;      // [B*K]
  uint32_t* umask;      // [E][Ipad/32] union of the selections of each slot
  float* z;             // [B*K][r]  B_e x
  uint16_t* ulist;      // [E][Ipad] ascending union list of each slot
  int32_t* ucnt;        // [E] union size of each slot
  int32_t* coff;        // [E+1] first gather work item (channel chunk) of each slot
};

constexpr int kCounters = 1024;
// counter indices
constexpr int kCntRouterAll = 1;      // router: token groups finished
constexpr int kCntRouterGroup = 8;    // router: CTAs finished per token group (32 groups)
constexpr int kCntFusedSlices = 64;   // single-launch path: contributions per output slice (16)
constexpr int kCntGatherWork = 2;     // multi-kernel path: next gather work item
constexpr int kCntUnion = 3;          // multi-kernel path: union CTAs finished
constexpr int kCntGatherRun = 4;      // multi-kernel path: union channels per gather work item

struct Dims {
  int d, inter, ipad, experts, top_e, rank, renorm;
};

// Device pointers of the optional trace (all may be null).
struct TraceDev {
  int32_t* expert_ids;
  float* expert_w;
  uint16_t* sel;
  int32_t* sel_count;
  int32_t* union_count;
  float* scores;
};

}  // namespace msb
