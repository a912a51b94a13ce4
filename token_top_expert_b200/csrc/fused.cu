// Single-launch sparse-MoE block for decode batches of up to 16 tokens (the hot path).
//
// One thread-block cluster per (token, routed expert) pair: 16 CTAs for one token, 8
// for several (so that a batch is resident in about one wave).  Every exchange inside a
// cluster is a one-way push: the producer writes into the consumers' shared memory with
// st.async / red.async, and each consumer waits on its own mbarrier for the exact byte
// count it expects, so no exchange costs a cluster-wide barrier.  Across clusters only
// FP32 reduction-adds into the token's accumulator row meet; the last contribution to an
// output slice writes it as BF16.
//
//  A  router: each CTA computes its E/cs logits x . W_router[e] (rows staged by bulk
//     copies before the grid dependency wait) and pushes them to every CTA; the CTA
//     owning a logit ranks it exactly against all E and pushes the K winners into every
//     CTA's rank table; cluster c of the token takes its c-th expert.
//  B  z = B_e x (pushed) while the sketch tiles are in flight; then the sketch scores of
//     the CTA's 16-row tiles on the tensor cores (the packed codes are the bf16 A
//     fragment), pushed with one max per warp to every CTA.
//  C  exact top-k: every CTA selects the same k channels (histogram below the cluster's
//     largest score, ballot prefixes, the k-th key's bin ranked directly when it is not
//     taken whole; ties to the lower index); the CTAs interleave over the ascending list
//     and issue bulk copies of their channel records; A_e z on the CTA's output slice.
//  D  records in batches as they land (BF16 or 4-bit group-affine records): gate.x and
//     up.x on the CUDA cores with one transposed warp reduction per batch, h =
//     silu(gate.x) * up.x, and every thread adds h * down over its 8-element groups.
//  E  combine: each CTA pushes its partial output, slice by slice, to the slice's owner;
//     the owner sums the partials, adds A_e z, scales by the router weight and
//     reduction-adds into the FP32 accumulator; the last of the K contributions to a
//     slice converts it to BF16 and re-zeroes it.
//
// x comes from device memory (one bulk copy) or, for pinned and mapped host buffers,
// from the host link (each CTA reads a piece and pushes it to the cluster).  The launch
// uses programmatic stream serialisation: barrier set-up and the router rows' copy (and
// x, when the caller declared it ready) run before griddepcontrol.wait.  Every wait is
// bounded; an expired wait sets the sticky error word and the CTA still takes every
// exchange and barrier step.
//
// "KAIST drops calibration from MoE decoding ...": "Top-k instead of a threshold"
// (fixed read budget), "A reader built from weights alone" (ternary sketch filter
// + low-rank compensation).  No TMA multicast and no peer memory is used.
#include "block_scan.cuh"
#include "common.cuh"
#include "fused.h"
#include "launch.h"

namespace msb {

constexpr int kFT = 256;       // threads per CTA
constexpr int kFW = kFT / 32;  // warps per CTA
constexpr int kRingMax = 16;   // record slots
constexpr int kSmemMax = 227 * 1024;
constexpr int kSmemPair = 113 * 1024;  // fallback pairing limit if the device cannot be queried
constexpr int kSelBins = 2048;         // select histogram: 256 bins per octave below the largest key
constexpr int kSelShift = 15;
constexpr int kCandMax = 64;           // keys of the k-th key's bin ranked directly
constexpr int kWordsMax = (MSB_MAX_INTER + 31) / 32;
constexpr int kMyselMax = 512;         // channels one CTA reads at most
#ifdef MSB_INSTRUMENTED
constexpr int kMarks = 16;             // phase marks per CTA
#endif

// mbarriers: fixed ones, then one per record slot
enum { kBarRows = 0, kBarX, kBarLogits, kBarIds, kBarSketch, kBarLow, kBarScores, kBarZ, kBarY, kBarRing };

struct FusedParams {
  const uint16_t* x;
  const uint16_t* router_t;
  const uint16_t* records;
  const uint32_t* sketch;
  const float* alpha;
  const uint16_t* lr_a;
  const uint16_t* lr_b;
  uint16_t* out;
  uint32_t* err;
  uint32_t* slice_cnt;  // [cs] arrival counters, one per output slice
  float* y_acc;         // [d] FP32 accumulator, zero between calls
#ifdef MSB_INSTRUMENTED
  unsigned long long* marks;  // [grid][kMarks] phase timestamps, or null
  uint32_t skip;              // 1: CTA 0 never issues its first record copy
  uint64_t wait_ns;           // bounded-wait limit
#endif
  TraceDev tr;
  Dims D;
  int k, dense, cs;
  int rpc;     // router rows per CTA
  int tpc;     // sketch row tiles per CTA
  int slice;   // output elements owned per CTA (d / cs)
  int ring;    // record slots
  int rs;      // ring slot stride (elements): 3d + 8, so that the rows of consecutive slots
               // fall 16 bytes apart in the shared-memory banks (conflict-free ldmatrix)
  int rrs;     // router row stride in shared memory (elements): d + 8, for the same reason
  int epad;    // logits padded to a multiple of 64 (with -inf)
  // shared-memory carve-up (byte offsets from the dynamic base)
  int o_misc, o_lr, o_rbuf, o_mysel, o_big;
  int o_x, o_xperm, o_logits, o_keys, o_hist, o_part;  // inside big (phases A-C)
  int o_alpha, o_brows;                                  // inside big (phase B)
  int smem;
  uint32_t x1_bytes, sc_bytes, z_bytes, y_bytes;  // bytes each CTA expects per exchange
  int q4;        // records are 4-bit (group-wise affine, 64 weights per group)
  uint32_t rec_bytes;  // bytes of one channel record (6d for BF16)
  int x_ready;   // nothing earlier on the stream writes x: fetch it before the grid
                 // dependency wait
  int x_mapped;  // x and out are pinned host memory mapped into the device's address space:
                 // each CTA reads its piece of x over the host link and pushes it to the
                 // cluster; out is written across the link by the slices' last contributors
};

struct Misc {
  uint64_t bar[kBarRing + kRingMax];
  uint2 rk[MSB_MAX_TOP_E];  // routed experts in rank order: (expert id, logit bits), pushed
                            // by the CTA that owns the expert's router row
  float wk[MSB_MAX_TOP_E];  // combine weights of the routed experts, rank order
  uint32_t cmax, kb, rem, cnt, ccount, kth, need;
  uint32_t info[2];
  uint32_t wt[kFW];
  float red8[kFW][8];    // per-warp sums of up to 8 dot products (logits; gate/up of a batch)
  float h[8];            // h of a batch's records
  uint32_t ck[kCandMax], ci[kCandMax];
  uint32_t csel[kWordsMax];  // selected keys of the k-th key's bin
  uint32_t selw[kWordsMax];  // selection bitmap over the channels
  uint32_t pref[kWordsMax];  // exclusive prefix of popc(selw)
  float z[MSB_MAX_RANK];     // B_e x
  int last;
};

// the kernel's dynamic shared memory (carved up by the offsets in FusedParams)
extern __shared__ __align__(128) uint8_t g_sm[];
// this CTA's share of the selected channels (positions q, q + cs, q + 2 cs, ... of the
// ascending list)
#define MYSEL(P) reinterpret_cast<uint16_t*>(g_sm + (P).o_mysel)

// ---------------------------------------------------------------- cluster PTX
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// address of the same shared-memory location in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa(uint32_t a, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}
// remote store of one word, completion counted (4 bytes) on the remote mbarrier
__device__ __forceinline__ void st_async(uint32_t ra, uint32_t v, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(ra),
               "r"(v), "r"(rbar)
               : "memory");
}
__device__ __forceinline__ void st_async2(uint32_t ra, uint32_t a, uint32_t b, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.b32 [%0], {%1,%2}, [%3];" ::"r"(ra),
               "r"(a), "r"(b), "r"(rbar)
               : "memory");
}
__device__ __forceinline__ void st_async4(uint32_t ra, float a, float b, float c, float d, uint32_t rbar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1,%2,%3,%4}, [%5];" ::"r"(ra),
      "f"(a), "f"(b), "f"(c), "f"(d), "r"(rbar)
      : "memory");
}
// remote max of one word, completion counted (4 bytes) on the remote mbarrier
__device__ __forceinline__ void red_async_max(uint32_t ra, uint32_t v, uint32_t rbar) {
  asm volatile(
      "red.async.relaxed.cluster.shared::cluster.mbarrier::complete_tx::bytes.max.u32 [%0], %1, [%2];" ::"r"(
          ra),
      "r"(v), "r"(rbar)
      : "memory");
}
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
// arrive without release semantics: orders nothing, only counts (the exchanges it follows
// are each tracked by the receiver's own mbarrier)
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// atomic add with acquire-release semantics at GPU scope; returns the old value
__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
// 16-byte load that bypasses L1 (pinned host memory the host rewrites between calls:
// a CTA never meets a line an earlier launch left in its SM); loads of a warp coalesce
// into one transfer across the host link
__device__ __forceinline__ uint4 ld_fresh16(const void* p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

#ifdef MSB_INSTRUMENTED
#define MARK(i)                                                                \
  do {                                                                         \
    if (P.marks && threadIdx.x == 0) P.marks[blockIdx.x * kMarks + (i)] = globaltimer_ns(); \
  } while (0)
#define WAIT_LIMIT (P.wait_ns)
#else
#define MARK(i) \
  do {          \
  } while (0)
#define WAIT_LIMIT kWaitLimitNs
#endif

// Bounded wait: the common case (phase already complete) inline, the spin out of line.
__device__ __noinline__ bool wait_slow(uint64_t* bar, uint32_t parity, uint32_t* err, uint64_t limit) {
  return mbar_wait(bar, parity, err, limit);
}
#define wait_phase(bar, parity, err) \
  (mbar_try_wait((bar), (parity)) || wait_slow((bar), (parity), (err), WAIT_LIMIT))

// Order-preserving key of a logit: integer order is value order, -0 equals +0, and a
// NaN ranks below everything.
__device__ __forceinline__ uint32_t logit_key(float v) {
  uint32_t b = __float_as_uint(v);
  if (v != v) return 0u;
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Router top-K, distributed over the cluster: the CTA that owns router rows [e_lo, e_hi)
// ranks each of its logits exactly against all E (rank = #{e' : l_e' > l_e} + #{e' < e :
// l_e' == l_e}, one warp per logit, one ballot per 32 logits) and, for a rank r < K,
// pushes (e, l_e) into slot r of every CTA's M.rk.  The ranks form a permutation of 0..E-1,
// so every CTA receives exactly K pushes.  A non-finite logit flags the call.
__device__ __forceinline__ void router_rank(const FusedParams& P, const float* logits, int q) {
  Misc& M = *reinterpret_cast<Misc*>(g_sm + P.o_misc);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = P.D.experts, K = P.D.top_e;
  const int e_lo = min(E, q * P.rpc), e_hi = min(E, e_lo + P.rpc);
  const uint32_t rbar = smem_addr(&M.bar[kBarIds]);
#pragma unroll 1
  for (int ee = e_lo + warp; ee < e_hi; ee += kFW) {
    const float v = logits[ee];
    const uint32_t kv = logit_key(v);
    uint32_t rank = 0;
#pragma unroll 4
    for (int j0 = 0; j0 < E; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t ku = j < E ? logit_key(logits[j]) : 0u;
      rank += (uint32_t)__popc(__ballot_sync(0xffffffffu, j < E && (ku > kv || (ku == kv && j < ee))));
    }
    if (lane == 0 && !isfinite(v)) atomicOr(P.err, kErrNonFinite);
    if (rank < (uint32_t)K && lane < P.cs)
      st_async2(mapa(smem_addr(&M.rk[rank]), lane), (uint32_t)ee, __float_as_uint(v), mapa(rbar, lane));
  }
}

// Warp 0, after the routing: the combine weights of the K routed experts into M.wk
// (rank order): softmax over the K routed logits (renorm) or over all E logits.
// rk[0] holds the largest logit.
__device__ __noinline__ void router_weights(const float* logits, int E, int K, int renorm, Misc& M) {
  const int lane = threadIdx.x & 31;
  const float mx = __uint_as_float(M.rk[0].y);
  const float pl = lane < K ? __expf(__uint_as_float(M.rk[lane].y) - mx) : 0.f;
  float denom = 0.f;
  if (renorm) {
    denom = pl;
  } else {
#pragma unroll 1
    for (int i = lane; i < E; i += 32) denom += __expf(logits[i] - mx);
  }
  denom = warp_sum(denom);
  if (lane < K) M.wk[lane] = __fdividef(pl, denom);
}

// Trace of token tok's routing (one CTA): expert ids, weights, and the channels read per
// expert.
// (The per-expert union count is written for a single token; batches that trace it take
// the multi-kernel path.)
__device__ __noinline__ void trace_routing(const TraceDev& tr, const Misc& M, int E, int K, int k, int tok) {
  const int tid = threadIdx.x;
  if (tid < K && tr.expert_ids) tr.expert_ids[tok * K + tid] = (int)M.rk[tid].x;
  if (tid < K && tr.expert_w) tr.expert_w[tok * K + tid] = M.wk[tid];
  if (tr.union_count)
#pragma unroll 1
    for (int i = tid; i < E; i += kFT) {
      int c = 0;
#pragma unroll 1
      for (int j = 0; j < K; ++j) c = ((int)M.rk[j].x == i) ? k : c;
      tr.union_count[i] = c;
    }
}

// Sketch scores of this CTA's nt row tiles: warp w takes chunks [kc0, kc1) of every
// tile; the packed 2-bit codes are the bf16 A fragments (+-2 or 0), x is B.
// Partial sums go to part_w[tile*16 + row].
__device__ __noinline__ void score_tiles(const uint2* codes, const uint4* xperm, int nt, int KC,
                                         float* part_w) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kc0 = warp * KC / kFW, kc1 = (warp + 1) * KC / kFW;
  const int g = lane >> 2, c = lane & 3;
  const uint4* xp = xperm + c * 2;
#pragma unroll 1
  for (int tl = 0; tl < nt; ++tl) {
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 2
    for (int kc = kc0; kc < kc1; ++kc) {
      const uint2 w = codes[((size_t)tl * KC + kc) * 32 + lane];
      uint4 xa = make_uint4(0u, 0u, 0u, 0u), xb = xa;
      if (g == 0) { xa = xp[kc * 8]; xb = xp[kc * 8 + 1]; }
      // four independent 16-column steps (no accumulator chain between them)
      float m0[4] = {0.f, 0.f, 0.f, 0.f}, m1[4] = {0.f, 0.f, 0.f, 0.f};
      float m2[4] = {0.f, 0.f, 0.f, 0.f}, m3[4] = {0.f, 0.f, 0.f, 0.f};
      mma_bf16(m0, w.x & kSketchMask, w.y & kSketchMask, (w.x << 2) & kSketchMask,
               (w.y << 2) & kSketchMask, xa.x, xa.y);
      mma_bf16(m1, (w.x << 4) & kSketchMask, (w.y << 4) & kSketchMask, (w.x << 6) & kSketchMask,
               (w.y << 6) & kSketchMask, xa.z, xa.w);
      mma_bf16(m2, (w.x << 8) & kSketchMask, (w.y << 8) & kSketchMask, (w.x << 10) & kSketchMask,
               (w.y << 10) & kSketchMask, xb.x, xb.y);
      mma_bf16(m3, (w.x << 12) & kSketchMask, (w.y << 12) & kSketchMask, (w.x << 14) & kSketchMask,
               (w.y << 14) & kSketchMask, xb.z, xb.w);
      acc0 += (m0[0] + m1[0]) + (m2[0] + m3[0]);
      acc1 += (m0[2] + m1[2]) + (m2[2] + m3[2]);
    }
    if (c == 0) {
      part_w[tl * kRowTile + g] = acc0;
      part_w[tl * kRowTile + g + 8] = acc1;
    }
  }
}

__device__ __forceinline__ uint32_t sel_bin(uint32_t maxkey, uint32_t key) {
  return min((uint32_t)(kSelBins - 1), (maxkey - key) >> kSelShift);
}

// Heavy ties in the k-th key's bin (more than kCandMax keys): exact radix descent
// over all keys, then warp 0 walks the words in index order and takes the equal
// keys lowest index first.  Writes M.selw.  Ends with a barrier.
__device__ __noinline__ void select_fallback(const uint32_t* keys, int n, int k, uint32_t* hist,
                                             Misc& M) {
  uint32_t kth, need;
  radix_kth_smem<kFT>(keys, n, k, hist, M.info, &kth, &need);
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    uint32_t taken = 0;
#pragma unroll 1
    for (int c = 0; c < (n + 31) / 32; ++c) {
      const int j = 32 * c + lane;
      const uint32_t key = j < n ? keys[j] : 0u;
      const uint32_t gtb = __ballot_sync(0xffffffffu, j < n && key > kth);
      const uint32_t eqb = __ballot_sync(0xffffffffu, j < n && key == kth);
      uint32_t take = 0;
      if (taken < need) {
        const uint32_t left = need - taken;
        if ((uint32_t)__popc(eqb) <= left) {
          take = eqb;
        } else {  // the `left` lowest set bits of eqb
          const uint32_t top = __fns(eqb, 0, (int)left);
          take = eqb & (top >= 31 ? 0xffffffffu : ((2u << top) - 1u));
        }
      }
      taken += (uint32_t)__popc(take);
      if (lane == 0) M.selw[c] = gtb | take;
    }
  }
  __syncthreads();
}

// Exclusive prefix over the warp of v (v < 2^NB) by bit-sliced ballots: no shuffle chain.
template <int NB>
__device__ __forceinline__ uint32_t warp_excl_prefix(uint32_t v) {
  const uint32_t lt = (1u << (threadIdx.x & 31)) - 1u;
  uint32_t pre = 0;
#pragma unroll
  for (int b = 0; b < NB; ++b) pre += (uint32_t)__popc(__ballot_sync(0xffffffffu, (v >> b) & 1u) & lt) << b;
  return pre;
}

// Exact top-k of the n channel keys (float bits of non-negative scores, so integer
// order is value order), ties to the lower index, as a bitmap M.selw over the
// channels.  Keys are binned by (maxkey - key) >> 15 (256 bins per octave below the
// largest key, bin 0 the largest, the last bin catching the rest); one counting pass,
// per-warp bin totals and a ballot prefix find the bin of the k-th key.  If that bin
// is taken whole the bitmap is one ballot per word; otherwise its keys are ranked
// directly (ties to the lower index).  Key j is read by thread j % 256, so a warp's
// ballot over one stride of 256 keys is one bitmap word.  hist (kSelBins words), M.csel
// and M.ccount must be zero on entry.  Ends with a barrier.
__device__ __noinline__ void select_topk(const uint32_t* keys, int n, int k, uint32_t maxkey,
                                         uint32_t* hist, Misc& M) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
#pragma unroll 1
  for (int j = tid; j < n; j += kFT) atomicAdd(&hist[sel_bin(maxkey, keys[j])], 1u);
  __syncthreads();
  // thread t owns bins [8t, 8t + 8): warp totals, then the warp and lane of the k-th key
  const uint4 h0 = reinterpret_cast<const uint4*>(hist)[2 * tid];
  const uint4 h1 = reinterpret_cast<const uint4*>(hist)[2 * tid + 1];
  const uint32_t local = ((h0.x + h0.y) + (h0.z + h0.w)) + ((h1.x + h1.y) + (h1.z + h1.w));
  const uint32_t wtot = __reduce_add_sync(0xffffffffu, local);
  if (lane == 0) M.wt[warp] = wtot;
  __syncthreads();
  uint32_t above = 0;
#pragma unroll
  for (int w = 0; w < kFW; ++w) above += w < warp ? M.wt[w] : 0u;
  const uint32_t kk = (uint32_t)k;
  if (above < kk && kk <= above + wtot) {  // (warp-uniform)
    above += warp_excl_prefix<13>(local);  // local <= n <= 4096
    if (above < kk && kk <= above + local) {
      const uint32_t c[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (above < kk && kk <= above + c[i]) { M.kb = 8 * tid + i; M.rem = kk - above; M.cnt = c[i]; }
        above += c[i];
      }
    }
  }
  __syncthreads();
  const uint32_t kb = M.kb, rem = M.rem, cnt = M.cnt;
  const bool whole = (cnt == rem);
  if (!whole) {
    if (cnt > (uint32_t)kCandMax) {
      select_fallback(keys, n, k, hist, M);
      return;
    }
    // the keys of bin kb with their indices (warp-aggregated slots), each ranked among
    // them by (key desc, index asc); the first `rem` are taken
    const uint32_t lt = (1u << lane) - 1u;
#pragma unroll 1
    for (int j0 = warp * 32; j0 < n; j0 += kFT) {
      const int j = j0 + lane;
      const uint32_t key = j < n ? keys[j] : 0u;
      const bool m = j < n && sel_bin(maxkey, key) == kb;
      const uint32_t mb = __ballot_sync(0xffffffffu, m);
      if (mb) {
        const int leader = __ffs(mb) - 1;
        uint32_t slot0 = 0;
        if (lane == leader) slot0 = atomicAdd(&M.ccount, (uint32_t)__popc(mb));
        slot0 = __shfl_sync(0xffffffffu, slot0, leader) + __popc(mb & lt);
        if (m) {
          M.ck[slot0] = key;
          M.ci[slot0] = (uint32_t)j;
        }
      }
    }
    __syncthreads();
    if (tid < (int)cnt) {
      const uint32_t mk = M.ck[tid], mi = M.ci[tid];
      uint32_t rank = 0;
#pragma unroll 1
      for (int i = 0; i < (int)cnt; ++i) {
        const uint32_t ok_ = M.ck[i];
        rank += (ok_ > mk) || (ok_ == mk && M.ci[i] < mi);
      }
      if (rank < rem) atomicOr(&M.csel[mi >> 5], 1u << (mi & 31));
    }
    __syncthreads();
  }
  // the bitmap: word 8 s + w is warp w's ballot over stride s
#pragma unroll 1
  for (int j0 = warp * 32; j0 < n; j0 += kFT) {
    const int j = j0 + lane;
    const uint32_t b = j < n ? sel_bin(maxkey, keys[j]) : 0xffffffffu;
    const uint32_t w = __ballot_sync(0xffffffffu, b < kb || (whole && b == kb));
    if (lane == 0) M.selw[j0 >> 5] = whole ? w : (w | M.csel[j0 >> 5]);
  }
  __syncthreads();
}

// Warp 0: each selection word's exclusive prefix of popcounts into M.pref (ballot
// prefix, 32 words at a time).  A selection of the wrong size (not k channels) flags the
// call and fills this CTA's share with channel 0 (positions_place then overwrites what
// it can).
__device__ __noinline__ void positions_prefix(int nw, int k, int nmine, Misc& M, uint16_t* mysel, uint32_t* err) {
  const int lane = threadIdx.x & 31;
  uint32_t carry = 0;
#pragma unroll 1
  for (int cb = 0; cb < nw; cb += 32) {
    const int c = cb + lane;
    const uint32_t cnt = c < nw ? (uint32_t)__popc(M.selw[c]) : 0u;
    const uint32_t p = carry + warp_excl_prefix<6>(cnt);
    if (c < nw) M.pref[c] = p;
    carry = __shfl_sync(0xffffffffu, p + cnt, 31);
  }
  if (carry != (uint32_t)k) {
#pragma unroll 1
    for (int t = lane; t < nmine; t += 32) mysel[t] = 0;
    if (lane == 0) atomicOr(err, kErrInternal);
  }
}

// All threads, after positions_prefix and a barrier: this CTA's share of the ascending
// selected list into mysel -- the channels at positions p = q + t * 2^lgcs (t < nmine),
// so that the CTAs of the cluster interleave over the list.  Thread j % 256 places
// channel j: its position is its word's prefix plus the set bits below it.
__device__ __forceinline__ void positions_place(int n, int q, int lgcs, int nmine, const Misc& M, uint16_t* mysel) {
  const uint32_t cm = (1u << lgcs) - 1u;
#pragma unroll 1
  for (int j = threadIdx.x; j < n; j += kFT) {
    const uint32_t w = M.selw[j >> 5], bit = 1u << (j & 31);
    if (w & bit) {
      const uint32_t p = M.pref[j >> 5] + (uint32_t)__popc(w & (bit - 1u));
      if ((p & cm) == (uint32_t)q && (p >> lgcs) < (uint32_t)nmine) mysel[p >> lgcs] = (uint16_t)j;
    }
  }
}

// Warp 0 of one CTA per cluster: the pair's whole ascending selected list (k entries)
// and its size into trace row rc (dense: every channel).
__device__ __noinline__ void trace_selection(const FusedParams& P, const Misc& M, int nw, int rc) {
  const int lane = threadIdx.x & 31, k = P.k;
  if (lane == 0 && P.tr.sel_count) P.tr.sel_count[rc] = k;
  if (!P.tr.sel) return;
  uint16_t* out = P.tr.sel + (size_t)rc * k;
  if (P.dense) {
#pragma unroll 1
    for (int j = lane; j < k; j += 32) out[j] = (uint16_t)j;
    return;
  }
  const uint32_t lt = (1u << lane) - 1u;
#pragma unroll 1
  for (int c = 0; c < nw; ++c) {
    const uint32_t w = M.selw[c];
    const uint32_t pos = M.pref[c] + __popc(w & lt);
    if (((w >> lane) & 1u) && pos < (uint32_t)k) out[pos] = (uint16_t)(32 * c + lane);
  }
}

// acc + (8 bf16 of a) . z[0..8)
__device__ __forceinline__ float dot8f(uint4 a, const float* z, float acc) {
  acc = fmaf(bf16_lo(a.x), z[0], acc);
  acc = fmaf(bf16_hi(a.x), z[1], acc);
  acc = fmaf(bf16_lo(a.y), z[2], acc);
  acc = fmaf(bf16_hi(a.y), z[3], acc);
  acc = fmaf(bf16_lo(a.z), z[4], acc);
  acc = fmaf(bf16_hi(a.z), z[5], acc);
  acc = fmaf(bf16_lo(a.w), z[6], acc);
  acc = fmaf(bf16_hi(a.w), z[7], acc);
  return acc;
}

// A_e z on this CTA's output slice: lr[i] = sum_rho A[i][rho] * z[rho] (A: the slice's
// rows, global, [slice][r] bf16).  Rows of r % 8 == 0 go by 16-byte loads.
__device__ __noinline__ void lowrank_slice(const uint16_t* A, int slice, int r, const float* z, float* lr) {
#pragma unroll 1
  for (int i = threadIdx.x; i < slice; i += kFT) {
    const uint16_t* arow = A + (size_t)i * r;
    float acc = 0.f;
    if ((r & 7) == 0) {
      // up to 8 16-byte loads of the row in flight at once, then their products
#pragma unroll 1
      for (int c0 = 0; c0 < r; c0 += 64) {
        uint4 a[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          a[u] = c0 + 8 * u < r ? __ldg(reinterpret_cast<const uint4*>(arow + c0 + 8 * u)) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (c0 + 8 * u < r) acc = dot8f(a[u], z + c0 + 8 * u, acc);
      }
    } else {
#pragma unroll 1
      for (int rho = 0; rho < r; ++rho) acc = fmaf(__uint_as_float((uint32_t)__ldg(arow + rho) << 16), z[rho], acc);
    }
    lr[i] = acc;
  }
}

// y[0..8) += h * (8 bf16 of v)
__device__ __forceinline__ void axpy8(float (&y)[8], float h, uint4 v) {
  y[0] = fmaf(h, bf16_lo(v.x), y[0]);
  y[1] = fmaf(h, bf16_hi(v.x), y[1]);
  y[2] = fmaf(h, bf16_lo(v.y), y[2]);
  y[3] = fmaf(h, bf16_hi(v.y), y[3]);
  y[4] = fmaf(h, bf16_lo(v.z), y[4]);
  y[5] = fmaf(h, bf16_hi(v.z), y[5]);
  y[6] = fmaf(h, bf16_lo(v.w), y[6]);
  y[7] = fmaf(h, bf16_hi(v.w), y[7]);
}


// score = alpha * |sum of the 8 warps' partials| / 2 for this CTA's nrows rows, pushed
// to every CTA of the cluster (keys at rows lt0*16 ...; four threads per row, each
// pushing to a quarter of the cluster), with one max per warp into each CTA's cmax.
__device__ __forceinline__ void push_scores(const FusedParams& P, Misc& M, const float* part,
                                         const float* alpha_s, uint32_t* keys, int nrows, int lt0,
                                         int rc, int q) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, CS = P.cs;
  const int per = CS / 4;  // destinations per thread: four threads share a row
  const uint32_t rbar_s = smem_addr(&M.bar[kBarScores]);
#pragma unroll 1
  for (int i0 = 0; i0 < 4 * nrows; i0 += kFT) {
    const int item = i0 + tid, row = item >> 2, d0 = (item & 3) * per;
    uint32_t key = 0;
    if (row < nrows) {
      float sc = 0.f;
#pragma unroll
      for (int w = 1; w < kFW; ++w) sc += part[w * P.tpc * kRowTile + row];
      sc = alpha_s[row] * fabsf(sc + part[row]) * 0.5f;
      key = __float_as_uint(sc);
      if (P.tr.scores && d0 == 0) P.tr.scores[(size_t)rc * P.D.ipad + lt0 * kRowTile + row] = sc;
      const uint32_t la = smem_addr(keys + lt0 * kRowTile + row);
#pragma unroll 1
      for (int dst = d0; dst < d0 + per; ++dst) st_async(mapa(la, dst), key, mapa(rbar_s, dst));
    }
    const uint32_t m = __reduce_max_sync(0xffffffffu, key);
    if (i0 + warp * 32 < 4 * nrows && lane < CS)
      red_async_max(mapa(smem_addr(&M.cmax), lane), m, mapa(rbar_s, lane));
  }
}

// After a wait of this CTA ran out: wait (bounded) for every barrier whose bytes may
// still be landing -- the copies into this CTA and the other CTAs' pushes -- so that
// nothing lands in its shared memory after it has exited.
__device__ __noinline__ void quiesce(Misc& M, int dense, uint32_t* err, uint64_t limit) {
  if (threadIdx.x != 0) return;
#pragma unroll 1
  for (int b = kBarRows; b < kBarRing; ++b)  // (the sketch barrier is armed off the dense path)
    if (b != kBarSketch || !dense) mbar_wait(&M.bar[b], 0, err, limit);
}

// Issue the bulk copy of channel `ch`'s record into ring slot `slot`.
__device__ __forceinline__ void issue_record(const FusedParams& P, Misc& M, uint16_t* ring, int e,
                                             int ch, int slot) {
  const size_t idx = (size_t)e * P.D.inter + ch;
  const uint32_t rb = P.rec_bytes;
  const void* src = P.q4 ? static_cast<const void*>(reinterpret_cast<const uint8_t*>(P.records) + idx * rb)
                         : static_cast<const void*>(P.records + idx * 3 * P.D.d);
  mbar_arrive_expect_tx(&M.bar[kBarRing + slot], rb);
  bulk_g2s(ring + (size_t)slot * P.rs, src, rb, &M.bar[kBarRing + slot]);
}


// On a failed wait: wait (bounded) for this CTA's record copies still in flight,
// so that none lands after the CTA has exited.
__device__ __noinline__ void drain_ring(Misc& M, int issued, int landed, int ring, uint32_t* err,
                                        uint64_t limit) {
  if (threadIdx.x != 0) return;
#pragma unroll 1
  for (int i = landed; i < issued; ++i)
    mbar_wait(&M.bar[kBarRing + i % ring], (uint32_t)(i / ring) & 1u, err, limit);
}

// ---------------------------------------------------------------- the kernel's phases
// Each phase is its own function so that the code a launch runs stays small and in one
// piece (the per-launch instruction fetch is the cost that matters at this size); the
// shared-memory views are recomputed from the parameters in each.

__device__ __forceinline__ Misc& misc(const FusedParams& P) { return *reinterpret_cast<Misc*>(g_sm + P.o_misc); }
__device__ __forceinline__ uint8_t* big_of(const FusedParams& P) { return g_sm + P.o_big; }
template <typename T>
__device__ __forceinline__ T* in_big(const FusedParams& P, int off) { return reinterpret_cast<T*>(g_sm + P.o_big + off); }

// Barrier set-up, the router rows' copy, zero-fills; before the grid dependency wait.
__device__ __forceinline__ void phase_prologue(const FusedParams& P, int q) {
  Misc& M = misc(P);
  const int tid = threadIdx.x, d = P.D.d, E = P.D.experts;
  if (tid == 0) {
#pragma unroll 1
    for (int i = 0; i < kBarRing + P.ring; ++i) mbar_init(&M.bar[i], 1);

    M.cmax = 0u;
    M.ccount = 0u;
    fence_mbar_init();
    const int e_lo = min(E, q * P.rpc), e_hi = min(E, e_lo + P.rpc);
    mbar_arrive_expect_tx(&M.bar[kBarRows], (uint32_t)(e_hi - e_lo) * 2u * d);
    uint16_t* rows = reinterpret_cast<uint16_t*>(big_of(P));
#pragma unroll 1
    for (int j = 0; j < e_hi - e_lo; ++j)
      bulk_g2s(rows + (size_t)j * P.rrs, P.router_t + (size_t)(e_lo + j) * d, 2u * d, &M.bar[kBarRows]);
    // bytes the other CTAs will push into this one
    mbar_arrive_expect_tx(&M.bar[kBarLogits], P.x1_bytes);
    mbar_arrive_expect_tx(&M.bar[kBarIds], 8u * (uint32_t)P.D.top_e);
    mbar_arrive_expect_tx(&M.bar[kBarScores], P.sc_bytes);
    mbar_arrive_expect_tx(&M.bar[kBarZ], P.z_bytes);
    mbar_arrive_expect_tx(&M.bar[kBarY], P.y_bytes);
  }
  if (tid < kWordsMax) M.csel[tid] = 0u;

  float* logits = in_big<float>(P, P.o_logits);
  if (E + tid < P.epad) logits[E + tid] = -INFINITY;
  if (!P.dense) {
    uint4* hist = in_big<uint4>(P, P.o_hist);
#pragma unroll 1
    for (int i = tid; i < kSelBins / 4; i += kFT) hist[i] = make_uint4(0u, 0u, 0u, 0u);
  }
}

// The warp sums of 8 values at once by a transposed butterfly (9 shuffles instead of 40):
// afterwards lane l holds the sum over the warp of v[(l >> 2) & 7].
__device__ __forceinline__ float warp_sum8(const float (&v)[8]) {
  const int lane = threadIdx.x & 31;
  const bool u16 = lane & 16, u8 = lane & 8, u4 = lane & 4;
  float a[4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
    a[j] = (u16 ? v[j + 4] : v[j]) + __shfl_xor_sync(0xffffffffu, u16 ? v[j] : v[j + 4], 16);
  float b[2];
#pragma unroll
  for (int j = 0; j < 2; ++j)
    b[j] = (u8 ? a[j + 2] : a[j]) + __shfl_xor_sync(0xffffffffu, u8 ? a[j] : a[j + 2], 8);
  float c = (u4 ? b[1] : b[0]) + __shfl_xor_sync(0xffffffffu, u4 ? b[0] : b[1], 4);
  c += __shfl_xor_sync(0xffffffffu, c, 2);
  c += __shfl_xor_sync(0xffffffffu, c, 1);
  return c;
}

// acc + (8 bf16 of a) . xf[0..8)
__device__ __forceinline__ float dot8xf(uint4 a, const float (&xf)[8], float acc) {
  acc = fmaf(bf16_lo(a.x), xf[0], acc);
  acc = fmaf(bf16_hi(a.x), xf[1], acc);
  acc = fmaf(bf16_lo(a.y), xf[2], acc);
  acc = fmaf(bf16_hi(a.y), xf[3], acc);
  acc = fmaf(bf16_lo(a.z), xf[4], acc);
  acc = fmaf(bf16_hi(a.z), xf[5], acc);
  acc = fmaf(bf16_lo(a.w), xf[6], acc);
  acc = fmaf(bf16_hi(a.w), xf[7], acc);
  return acc;
}

// A: logits of this CTA's router rows, 8 rows at a time (each thread its 8-element
// groups of every row, one transposed warp reduction, the warps' sums in shared memory),
// pushed to every CTA of the cluster.  Returns ok.
template <int IT>
__device__ __forceinline__ bool phase_router(const FusedParams& P, int q, bool ok, const float (&xf)[IT][8]) {
  Misc& M = misc(P);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, d = P.D.d, E = P.D.experts;
  const int e_lo = min(E, q * P.rpc), e_hi = min(E, e_lo + P.rpc);
  const uint32_t rbar = smem_addr(&M.bar[kBarLogits]);
  const uint32_t la = smem_addr(in_big<float>(P, P.o_logits) + e_lo);
  const uint16_t* rows = reinterpret_cast<const uint16_t*>(big_of(P));
#pragma unroll 1
  for (int r0 = 0; r0 < e_hi - e_lo; r0 += 8) {
    const int nb = min(8, e_hi - e_lo - r0);
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = 0.f;
    // rows past nb repeat row nb - 1 (their sums are dropped), so that all eight loads
    // issue together
#pragma unroll
    for (int it = 0; it < IT; ++it) {
      const int el = (it * kFT + tid) * 8;
      if (el < d) {
        uint4 a[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          a[j] = *reinterpret_cast<const uint4*>(rows + (size_t)(r0 + min(j, nb - 1)) * P.rrs + el);
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = dot8xf(a[j], xf[it], v[j]);
      }
    }
    const float sw = warp_sum8(v);
    if ((lane & 3) == 0) M.red8[warp][lane >> 2] = sw;
    __syncthreads();
    if (tid < nb * P.cs) {  // one thread per (row, destination)
      const int row = tid / P.cs, dst = tid - row * P.cs;
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < kFW; ++w) acc += M.red8[w][row];
      st_async(mapa(la + 4u * (r0 + row), dst), __float_as_uint(acc), mapa(rbar, dst));
    }
    __syncthreads();
  }
  return wait_phase(&M.bar[kBarLogits], 0, P.err) && ok;
}

// The copies of routed expert e: sketch tiles and alpha of this CTA's rows, B_e rows of
// its z entries; the A_e rows of its output slice into L2 (thread 0).
__device__ __forceinline__ void issue_expert(const FusedParams& P, int e, int q, int nt, int lt0, int nz) {
  Misc& M = misc(P);
  const int d = P.D.d, r = P.D.rank, KC = d / kColChunk, CS = P.cs;
  const int ntile_all = P.D.ipad / kRowTile;
  fence_proxy_async();  // the router rows were read through the generic proxy
  // the B_e rows first: z is formed while the (larger) sketch tiles are in flight
  mbar_arrive_expect_tx(&M.bar[kBarLow], (uint32_t)nz * 2u * d);
  uint16_t* brows = in_big<uint16_t>(P, P.o_brows);
#pragma unroll 1
  for (int i = 0; i < nz; ++i)
    bulk_g2s(brows + (size_t)i * d, P.lr_b + ((size_t)e * r + q + i * CS) * d, 2u * d, &M.bar[kBarLow]);
  if (!P.dense) {
    const uint32_t code_bytes = (uint32_t)nt * KC * kChunkWords * 4u;
    mbar_arrive_expect_tx(&M.bar[kBarSketch], code_bytes + (uint32_t)nt * kRowTile * 4u);
    if (nt) {
      bulk_g2s(big_of(P), P.sketch + ((size_t)e * ntile_all + lt0) * KC * kChunkWords, code_bytes,
               &M.bar[kBarSketch]);
      bulk_g2s(in_big<float>(P, P.o_alpha), P.alpha + (size_t)e * P.D.ipad + (size_t)lt0 * kRowTile,
               nt * kRowTile * 4u, &M.bar[kBarSketch]);
    }
  }
  if (r > 0) prefetch_l2(P.lr_a + ((size_t)e * d + (size_t)q * P.slice) * r, 2u * P.slice * r);
}

// z entries of this CTA: z[q + i CS] = B_e[q + i CS] . x for i < nz, 8 rows at a time with
// every thread on its 8-element groups (rows past the chunk repeat its last row, their
// sums dropped), one transposed warp reduction, the warps' sums in shared memory; each
// entry pushed to every CTA of the cluster.  Rows staged in shared memory at stride d.
template <int IT>
__device__ __forceinline__ void push_z(const FusedParams& P, int q, int nz, const float (&xf)[IT][8]) {
  Misc& M = misc(P);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, d = P.D.d, CS = P.cs;
  const uint16_t* brows = in_big<const uint16_t>(P, P.o_brows);
  const uint32_t rbar = smem_addr(&M.bar[kBarZ]);
#pragma unroll 1
  for (int r0 = 0; r0 < nz; r0 += 8) {
    const int nb = min(8, nz - r0);
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = 0.f;
#pragma unroll
    for (int it = 0; it < IT; ++it) {
      const int el = (it * kFT + tid) * 8;
      if (el < d) {
        uint4 a[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) a[j] = *reinterpret_cast<const uint4*>(brows + (size_t)(r0 + min(j, nb - 1)) * d + el);
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = dot8xf(a[j], xf[it], v[j]);
      }
    }
    const float sw = warp_sum8(v);
    if ((lane & 3) == 0) M.red8[warp][lane >> 2] = sw;
    __syncthreads();
    if (tid < nb * CS) {  // one thread per (row, destination)
      const int row = tid / CS, dst = tid - row * CS;
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < kFW; ++w) acc += M.red8[w][row];
      st_async(mapa(smem_addr(&M.z[q + (r0 + row) * CS]), dst), __float_as_uint(acc), mapa(rbar, dst));
    }
    __syncthreads();
  }
}

// B: the x permutation for scoring and z = B_e x (pushed) while the sketch tiles fly;
// then the sketch scores of this CTA's rows on the tensor cores, pushed with the warps'
// largest keys.  Returns ok.
template <int IT>
__device__ __forceinline__ bool phase_scores(const FusedParams& P, int q, int pr, int nt, int lt0, int nz,
                                          bool ok, const float (&xf)[IT][8]) {
  Misc& M = misc(P);
  const int warp = threadIdx.x >> 5, KC = P.D.d / kColChunk;
  float* part = in_big<float>(P, P.o_part);
  if (!P.dense) {
    // xperm[kc][c][s][p] = the bf16 pair of x at column 64*kc + 16*s + 2*c + 8*p (built
    // while the sketch tiles are in flight)
    uint32_t* xperm = in_big<uint32_t>(P, P.o_xperm);
    const uint32_t* x32 = in_big<const uint32_t>(P, P.o_x);
#pragma unroll 1
    for (int i = threadIdx.x; i < P.D.d / 2; i += kFT) {
      const int kc = i >> 5, c = (i >> 3) & 3, q8 = i & 7;
      xperm[i] = x32[kc * 32 + 8 * (q8 >> 1) + c + 4 * (q8 & 1)];
    }
  }
  // z = B_e x, pushed, while the sketch tiles are still in flight
  if (nz > 0) {
    ok = wait_phase(&M.bar[kBarLow], 0, P.err) && ok;
    push_z<IT>(P, q, nz, xf);
  }
  if (!P.dense) {
    ok = wait_phase(&M.bar[kBarSketch], 0, P.err) && ok;
    __syncthreads();  // xperm complete
    MARK(4);
    if (nt > 0)
      score_tiles(reinterpret_cast<const uint2*>(big_of(P)), in_big<const uint4>(P, P.o_xperm), nt, KC,
                  part + warp * P.tpc * kRowTile);
    __syncthreads();
    MARK(5);
    push_scores(P, M, part, in_big<float>(P, P.o_alpha), in_big<uint32_t>(P, P.o_keys), nt * kRowTile, lt0,
                pr, q);
  }
  return ok;
}

// C: exact top-k over the cluster's scores (or, dense, every channel) and this CTA's
// share of it into M.mysel; then the first record copies.  Returns ok.
__device__ __forceinline__ bool phase_select(const FusedParams& P, int e, int q, int pr, int tok, int nmine,
                                          int lgcs, bool ok) {
  Misc& M = misc(P);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, I = P.D.inter;
  const int nw = (I + 31) / 32;
  if (!P.dense) {
    ok = wait_phase(&M.bar[kBarScores], 0, P.err) && ok;
    MARK(7);
    select_topk(in_big<uint32_t>(P, P.o_keys), I, P.k, M.cmax, in_big<uint32_t>(P, P.o_hist), M);
    MARK(8);
    if (warp == 0) positions_prefix(nw, P.k, nmine, M, MYSEL(P), P.err);
    __syncthreads();
    positions_place(I, q, lgcs, nmine, M, MYSEL(P));
    __syncthreads();
  } else {
    if (warp == 0)
#pragma unroll 1
      for (int t = lane; t < nmine; t += 32) MYSEL(P)[t] = (uint16_t)(q + (t << lgcs));
    __syncthreads();  // (the dense path had no barrier since phase A: big is free now)
  }
  MARK(9);
  if (q == 0 && (P.tr.sel || P.tr.sel_count) && warp == 0) trace_selection(P, M, nw, pr);
  if (q == 0 && pr == tok * P.D.top_e && (P.tr.expert_ids || P.tr.expert_w || P.tr.union_count))
    trace_routing(P.tr, M, P.D.experts, P.D.top_e, P.k, tok);
  // the ring now takes over `big`: every thread is past its last use of phases A-C
  if (warp == 0 && ok) {
    fence_proxy_async();
    uint16_t* ring = reinterpret_cast<uint16_t*>(big_of(P));
    const int nfirst = min(P.ring, nmine);
#ifdef MSB_INSTRUMENTED
    if (lane < nfirst && !(P.skip == 1u && blockIdx.x == 0 && lane == 0))
#else
    if (lane < nfirst)
#endif
      issue_record(P, M, ring, e, MYSEL(P)[lane], lane);
  }
  return ok;
}

// D: the records in batches as they land (the first batch of one record, so that a
// slot frees early, then up to bmax = min(4, ring / 2)).  gate.x and up.x of a batch: each
// thread its 8-element groups of every gate and up row, one transposed warp reduction of
// the (up to) 8 values, the warps' sums in shared memory; h = silu(gate.x) * up.x; then
// every thread adds h * down over its groups.  After the first barrier of a batch the
// previous batch's slots are refilled.  Then y is pushed, slice by slice, to each slice's
// owner.  Returns ok.
template <int IT>
__device__ __forceinline__ bool phase_records(const FusedParams& P, int e, int q, int nmine, bool ok,
                                              const float (&xf)[IT][8]) {
  Misc& M = misc(P);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, d = P.D.d;
  const uint16_t* ring = reinterpret_cast<const uint16_t*>(big_of(P));
  const int bmax = max(1, min(4, P.ring / 2));
  float y[IT][8];
#pragma unroll
  for (int it = 0; it < IT; ++it)
#pragma unroll
    for (int i = 0; i < 8; ++i) y[it][i] = 0.f;
  int s0 = 0, pb0 = 0, pnb = 0;  // first slot of this batch; first slot and size of the previous
  uint32_t par0 = 0;             // phase parity of slot s0
  int issued = ok ? min(P.ring, nmine) : 0, landed = 0;
#pragma unroll 1
  for (int i = 0; i < nmine;) {
    const int nb = i == 0 ? 1 : min(bmax, nmine - i);
    if (ok) {
#pragma unroll 1
      for (int j = 0; j < nb && ok; ++j) {
        const int sl = s0 + j < P.ring ? s0 + j : s0 + j - P.ring;
        ok = wait_phase(&M.bar[kBarRing + sl], s0 + j < P.ring ? par0 : par0 ^ 1u, P.err);
      }
      if (ok) landed = i + nb;
    }
    {
      // value 2j: gate_j . x, value 2j + 1: up_j . x (record j of the batch; records past
      // nb repeat record nb - 1, their sums dropped, so that all eight loads issue together)
      float v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = 0.f;
      const uint16_t* rec[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int jj = s0 + min(j, nb - 1);
        rec[j] = ring + (size_t)(jj < P.ring ? jj : jj - P.ring) * P.rs;
      }
#pragma unroll
      for (int it = 0; it < IT; ++it) {
        const int el = (it * kFT + tid) * 8;
        if (el < d) {
          uint4 a[8];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            a[2 * j] = *reinterpret_cast<const uint4*>(rec[j] + el);
            a[2 * j + 1] = *reinterpret_cast<const uint4*>(rec[j] + d + el);
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) v[j] = dot8xf(a[j], xf[it], v[j]);
        }
      }
      const float sw = warp_sum8(v);
      if ((lane & 3) == 0) M.red8[warp][lane >> 2] = sw;
    }
    ok = __syncthreads_and(ok);
    // every thread has finished the previous batch: refill its slots (warp 1, while warp 0
    // forms h)
    if (tid == 32 && ok && pnb > 0 && issued < nmine) {
      uint16_t* wring = reinterpret_cast<uint16_t*>(big_of(P));
      fence_proxy_async();
#pragma unroll 1
      for (int j = 0; j < pnb && issued < nmine; ++j, ++issued)
        issue_record(P, M, wring, e, MYSEL(P)[issued], pb0 + j < P.ring ? pb0 + j : pb0 + j - P.ring);
    }
    if (i == 0) MARK(11);
    if (tid < nb) {
      float g = 0.f, u = 0.f;
#pragma unroll
      for (int w = 0; w < kFW; ++w) {
        g += M.red8[w][2 * tid];
        u += M.red8[w][2 * tid + 1];
      }
      M.h[tid] = __fdividef(g, 1.0f + __expf(-g)) * u;
    }
    __syncthreads();
    // y += h_j * down_j over this thread's groups, two records at a time (a missing
    // second record repeats the first with h = 0)
#pragma unroll 1
    for (int j = 0; j < nb; j += 2) {
      const int ja = s0 + j, jb = s0 + min(j + 1, nb - 1);
      const uint16_t* reca = ring + (size_t)(ja < P.ring ? ja : ja - P.ring) * P.rs + 2 * d;
      const uint16_t* recb = ring + (size_t)(jb < P.ring ? jb : jb - P.ring) * P.rs + 2 * d;
      const float ha = M.h[j], hb = j + 1 < nb ? M.h[j + 1] : 0.f;
#pragma unroll
      for (int it = 0; it < IT; ++it) {
        const int el = (it * kFT + tid) * 8;
        if (el < d) {
          const uint4 va = *reinterpret_cast<const uint4*>(reca + el);
          const uint4 vb = *reinterpret_cast<const uint4*>(recb + el);
          axpy8(y[it], ha, va);
          axpy8(y[it], hb, vb);
        }
      }
    }
    pb0 = s0;
    pnb = nb;
    s0 += nb;
    if (s0 >= P.ring) { s0 -= P.ring; par0 ^= 1u; }
    i += nb;
  }
  if (!ok) drain_ring(M, issued, landed, P.ring, P.err, WAIT_LIMIT);
  // every thread waits for the drain: no thread pushes or arrives at the cluster barrier
  // ahead of it (the arrive is warp-aligned, and every push of this CTA must be issued
  // before any CTA of the cluster can pass the barrier)
  __syncthreads();
  MARK(12);
  // push each 8-element group to the owner of its slice: rbuf[q][offset in slice]
  const uint32_t rbuf = smem_addr(g_sm + P.o_rbuf), rbar_y = smem_addr(&M.bar[kBarY]);
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int el = (it * kFT + tid) * 8;
    if (el < d) {
      const int owner = el / P.slice, off = el - owner * P.slice;
      const uint32_t ra = mapa(rbuf + 4u * (q * P.slice + off), owner), rb = mapa(rbar_y, owner);
      st_async4(ra, y[it][0], y[it][1], y[it][2], y[it][3], rb);
      st_async4(ra + 16u, y[it][4], y[it][5], y[it][6], y[it][7], rb);
    }
  }
  return ok;
}

// ---------------------------------------------------------------- 4-bit channel records
// Record of one channel (group-wise affine, 64 weights per group): the nibble codes of the
// gate row, the up row and the down column (byte i: element 2i in bits 0-3, 2i + 1 in bits
// 4-7), then each vector's (scale, bias) BF16 pairs; the weight is s * q + b.

// code k of a byte lane as an exact float: the byte placed in the mantissa of 2^23
__device__ __forceinline__ float nib(uint32_t bytes, uint32_t sel) {
  return __uint_as_float(__byte_perm(bytes, 0x4B000000u, sel)) - 8388608.0f;
}

// acc + sum of the 8 codes of c (elements 0..7 in order) times xf[0..8)
__device__ __forceinline__ float dot8q(uint32_t c, const float (&xf)[8], float acc) {
  const uint32_t lo = c & 0x0F0F0F0Fu, hi = (c >> 4) & 0x0F0F0F0Fu;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc = fmaf(nib(lo, 0x7650u | i), xf[2 * i], acc);
    acc = fmaf(nib(hi, 0x7650u | i), xf[2 * i + 1], acc);
  }
  return acc;
}

// y[0..8) += hs * (the 8 codes of c)
__device__ __forceinline__ void axpy8q(float (&y)[8], float hs, uint32_t c) {
  const uint32_t lo = c & 0x0F0F0F0Fu, hi = (c >> 4) & 0x0F0F0F0Fu;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    y[2 * i] = fmaf(hs, nib(lo, 0x7650u | i), y[2 * i]);
    y[2 * i + 1] = fmaf(hs, nib(hi, 0x7650u | i), y[2 * i + 1]);
  }
}

// D on 4-bit records: the batches, waits, refills and pushes of phase_records; each
// thread's 8 elements lie in one group, so gate.x over them is s * (q . x) + b * sum(x)
// and the down update is (h s) q plus h b, the latter summed once per record.
template <int IT>
__device__ __forceinline__ bool phase_records_q4(const FusedParams& P, int e, int q, int nmine, bool ok,
                                                 const float (&xf)[IT][8]) {
  Misc& M = misc(P);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, d = P.D.d;
  const uint8_t* ring8 = big_of(P);
  const size_t slotb = 2u * (size_t)P.rs;                  // slot stride = record bytes
  const int G = d / 64;
  const uint32_t pb = 3u * (uint32_t)d / 2u;               // offset of the (scale, bias) pairs
  const int bmax = max(1, min(4, P.ring / 2));
  float xsum[IT];
#pragma unroll
  for (int it = 0; it < IT; ++it)
    xsum[it] = ((xf[it][0] + xf[it][1]) + (xf[it][2] + xf[it][3])) + ((xf[it][4] + xf[it][5]) + (xf[it][6] + xf[it][7]));
  float y[IT][8], yb[IT];
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    yb[it] = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) y[it][i] = 0.f;
  }
  int s0 = 0, pb0 = 0, pnb = 0;
  uint32_t par0 = 0;
  int issued = ok ? min(P.ring, nmine) : 0, landed = 0;
#pragma unroll 1
  for (int i = 0; i < nmine;) {
    const int nb = i == 0 ? 1 : min(bmax, nmine - i);
    if (ok) {
#pragma unroll 1
      for (int j = 0; j < nb && ok; ++j) {
        const int sl = s0 + j < P.ring ? s0 + j : s0 + j - P.ring;
        ok = wait_phase(&M.bar[kBarRing + sl], s0 + j < P.ring ? par0 : par0 ^ 1u, P.err);
      }
      if (ok) landed = i + nb;
    }
    {
      float v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = 0.f;
      const uint8_t* rec[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int jj = s0 + min(j, nb - 1);
        rec[j] = ring8 + (size_t)(jj < P.ring ? jj : jj - P.ring) * slotb;
      }
#pragma unroll
      for (int it = 0; it < IT; ++it) {
        const int el = (it * kFT + tid) * 8;
        if (el < d) {
          const int g = el / 64;
          uint32_t c[8], sb[8];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            c[2 * j] = *reinterpret_cast<const uint32_t*>(rec[j] + el / 2);
            c[2 * j + 1] = *reinterpret_cast<const uint32_t*>(rec[j] + d / 2 + el / 2);
            sb[2 * j] = *reinterpret_cast<const uint32_t*>(rec[j] + pb + 4 * g);
            sb[2 * j + 1] = *reinterpret_cast<const uint32_t*>(rec[j] + pb + 4 * (G + g));
          }
#pragma unroll
          for (int j = 0; j < 8; ++j)
            v[j] = fmaf(bf16_lo(sb[j]), dot8q(c[j], xf[it], 0.f), fmaf(bf16_hi(sb[j]), xsum[it], v[j]));
        }
      }
      const float sw = warp_sum8(v);
      if ((lane & 3) == 0) M.red8[warp][lane >> 2] = sw;
    }
    ok = __syncthreads_and(ok);
    if (tid == 32 && ok && pnb > 0 && issued < nmine) {
      uint16_t* wring = reinterpret_cast<uint16_t*>(big_of(P));
      fence_proxy_async();
#pragma unroll 1
      for (int j = 0; j < pnb && issued < nmine; ++j, ++issued)
        issue_record(P, M, wring, e, MYSEL(P)[issued], pb0 + j < P.ring ? pb0 + j : pb0 + j - P.ring);
    }
    if (i == 0) MARK(11);
    if (tid < nb) {
      float gs = 0.f, us = 0.f;
#pragma unroll
      for (int w = 0; w < kFW; ++w) {
        gs += M.red8[w][2 * tid];
        us += M.red8[w][2 * tid + 1];
      }
      M.h[tid] = __fdividef(gs, 1.0f + __expf(-gs)) * us;
    }
    __syncthreads();
    // y += h_j * down_j: (h s) q per element, h b once per record
#pragma unroll 1
    for (int j = 0; j < nb; j += 2) {
      const int ja = s0 + j, jb = s0 + min(j + 1, nb - 1);
      const uint8_t* reca = ring8 + (size_t)(ja < P.ring ? ja : ja - P.ring) * slotb;
      const uint8_t* recb = ring8 + (size_t)(jb < P.ring ? jb : jb - P.ring) * slotb;
      const float ha = M.h[j], hb = j + 1 < nb ? M.h[j + 1] : 0.f;
#pragma unroll
      for (int it = 0; it < IT; ++it) {
        const int el = (it * kFT + tid) * 8;
        if (el < d) {
          const int g = el / 64;
          const uint32_t ca = *reinterpret_cast<const uint32_t*>(reca + d + el / 2);
          const uint32_t cb = *reinterpret_cast<const uint32_t*>(recb + d + el / 2);
          const uint32_t sa = *reinterpret_cast<const uint32_t*>(reca + pb + 4 * (2 * G + g));
          const uint32_t sbb = *reinterpret_cast<const uint32_t*>(recb + pb + 4 * (2 * G + g));
          axpy8q(y[it], ha * bf16_lo(sa), ca);
          axpy8q(y[it], hb * bf16_lo(sbb), cb);
          yb[it] = fmaf(ha, bf16_hi(sa), fmaf(hb, bf16_hi(sbb), yb[it]));
        }
      }
    }
    pb0 = s0;
    pnb = nb;
    s0 += nb;
    if (s0 >= P.ring) { s0 -= P.ring; par0 ^= 1u; }
    i += nb;
  }
#pragma unroll
  for (int it = 0; it < IT; ++it)
#pragma unroll
    for (int i = 0; i < 8; ++i) y[it][i] += yb[it];
  if (!ok) drain_ring(M, issued, landed, P.ring, P.err, WAIT_LIMIT);
  __syncthreads();
  MARK(12);
  const uint32_t rbuf = smem_addr(g_sm + P.o_rbuf), rbar_y = smem_addr(&M.bar[kBarY]);
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int el = (it * kFT + tid) * 8;
    if (el < d) {
      const int owner = el / P.slice, off = el - owner * P.slice;
      const uint32_t ra = mapa(rbuf + 4u * (q * P.slice + off), owner), rb = mapa(rbar_y, owner);
      st_async4(ra, y[it][0], y[it][1], y[it][2], y[it][3], rb);
      st_async4(ra + 16u, y[it][4], y[it][5], y[it][6], y[it][7], rb);
    }
  }
  return ok;
}

// E: the owner of slice q sums the cluster's partials of it, adds A_e z, weights by
// the router and reduction-adds into the FP32 accumulator; the last of the K
// contributions converts the slice to BF16 and re-zeroes it.  Returns ok.
__device__ __forceinline__ bool phase_combine(const FusedParams& P, int q, int rc, int tok, bool ok) {
  Misc& M = misc(P);
  const int tid = threadIdx.x, K = P.D.top_e;
  const float* lr = reinterpret_cast<const float*>(g_sm + P.o_lr);
  const float* rbuf = reinterpret_cast<const float*>(g_sm + P.o_rbuf);
  float* yacc = P.y_acc + (size_t)tok * P.D.d;     // token tok's accumulator row
  uint32_t* cnt = P.slice_cnt + tok * P.cs;         // and its slices' arrival counters
  ok = wait_phase(&M.bar[kBarY], 0, P.err) && ok;
  MARK(13);
  const float we = M.wk[rc];
  if (ok) {
#pragma unroll 1
    for (int j = tid; j < P.slice / 4; j += kFT) {
      float4 acc = P.D.rank > 0 ? *reinterpret_cast<const float4*>(lr + 4 * j) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
      for (int src = 0; src < P.cs; ++src) {
        const float4 v = *reinterpret_cast<const float4*>(rbuf + src * P.slice + 4 * j);
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
      }
      red_add_v4(yacc + q * P.slice + 4 * j, we * acc.x, we * acc.y, we * acc.z, we * acc.w);
    }
  }
  // the CTA's reduction-adds precede (barrier, then the release of the counter's atomic)
  // its count; the last contributor's acquire makes every other contribution visible
  __syncthreads();
  if (tid == 0) M.last = (atom_add_acq_rel_gpu(cnt + q, 1u) == (uint32_t)(K - 1));
  __syncthreads();
  if (M.last) {
    // every contribution to this slice has arrived: convert, re-zero, reset
#pragma unroll 1
    for (int j = tid; j < P.slice / 4; j += kFT) {
      float4* p = reinterpret_cast<float4*>(yacc + q * P.slice) + j;
      const float4 v = __ldcg(p);
      __stcg(p, make_float4(0.f, 0.f, 0.f, 0.f));
      const uint32_t lo = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v.x)) |
                          ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v.y)) << 16);
      const uint32_t hi = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v.z)) |
                          ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v.w)) << 16);
      reinterpret_cast<uint2*>(P.out + (size_t)tok * P.D.d + q * P.slice)[j] = make_uint2(lo, hi);
    }
    if (tid == 0) cnt[q] = 0u;
  }
  return ok;
}

template <int IT, bool Q4>  // IT = ceil(d / 2048): 8-element groups per thread; Q4: 4-bit records
__global__ void __launch_bounds__(kFT, 2) fused_block_kernel(const __grid_constant__ FusedParams P) {
  const int CS = P.cs;
  const int q = (int)cluster_rank();
  // token tok, routed expert of rank rc: one cluster per (token, expert) pair; pr is the
  // pair's row in the trace
  const int tok = blockIdx.x / (CS * P.D.top_e);
  const int rc = blockIdx.x / CS - tok * P.D.top_e;
  const int pr = blockIdx.x / CS;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int d = P.D.d, r = P.D.rank;
  Misc& M = misc(P);

  phase_prologue(P, q);
  MARK(0);
  __syncthreads();
  // barrier inits, cmax = 0 and the zero-fills above precede any remote access
  cluster_arrive();
  // x: one bulk copy, or (in mapped host memory) CTA q reads the q-th of CS equal pieces
  // across the host link, one coalesced 16-byte load per thread, and pushes it to every
  // CTA of the cluster once every CTA has initialised its barriers.  x and the
  // accumulator may be written by the previous launch, so x is fetched after the grid
  // dependency wait -- unless the caller declared x ready (nothing earlier on the stream
  // writes it), in which case the fetch overlaps the previous launch.
  uint16_t* xs = in_big<uint16_t>(P, P.o_x);
  const int xv = d / (8 * CS);  // 16-byte vectors per piece
  uint4 xpiece = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll 1
  for (int pass = 0; pass < 2; ++pass) {
    if (pass == 1) {
      pdl_wait();
      pdl_trigger();  // the next launch may start its weight-only prologue
    }
    if (pass == (P.x_ready ? 0 : 1)) {
      if (tid == 0) {
        mbar_arrive_expect_tx(&M.bar[kBarX], 2u * d);
        if (!P.x_mapped) bulk_g2s(xs, P.x + (size_t)tok * d, 2u * d, &M.bar[kBarX]);
      }
      if (P.x_mapped && tid < xv) xpiece = ld_fresh16(P.x + (size_t)tok * d + 8 * (q * xv + tid));
      cluster_wait();  // every CTA of the cluster has initialised its barriers
      if (P.x_mapped && tid < xv) {
        const uint32_t la = smem_addr(xs + 8 * (q * xv + tid)), rb = smem_addr(&M.bar[kBarX]);
#pragma unroll 1
        for (int dst = 0; dst < CS; ++dst)
          st_async4(mapa(la, dst), __uint_as_float(xpiece.x), __uint_as_float(xpiece.y),
                    __uint_as_float(xpiece.z), __uint_as_float(xpiece.w), mapa(rb, dst));
      }
    }
  }
  bool ok = wait_phase(&M.bar[kBarX], 0, P.err);
  ok = wait_phase(&M.bar[kBarRows], 0, P.err) && ok;
  MARK(1);
  // this thread's 8-element groups of x as floats (for the router rows and the records;
  // x itself is overwritten by the ring later)
  float xf[IT][8];
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int el = (it * kFT + tid) * 8;
    const uint4 xv = el < d ? reinterpret_cast<const uint4*>(xs)[el / 8] : make_uint4(0u, 0u, 0u, 0u);
    xf[it][0] = bf16_lo(xv.x); xf[it][1] = bf16_hi(xv.x); xf[it][2] = bf16_lo(xv.y); xf[it][3] = bf16_hi(xv.y);
    xf[it][4] = bf16_lo(xv.z); xf[it][5] = bf16_hi(xv.z); xf[it][6] = bf16_lo(xv.w); xf[it][7] = bf16_hi(xv.w);
  }

  ok = phase_router<IT>(P, q, ok, xf);
  MARK(2);
  router_rank(P, in_big<float>(P, P.o_logits), q);
  ok = wait_phase(&M.bar[kBarIds], 0, P.err) && ok;
  int e = (int)M.rk[rc].x;
  if (e >= P.D.experts) {  // (only after an expired wait) keep a valid index; the call is flagged
    e = rc;
    if (tid == 0) atomicOr(P.err, kErrInternal);
  }
  MARK(3);
  const int ntile_all = P.D.ipad / kRowTile;
  const int lt0 = min(ntile_all, q * P.tpc), lt1 = min(ntile_all, lt0 + P.tpc);
  const int nt = lt1 - lt0;
  const int nz = r > q ? (r - q + CS - 1) / CS : 0;  // z rows q, q+CS, ... below r
  if (tid == 0) issue_expert(P, e, q, nt, lt0, nz);
  // combine weights (warp 0; read in phase E, many barriers later)
  if (warp == 0) router_weights(in_big<float>(P, P.o_logits), P.D.experts, P.D.top_e, P.D.renorm, M);

  ok = phase_scores<IT>(P, q, pr, nt, lt0, nz, ok, xf);
  MARK(6);
  const int lgcs = CS == 16 ? 4 : 3;  // (the cluster size is 8 or 16)
  const int nmine = P.k > q ? (P.k - q + CS - 1) >> lgcs : 0;
  ok = phase_select(P, e, q, pr, tok, nmine, lgcs, ok);
  // A_e z on this CTA's output slice while the first records fly (A_e from L2)
  if (r > 0) {
    ok = wait_phase(&M.bar[kBarZ], 0, P.err) && ok;
    lowrank_slice(P.lr_a + ((size_t)e * d + (size_t)q * P.slice) * r, P.slice, r, M.z,
                  reinterpret_cast<float*>(g_sm + P.o_lr));
  }
  MARK(10);
  if (Q4)
    ok = phase_records_q4<IT>(P, e, q, nmine, ok, xf);
  else
    ok = phase_records<IT>(P, e, q, nmine, ok, xf);
  // paired with the wait before exit: no CTA leaves before every CTA of the cluster has
  // issued its pushes (each receiver waits for its own bytes; after an expired wait the
  // quiesce below waits for them)
  cluster_arrive_relaxed();
  __syncthreads();   // lr complete (a CTA may have had no records, hence no barrier since)
  ok = phase_combine(P, q, rc, tok, ok);
  MARK(14);
  cluster_wait();
  // every push aimed at this CTA has now been issued: if any wait of this CTA ran out,
  // wait (bounded) for whatever may still be landing before the CTA exits
  if (__syncthreads_or(!ok)) quiesce(M, P.dense, P.err, WAIT_LIMIT);
#ifdef MSB_INSTRUMENTED
  if (P.marks && tid == 0) {
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    P.marks[blockIdx.x * kMarks + 15] = smid;
  }
#endif
}

// =====================================================================================
// host side
// =====================================================================================
namespace {
int g_max_clusters16[64];
int g_max_clusters8[64];
int g_pair_smem[64];  // largest dynamic shared memory that still lets two CTAs share an SM
bool g_ready[64];

int cur_dev() {
  int d = 0;
  cudaGetDevice(&d);
  return d;
}

int align_up(int v, int a) { return (v + a - 1) / a * a; }

using KernelFn = void (*)(FusedParams);

KernelFn kernel_for(int d, bool q4) {
  const int it = (d + 2047) / 2048;
  if (q4) return it <= 1 ? fused_block_kernel<1, true> : it <= 2 ? fused_block_kernel<2, true> : fused_block_kernel<4, true>;
  return it <= 1 ? fused_block_kernel<1, false> : it <= 2 ? fused_block_kernel<2, false> : fused_block_kernel<4, false>;
}

// Fill the carve-up for cluster size cs within `limit` bytes of shared memory.
bool plan(FusedParams& P, const Dims& D, int k, int cs, int limit) {
  const int d = D.d, E = D.experts, ipad = D.ipad, r = D.rank, I = D.inter;
  if (d % (8 * cs) != 0 || D.top_e < 1) return false;
  P.cs = cs;
  P.rpc = (E + cs - 1) / cs;
  P.tpc = (ipad / kRowTile + cs - 1) / cs;
  P.slice = d / cs;
  P.epad = (E + 63) / 64 * 64;
  const int per_cta = (k + cs - 1) / cs;  // channels a CTA reads
  if (per_cta > kMyselMax) return false;
  int o = 0;
  P.o_misc = o;  o = align_up(o + (int)sizeof(Misc), 128);
  P.o_lr = o;    o = align_up(o + 4 * P.slice, 128);
  P.o_rbuf = o;  o = align_up(o + 4 * d, 128);
  P.o_mysel = o; o = align_up(o + 2 * per_cta, 128);
  P.o_big = o;
  // phase A/B region at the start of big: router rows, then (reused) sketch tiles,
  // alpha and B_e rows
  P.rrs = d + 8;
  // ring slot stride in elements: BF16 records 16 bytes apart in the banks; 4-bit records
  // are read 4 bytes per thread, conflict-free at their own (16-byte multiple) size
  P.rec_bytes = P.q4 ? (uint32_t)(((size_t)3 * d / 2 + (size_t)3 * (d / 64) * 4 + 15) / 16 * 16) : 6u * d;
  P.rs = P.q4 ? (int)(P.rec_bytes / 2) : 3 * d + 8;
  const int rows_b = align_up(P.rpc * 2 * P.rrs, 128);
  int b = P.dense ? 0 : P.tpc * (d / kColChunk) * kChunkWords * 4;
  b = align_up(b, 128);
  P.o_alpha = b;  b = align_up(b + 4 * P.tpc * kRowTile, 128);
  P.o_brows = b;  b = align_up(b + ((r + cs - 1) / cs) * 2 * d, 128);
  int s = rows_b > b ? rows_b : b;
  P.o_x = s;      s = align_up(s + 2 * d, 128);
  P.o_xperm = s;  s = align_up(s + 2 * d, 128);
  P.o_logits = s; s = align_up(s + 4 * P.epad, 128);
  P.o_keys = s;   s = align_up(s + 4 * ipad, 128);
  P.o_hist = s;   s = align_up(s + (P.dense ? 0 : 4 * kSelBins), 128);
  P.o_part = s;   s = align_up(s + 4 * kFW * P.tpc * kRowTile, 128);
  const int need_abc = s;
  const int rec = 2 * P.rs;
  const int avail = limit - o;
  int ring = avail / rec;
  if (ring > kRingMax) ring = kRingMax;
  if (ring > per_cta) ring = per_cta < 1 ? 1 : per_cta;
  if (ring < 1 || need_abc > avail) return false;
  // a record's slot is refilled one record later: with refills the ring needs two slots
  if (per_cta > ring && ring < 2) return false;
  P.ring = ring;
  const int bigb = ring * rec > need_abc ? ring * rec : need_abc;
  P.smem = o + bigb;
  // bytes pushed into each CTA: every logit; every sketch row's key and one max per
  // (CTA, warp of rows); every z entry; every partial output element
  uint32_t maxmsgs = 0;
  const int ntile_all = ipad / kRowTile;
  for (int qq = 0; qq < cs; ++qq) {
    const int t0 = qq * P.tpc < ntile_all ? qq * P.tpc : ntile_all;
    const int t1 = t0 + P.tpc < ntile_all ? t0 + P.tpc : ntile_all;
    const int nrows = (t1 - t0) * kRowTile;
    maxmsgs += (uint32_t)((4 * nrows + 31) / 32);  // one max per warp of (row, quarter) items
  }
  P.x1_bytes = 4u * (uint32_t)E;
  P.sc_bytes = P.dense ? 0u : 4u * ((uint32_t)ipad + maxmsgs);
  P.z_bytes = 4u * (uint32_t)r;
  P.y_bytes = 4u * (uint32_t)d;
  (void)I;
  return P.smem <= limit;
}

// Prefer 16-CTA clusters small enough to pair on an SM (all K clusters then fit the
// GPCs), then 16-CTA clusters at any size when all K are resident, then 8-CTA
// clusters; otherwise decline (the multi-kernel path runs).  With several tokens (B K
// clusters) 8-CTA clusters that pair on an SM come first: twice the work per CTA, but
// the whole batch resident in one wave.
bool choose(FusedParams& P, const Dims& D, int k, int batch = 1) {
  const int dev = cur_dev();
  if (dev < 0 || dev >= 64 || !g_ready[dev]) return false;
  const int K = D.top_e;
  const int pair = g_pair_smem[dev];
  const bool have16 = g_max_clusters16[dev] >= 1, have8 = g_max_clusters8[dev] >= 1;
  if (batch > 1 && have8 && plan(P, D, k, 8, pair)) return true;
  if (have16 && plan(P, D, k, 16, pair)) return true;
  if (have16 && g_max_clusters16[dev] >= K && plan(P, D, k, 16, kSmemMax)) return true;
  if (have8 && plan(P, D, k, 8, pair)) return true;
  if (have8 && g_max_clusters8[dev] >= K && plan(P, D, k, 8, kSmemMax)) return true;
  if (have16 && plan(P, D, k, 16, kSmemMax)) return true;
  return false;
}

int query_clusters(KernelFn fn, int cs, int smem) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs * 16, 1, 1);
  cfg.blockDim = dim3(kFT, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  return n;
}
}  // namespace

int fused_setup() {
  const int dev = cur_dev();
  if (dev < 0 || dev >= 64) return MSB_ECUDA;
  for (KernelFn fn : {fused_block_kernel<1, false>, fused_block_kernel<2, false>, fused_block_kernel<4, false>,
                      fused_block_kernel<1, true>, fused_block_kernel<2, true>, fused_block_kernel<4, true>}) {
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax) !=
        cudaSuccess)
      return MSB_ECUDA;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
      cudaGetLastError();
    // one CTA of a cluster per SM where the GPC has room, rather than two on one SM
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeClusterSchedulingPolicyPreference,
                             cudaClusterSchedulingPolicySpread) != cudaSuccess)
      cudaGetLastError();
  }
  int per_sm = 0, reserved = 0;
  if (cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess) {
    cudaGetLastError();
    per_sm = 2 * (kSmemPair + 1024);
    reserved = 1024;
  }
  g_pair_smem[dev] = per_sm / 2 - reserved;
  if (g_pair_smem[dev] > kSmemMax) g_pair_smem[dev] = kSmemMax;
  g_max_clusters16[dev] = query_clusters(fused_block_kernel<1, false>, 16, kSmemMax);
  g_max_clusters8[dev] = query_clusters(fused_block_kernel<1, false>, 8, kSmemMax);
  g_ready[dev] = true;
  return MSB_OK;
}

void fused_plan_info(const Dims& D, int k, int batch, int* info) {
  FusedParams P{};
  P.dense = (k == D.inter);
  const int dev = cur_dev();
#pragma unroll 1
  for (int i = 0; i < 6; ++i) info[i] = 0;
  if (choose(P, D, k, batch)) {
    info[0] = P.cs;
    info[1] = 1;
    info[2] = P.ring;
    info[3] = P.smem;
  }
  if (dev >= 0 && dev < 64) {
    info[4] = g_max_clusters16[dev];
    info[5] = g_max_clusters8[dev];
  }
}

bool fused_supported(const Dims& D, int k, bool q4) {
  FusedParams P{};
  P.dense = (k == D.inter);
  P.q4 = q4 ? 1 : 0;
  return choose(P, D, k);
}


int launch_fused(const uint16_t* x, const uint16_t* router_t, const uint16_t* records,
                 const uint32_t* sketch, const float* alpha, int k, const uint16_t* lr_a,
                 const uint16_t* lr_b, uint16_t* out, const Dims& D, uint32_t* err,
                 uint32_t* counters, float* y_acc, const TraceDev& tr, cudaStream_t st, bool x_mapped,
                 bool x_ready, int batch, bool q4) {
  if (batch < 1 || batch > kFusedMaxBatch || (batch > 1 && tr.union_count)) return MSB_ENOTFUSED;
  FusedParams P{};
  P.q4 = q4 ? 1 : 0;
  P.x_mapped = x_mapped ? 1 : 0;
  P.x_ready = x_ready ? 1 : 0;
  P.x = x;
  P.router_t = router_t;
  P.records = records;
  P.sketch = sketch;
  P.alpha = alpha;
  P.lr_a = lr_a;
  P.lr_b = lr_b;
  P.out = out;
  P.err = err;
  P.slice_cnt = counters + kCntFusedSlices;
  P.y_acc = y_acc;
#ifdef MSB_INSTRUMENTED
  P.marks = debug_ctl().marks;
  P.skip = debug_ctl().skip;
  P.wait_ns = debug_ctl().wait_ns ? debug_ctl().wait_ns : kWaitLimitNs;
#endif
  P.tr = tr;
  P.D = D;
  P.k = k;
  P.dense = (k == D.inter);
  if (!choose(P, D, k, batch)) return MSB_ENOTFUSED;
  cudaLaunchConfig_t cfg = {};
  if (kCntFusedSlices + batch * P.cs > kCounters) return MSB_ENOTFUSED;
  cfg.gridDim = dim3(P.cs * D.top_e * batch, 1, 1);
  cfg.blockDim = dim3(kFT, 1, 1);
  cfg.dynamicSmemBytes = P.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[3];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = P.cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  attr[2].id = cudaLaunchAttributeClusterSchedulingPolicyPreference;
  attr[2].val.clusterSchedulingPolicyPreference = cudaClusterSchedulingPolicySpread;
  cfg.attrs = attr;
  cfg.numAttrs = 3;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel_for(D.d, P.q4 != 0), P);
  return e == cudaSuccess ? MSB_OK : MSB_ECUDA;
}

}  // namespace msb
