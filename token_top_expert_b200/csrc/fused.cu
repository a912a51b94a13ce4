// Single-launch batch-1 sparse-MoE block (the decode hot path).
//
// One thread-block cluster per routed expert (or two smaller clusters per
// expert).  Exchange inside a cluster goes through distributed shared memory and
// hardware cluster barriers; across clusters only through FP32 atomics into a
// small accumulator whose last contributor (per output slice) writes BF16.
//
//  A  router: the cluster's CTAs each score E/CS experts (x . W_router rows
//     staged by 1-D bulk copies), broadcast the logits over DSMEM; every CTA then
//     runs softmax + top-K and cluster c takes the c-th ranked expert.
//  B  sketch scores: each CTA stages its 16-row tiles of the packed 2-bit sketch,
//     scores them on the tensor cores (the packed codes are the bf16 A fragment),
//     broadcasts alpha*|T.x| to the cluster; z = B_e x rows alongside.
//  C  exact top-k: every CTA selects the same k channels (radix select, ties to the
//     lower index); each CTA streams its share of the 6d-byte channel records
//     through a shared-memory ring and accumulates SwiGLU(gate.x, up.x) * down.
//  D  partial outputs are reduce-added into the owning CTA's slice over DSMEM;
//     the owner adds A_e z, scales by the router weight and adds into the FP32
//     accumulator; the last contribution to a slice converts it to BF16.
//
// The kernel is launched with programmatic stream serialisation: everything that
// reads only weights (barrier set-up, router rows) runs before
// griddepcontrol.wait, so it overlaps the previous launch's tail.
//
// "KAIST drops calibration from MoE decoding ...": "Top-k instead of a threshold"
// (fixed read budget), "A reader built from weights alone" (ternary sketch filter
// + low-rank compensation).  No TMA multicast and no peer memory is used.
#include <cooperative_groups.h>

#include "block_scan.cuh"
#include "common.cuh"
#include "fused.h"

namespace cg = cooperative_groups;

namespace msb {

constexpr int kFT = 256;        // threads per CTA
constexpr int kFW = kFT / 32;   // warps per CTA
constexpr int kRingMax = 16;    // record slots
constexpr int kSmemMax = 227 * 1024;
constexpr int kSmemPair = 110 * 1024;  // fallback pairing limit if the device cannot be queried
constexpr int kAregs = 8;              // register quads for the slice's A_e rows (8 bf16 each)
constexpr int kMyselMax = 256;         // channels one CTA reads at most
constexpr int kSelBins = 2048;         // select histogram bins (256 per octave below the largest key)
constexpr int kCandMax = 64;           // keys ranked directly in the k-th key's bin

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
  float* y_acc;
  TraceDev tr;
  Dims D;
  int k, dense, cs, cpe;
  int epad;    // router logits padded to a multiple of 64 (with -inf)
  int rpc;     // router rows per CTA
  int tpc;     // sketch row tiles per CTA
  int zpc;     // z rows per CTA (max)
  int slice;   // output elements owned per CTA (d / cs)
  int ring;    // record slots
  int rs;      // ring slot stride in bf16 elements: 3d + 8 (16 bytes of stagger between
               // slots, so rows of consecutive slots fall in different banks)
  int group;   // channels per reduction group (<= ring)
  // shared-memory carve-up (byte offsets)
  int o_z, o_ylr, o_misc, o_big;  // shared-memory offsets
  int o_logits, o_xperm, o_keys, o_alpha, o_part, o_hist, o_xbig;  // offsets in big
  int o_aslice_off;  // A_e rows: byte offset inside big, past every other use of big
  int aslice_regs;   // 1: A_e rows of the slice are held in registers instead
  int smem;
};

struct Misc {
  uint64_t bar[2 + kRingMax];
  int ids[MSB_MAX_TOP_E];
  float lv[MSB_MAX_TOP_E];  // routed logits in rank order
  uint32_t info[2];
  float h[kRingMax];
  float red[kFW][2 * kRingMax];  // per-warp (gate . x, up . x) of a group's channels
  // channel select scratch
  uint32_t wt[kFW];            // per-warp totals of the bin scan
  uint32_t wgt[kFW], weq[kFW]; // per warp range: keys above the k-th, keys equal to it
  uint32_t kb, rem, cnt, ccount, kth, need;
  uint32_t ck[kCandMax];       // keys of the bin holding the k-th key, and their indices
  uint32_t ci[kCandMax];
  uint32_t cmax[16];           // largest score key of each CTA of the cluster
  uint32_t lmax;               // largest score key of this CTA
  uint32_t tie;                // router: a rank slot was claimed twice
  uint16_t mysel[kMyselMax];  // this CTA's share of the selected channels
  int last;
};

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// The kernel runs once per CTA per launch, so its code is fetched cold every time
// (on B200, cold straight-line code costs ~0.4 us per KB per SM).  It is written
// for a small footprint: loops with short bodies, shared helpers kept out of line,
// fast intrinsics for the few transcendental steps.

// Bounded wait on an mbarrier phase (shared by every wait site).
__device__ __noinline__ bool wait_phase(uint64_t* bar, uint32_t parity, uint32_t* err) {
  return mbar_wait(bar, parity, err);
}

// Router top-K over the E logits in shared memory (padded with -inf to Epad, a
// multiple of 64), by rank counting, P = 256/E threads per logit (at most 4) on
// 16-value vector steps.  Fast pass: rank = #{e' : l_e' > l_e}; the owner of rank
// j < K claims slot j.  Without ties among the top K every claim lands in its own
// slot and these ranks are exact; two logits with the same value have the same
// count, so a tie shows as a second claim on one slot, and then the exact pass
// ranks by #{e' : l_e' > l_e} + #{e' < e : l_e' == l_e} (ties to the lower index).
// M.ids must be -1 and M.tie 0 on entry.  Ends with a barrier.
__device__ __noinline__ void router_rank(const float* logits, int E, int Epad, int K, Misc& M,
                                         uint32_t* err) {
  const int tid = threadIdx.x;
  const int lgP = E <= 64 ? 2 : (E <= 128 ? 1 : 0);
  const int span = Epad >> lgP;
#pragma unroll 1
  for (int pass = 0; pass < 2; ++pass) {
#pragma unroll 1
    for (int base = 0; base < (E << lgP); base += kFT) {
      const int item = base + tid, ee = item >> lgP, h = item & ((1 << lgP) - 1);
      float gt = 0.f;
      float v = 0.f;
      if (ee < E) {
        v = logits[ee];
        if (pass == 0) {
          if (!isfinite(v)) atomicOr(err, kErrNonFinite);
          const float4* lp = reinterpret_cast<const float4*>(logits + h * span);
#pragma unroll 4
          for (int c = 0; c < span / 4; ++c) {
            const float4 u = lp[c];
            gt += (u.x > v ? 1.f : 0.f) + (u.y > v ? 1.f : 0.f);
            gt += (u.z > v ? 1.f : 0.f) + (u.w > v ? 1.f : 0.f);
          }
        } else {
          int r = 0;
#pragma unroll 1
          for (int j = h * span; j < (h + 1) * span; ++j) {
            const float u = logits[j];
            r += (u > v) || (u == v && j < ee);
          }
          gt = (float)r;
        }
      }
      if (lgP >= 1) gt += __shfl_xor_sync(0xffffffffu, gt, 1);
      if (lgP >= 2) gt += __shfl_xor_sync(0xffffffffu, gt, 2);
      const int rank = (int)gt;
      if (ee < E && h == 0 && rank < K) {
        if (atomicCAS(&M.ids[rank], -1, ee) != -1) M.tie = 1u;
        M.lv[rank] = v;
      }
    }
    __syncthreads();
    if (pass == 1 || M.tie == 0u) break;
    if (tid < K) M.ids[tid] = -1;
    __syncthreads();
  }
}

// Combine weight of the routed expert of rank j (every lane of the warp calls it,
// after router_rank): softmax over the K routed logits (renorm) or over all E
// logits.  lv[0] is the largest logit.
__device__ __forceinline__ float router_weight(const float* logits, int E, int K, int renorm,
                                               const Misc& M, int j) {
  const int lane = threadIdx.x & 31;
  const float mx = M.lv[0];
  const float pl = lane < K ? __expf(M.lv[lane] - mx) : 0.f;
  float denom = 0.f;
  if (renorm) {
    denom = pl;
  } else {
#pragma unroll 1
    for (int i = lane; i < E; i += 32) denom += __expf(logits[i] - mx);
  }
  denom = warp_sum(denom);
  return __fdividef(__shfl_sync(0xffffffffu, pl, j), denom);
}

// Exact top-k of the n channel scores (keys = float bits, so integer order is value
// order), ties to the lower index; writes this CTA's share, positions [c0, c1) of
// the ascending selected list, to M.mysel and (when trace is set) the whole list to
// trace.  Keys are binned by (maxkey - key) >> 15 (256 bins per octave below the
// largest key, bin 0 the largest, the last bin catching the rest): one counting
// pass and one scan find the bin of the k-th key, whose keys are then ranked
// directly; a bin with more than kCandMax keys falls back to a radix descent.
// hist: kSelBins zeroed words.  M.ccount must be 0 on entry.
__device__ __noinline__ void select_share(const uint32_t* keys, int n, int k, uint32_t maxkey,
                                          uint32_t* hist, Misc& M, int c0, int c1, uint16_t* trace) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
#pragma unroll 4
  for (int j = tid; j < n; j += kFT) atomicAdd(&hist[min((uint32_t)(kSelBins - 1), (maxkey - keys[j]) >> 15)], 1u);
  __syncthreads();
  // thread t owns bins [8t, 8t + 8)
  uint32_t c[8];
  {
    const uint4 a = reinterpret_cast<const uint4*>(hist)[2 * tid];
    const uint4 b = reinterpret_cast<const uint4*>(hist)[2 * tid + 1];
    c[0] = a.x; c[1] = a.y; c[2] = a.z; c[3] = a.w; c[4] = b.x; c[5] = b.y; c[6] = b.z; c[7] = b.w;
  }
  uint32_t local = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) local += c[i];
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) M.wt[warp] = incl;
  __syncthreads();
  uint32_t above = incl - local;
#pragma unroll
  for (int w = 0; w < kFW; ++w) above += w < warp ? M.wt[w] : 0u;
  const uint32_t kk = (uint32_t)k;
  if (above < kk && kk <= above + local) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (above < kk && kk <= above + c[i]) { M.kb = 8 * tid + i; M.rem = kk - above; M.cnt = c[i]; }
      above += c[i];
    }
  }
  __syncthreads();
  const uint32_t kb = M.kb, rem = M.rem, cnt = M.cnt;
  // scatter layout: warp w owns the indices [w * span, (w + 1) * span)
  const int span = 32 * ((n + kFT - 1) / kFT);
  const int wb = warp * span, we = min(n, wb + span);
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t kth, need;
  if (cnt > (uint32_t)kCandMax) {  // heavy ties: radix descent, then count per warp range
    radix_kth_smem<kFT>(keys, n, k, hist, M.info, &kth, &need);
    uint32_t ngt = 0, neq = 0;
#pragma unroll 4
    for (int j0 = wb; j0 < we; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t key = j < we ? keys[j] : 0u;
      ngt += __popc(__ballot_sync(0xffffffffu, j < we && key > kth));
      neq += __popc(__ballot_sync(0xffffffffu, j < we && key == kth));
    }
    if (lane == 0) { M.wgt[warp] = ngt; M.weq[warp] = neq; }
    __syncthreads();
  } else {
    // gather the bin's keys; keys of higher bins (larger keys) are counted per warp range
    uint32_t ngt = 0;
#pragma unroll 4
    for (int j0 = wb; j0 < we; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t key = j < we ? keys[j] : 0u;
      const uint32_t bin = min((uint32_t)(kSelBins - 1), (maxkey - key) >> 15);
      ngt += __popc(__ballot_sync(0xffffffffu, j < we && bin < kb));
      const bool m = j < we && bin == kb;
      const uint32_t mb = __ballot_sync(0xffffffffu, m);
      if (mb) {
        const int leader = __ffs(mb) - 1;
        uint32_t slot0 = 0;
        if (lane == leader) slot0 = atomicAdd(&M.ccount, (uint32_t)__popc(mb));
        slot0 = __shfl_sync(0xffffffffu, slot0, leader);
        if (m) {
          const uint32_t slot = slot0 + __popc(mb & lt);
          M.ck[slot] = key;
          M.ci[slot] = (uint32_t)j;
        }
      }
    }
    if (lane == 0) { M.wgt[warp] = ngt; M.weq[warp] = 0u; }
    __syncthreads();
    // rank inside the bin by (key desc, index asc); the k-th key sits at position rem - 1.
    // A candidate whose equal keys occupy positions [gt, gt + eq) is above the k-th key
    // if rem - 1 >= gt + eq, equal to it if gt <= rem - 1 < gt + eq.
    if (tid < (int)cnt) {
      const uint32_t mk = M.ck[tid], mi = M.ci[tid];
      uint32_t gt = 0, eq = 0;
#pragma unroll 4
      for (int i = 0; i < (int)cnt; ++i) {
        const uint32_t ok_ = M.ck[i];
        gt += ok_ > mk;
        eq += ok_ == mk;
      }
      const uint32_t pk = rem - 1u, w = mi / (uint32_t)span;
      if (pk >= gt + eq) {
        atomicAdd(&M.wgt[w], 1u);
      } else if (pk >= gt) {
        atomicAdd(&M.weq[w], 1u);
        M.kth = mk;
        M.need = rem - gt;
      }
    }
    __syncthreads();
    kth = M.kth;
    need = M.need;
  }
  uint32_t gtb = 0, eqb = 0;
#pragma unroll
  for (int w = 0; w < kFW; ++w) {
    gtb += w < warp ? M.wgt[w] : 0u;
    eqb += w < warp ? M.weq[w] : 0u;
  }
  const uint32_t ltm = (1u << lane) - 1u;
#pragma unroll 4
  for (int j0 = wb; j0 < we; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = j < we ? keys[j] : 0u;
    const uint32_t bg = __ballot_sync(0xffffffffu, j < we && key > kth);
    const uint32_t be = __ballot_sync(0xffffffffu, j < we && key == kth);
    const uint32_t eqr = eqb + __popc(be & ltm);
    if (((bg >> lane) & 1u) || (((be >> lane) & 1u) && eqr < need)) {
      const int pos = (int)(gtb + __popc(bg & ltm) + min(eqr, need));
      if (pos >= c0 && pos < c1) M.mysel[pos - c0] = (uint16_t)j;
      if (trace) trace[pos] = (uint16_t)j;
    }
    gtb += __popc(bg);
    eqb += __popc(be);
  }
  __syncthreads();
}

// Sketch scores of this CTA's nt row tiles: warp w takes chunks [kc0, kc1) of every
// tile; the packed 2-bit codes are the bf16 A fragments (+-2 or 0), x is B.
// Partial sums go to part[warp][tile*16 + row].
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

template <int IT>  // IT = ceil(d / 2048): 8-element groups per thread
__global__ void __launch_bounds__(kFT, 1) fused_block_kernel(const __grid_constant__ FusedParams P) {
  extern __shared__ __align__(128) uint8_t sm[];
  cg::cluster_group cluster = cg::this_cluster();
  const int CS = P.cs;
  const int q = (int)cluster.block_rank();
  const int cid = blockIdx.x / CS;
  const int rc = cid / P.cpe;     // which routed expert (rank order)
  const int half = cid % P.cpe;   // which cluster of that expert
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Dims D = P.D;
  const int d = D.d, E = D.experts, I = D.inter, ipad = D.ipad, r = D.rank, K = D.top_e;
  const int KC = d / kColChunk;

  float* zs = reinterpret_cast<float*>(sm + P.o_z);
  float* ylr = reinterpret_cast<float*>(sm + P.o_ylr);     // A_e z on this CTA's slice
  Misc& M = *reinterpret_cast<Misc*>(sm + P.o_misc);
  uint8_t* big = sm + P.o_big;
  // `big` is reused phase by phase (offsets from the plan):
  //   A: router rows at 0, logits (remote-written) after them
  //   B: sketch tiles at 0, B_e rows, alpha, partial sums, x fragments, scores (remote-written)
  //   C: the record ring at 0          D: the partial output at 0
  //   A_e rows sit past all of these (loaded in B, read after the ring drains)
  uint16_t* xs = reinterpret_cast<uint16_t*>(big + P.o_xbig);  // phases A-B (C reads x from L1/L2)
  float* logits = reinterpret_cast<float*>(big + P.o_logits);
  uint32_t* xperm = reinterpret_cast<uint32_t*>(big + P.o_xperm);
  uint32_t* keys = reinterpret_cast<uint32_t*>(big + P.o_keys);  // channel scores (float bits)
  float* alpha_s = reinterpret_cast<float*>(big + P.o_alpha);
  float* part = reinterpret_cast<float*>(big + P.o_part);
  uint32_t* hist = reinterpret_cast<uint32_t*>(big + P.o_hist);  // phase C select
  float* ybuf = reinterpret_cast<float*>(big);             // phase D: partial output (over the ring)

  // Every CTA of the cluster must be running before any DSMEM access targets it:
  // arrive now, wait just before the first remote access.
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");

  // ------------------------------------------------------------------ prologue (weights only)
  const int e_lo = min(E, q * P.rpc), e_hi = min(E, e_lo + P.rpc);
  const uint32_t rbytes = (uint32_t)(e_hi - e_lo) * 2u * d;
  if (tid == 0) {
#pragma unroll 1
    for (int i = 0; i < 2 + P.ring; ++i) mbar_init(&M.bar[i], 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&M.bar[0], rbytes);
    if (rbytes) bulk_g2s(big, P.router_t + (size_t)e_lo * d, rbytes, &M.bar[0]);
  }
#pragma unroll 1
  for (int i = tid; i < P.slice; i += kFT) ylr[i] = 0.f;
  for (int i = E + tid; i < P.epad; i += kFT) logits[i] = -INFINITY;
  if (tid < K) M.ids[tid] = -1;
  if (tid == 0) { M.lmax = 0u; M.ccount = 0u; M.tie = 0u; }
  // x and the workspace may be written by the previous launch: wait for it here.
  pdl_wait();
#pragma unroll 1
  for (int i = tid; i < d / 8; i += kFT)
    reinterpret_cast<uint4*>(xs)[i] = __ldg(reinterpret_cast<const uint4*>(P.x) + i);
  __syncthreads();

  // ------------------------------------------------------------------ phase A: router
  bool ok = wait_phase(&M.bar[0], 0, P.err);
  ok = __syncthreads_and(ok);
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  if (ok) {
    const uint16_t* rows = reinterpret_cast<const uint16_t*>(big);
#pragma unroll 1
    for (int row = warp; row < e_hi - e_lo; row += kFW) {
      const uint4* wr = reinterpret_cast<const uint4*>(rows + (size_t)row * d);
      const uint4* xr = reinterpret_cast<const uint4*>(xs);
      float acc = 0.f;
#pragma unroll 2
      for (int i = lane; i < d / 8; i += 32) acc = dot8(wr[i], xr[i], acc);
      acc = warp_sum(acc);
      if (lane < CS) cluster.map_shared_rank(logits, lane)[e_lo + row] = acc;
    }
  }
  cluster.sync();
  router_rank(logits, E, P.epad, K, M, P.err);
  int e = M.ids[rc];
  if (e < 0) {  // a rank left empty (non-finite logits): keep a valid index, the call is flagged
    e = rc;
    if (tid == 0) atomicOr(P.err, kErrNonFinite);
  }
  const float we = router_weight(logits, E, K, D.renorm, M, rc);
  if (blockIdx.x == 0) {
    if (warp == 0) {  // (the weight of a non-renormalised softmax is a warp-wide sum)
      const float wl = router_weight(logits, E, K, D.renorm, M, lane < K ? lane : 0);

      if (lane < K && P.tr.expert_ids) P.tr.expert_ids[lane] = M.ids[lane] < 0 ? lane : M.ids[lane];
      if (lane < K && P.tr.expert_w) P.tr.expert_w[lane] = wl;
    }
    if (P.tr.union_count)
#pragma unroll 1
      for (int i = tid; i < E; i += kFT) {
        int c = 0;
        for (int j = 0; j < K; ++j) c = (M.ids[j] == i) ? P.k : c;  // (-1 never matches)
        P.tr.union_count[i] = c;
      }
  }

  // ------------------------------------------------------------------ phase B: scores, z
  const int ntile_all = ipad / kRowTile;
  const int lt0 = min(ntile_all, q * P.tpc), lt1 = min(ntile_all, lt0 + P.tpc);
  const int nt = lt1 - lt0;
  const uint32_t code_bytes = P.dense ? 0u : (uint32_t)nt * KC * kChunkWords * 4u;
  const int nz = r > q ? (r - q + CS - 1) / CS : 0;  // z rows q, q+CS, ... below r
  const bool lr_out = (half == 0 && r > 0);
  uint16_t* brows = reinterpret_cast<uint16_t*>(big + code_bytes);
  uint16_t* aslice = reinterpret_cast<uint16_t*>(big + P.o_aslice_off);
  const bool lr_smem = lr_out && !P.aslice_regs;
  if (tid == 0 && ok) {
    uint32_t bytes = code_bytes + (P.dense ? 0u : (uint32_t)nt * kRowTile * 4u) + (uint32_t)nz * 2u * d;
    if (lr_smem) bytes += (uint32_t)P.slice * r * 2u;
    fence_proxy_async();
    mbar_arrive_expect_tx(&M.bar[1], bytes);
    if (code_bytes) {
      bulk_g2s(big, P.sketch + ((size_t)e * ntile_all + lt0) * KC * kChunkWords, code_bytes, &M.bar[1]);
      bulk_g2s(alpha_s, P.alpha + (size_t)e * ipad + (size_t)lt0 * kRowTile, nt * kRowTile * 4u,
               &M.bar[1]);
    }
#pragma unroll 1
    for (int i = 0; i < nz; ++i)
      bulk_g2s(brows + (size_t)i * d, P.lr_b + ((size_t)e * r + q + i * CS) * d, 2u * d, &M.bar[1]);
    if (lr_smem)
      bulk_g2s(aslice, P.lr_a + ((size_t)e * d + (size_t)q * P.slice) * r, (uint32_t)P.slice * r * 2u,
               &M.bar[1]);
  }
  // A_e rows of this CTA's output slice into registers (8 bf16 per quad), when they fit
  uint4 areg[kAregs];
  const int nachunk = (lr_out && P.aslice_regs) ? P.slice * r / 8 : 0;
#pragma unroll
  for (int u = 0; u < kAregs; ++u) {
    const int j = tid + u * kFT;
    areg[u] = make_uint4(0u, 0u, 0u, 0u);
    if (ok && j < nachunk)
      areg[u] = __ldg(reinterpret_cast<const uint4*>(P.lr_a + ((size_t)e * d + (size_t)q * P.slice) * r) + j);
  }
  // phase-B scratch in big (past the tiles and B_e rows, which are still landing)
#pragma unroll 1
  for (int i = tid; i < kFW * P.tpc * kRowTile; i += kFT) part[i] = 0.f;
  if (!P.dense)
#pragma unroll 1
    for (int i = tid; i < kSelBins / 4; i += kFT) reinterpret_cast<uint4*>(hist)[i] = make_uint4(0u, 0u, 0u, 0u);
  // xperm[kc][c][s][p] = the bf16 pair of x at column 64*kc + 16*s + 2*c + 8*p
#pragma unroll 1
  for (int i = tid; i < d / 2; i += kFT) {
    const int kc = i >> 5, c = (i >> 3) & 3, q8 = i & 7;
    xperm[i] = reinterpret_cast<const uint32_t*>(xs)[kc * 32 + 8 * (q8 >> 1) + c + 4 * (q8 & 1)];
  }
  ok = ok && wait_phase(&M.bar[1], 0, P.err);
  ok = __syncthreads_and(ok);
  if (ok && !P.dense && nt > 0)
    score_tiles(reinterpret_cast<const uint2*>(big), reinterpret_cast<const uint4*>(xperm), nt, KC,
                part + warp * P.tpc * kRowTile);
  // z rows: z[rho] = B_e[rho] . x, broadcast to the cluster
  if (ok && r > 0) {
#pragma unroll 1
    for (int i = warp; i < nz; i += kFW) {
      const uint4* br = reinterpret_cast<const uint4*>(brows + (size_t)i * d);
      const uint4* xr = reinterpret_cast<const uint4*>(xs);
      float acc = 0.f;
#pragma unroll 2
      for (int j = lane; j < d / 8; j += 32) acc = dot8(br[j], xr[j], acc);
      acc = warp_sum(acc);
      if (lane < CS) cluster.map_shared_rank(zs, lane)[q + i * CS] = acc;
    }
  }
  __syncthreads();
  const int nrows = (ok && !P.dense) ? nt * kRowTile : 0;
  // score = alpha * |sum of the 8 warps' partials| / 2 (into part's first row) ...
  uint32_t lmax = 0;
#pragma unroll 1
  for (int lr = tid; lr < nrows; lr += kFT) {
    float sc = 0.f;
#pragma unroll
    for (int w = 1; w < kFW; ++w) sc += part[w * P.tpc * kRowTile + lr];
    sc = alpha_s[lr] * fabsf(sc + part[lr]) * 0.5f;
    part[lr] = sc;
    lmax = max(lmax, __float_as_uint(sc));
    if (half == 0 && P.tr.scores) P.tr.scores[(size_t)rc * ipad + lt0 * kRowTile + lr] = sc;
  }
  lmax = __reduce_max_sync(0xffffffffu, lmax);
  if (lane == 0 && lmax) atomicMax(&M.lmax, lmax);
  __syncthreads();
  // ... then broadcast to every CTA of the cluster: item i -> (row i / CS, CTA i % CS),
  // with this CTA's largest key
  if (tid < CS) cluster.map_shared_rank(M.cmax, tid)[q] = M.lmax;
  const int lg = CS == 16 ? 4 : 3;
#pragma unroll 1
  for (int i = tid; i < nrows * CS; i += kFT)
    cluster.map_shared_rank(keys, i & (CS - 1))[lt0 * kRowTile + (i >> lg)] =
        __float_as_uint(part[i >> lg]);
  cluster.sync();
  pdl_trigger();  // the next launch may start its weight-only prologue

  // ------------------------------------------------------------------ phase C: top-k, records
  // this CTA's share of the k channels: positions [c0, c1) of the ascending list
  const int NQ = CS * P.cpe, gq = half * CS + q;
  const int c0 = gq * P.k / NQ, c1 = (gq + 1) * P.k / NQ;
  const int nmine = c1 - c0;
  if (!P.dense) {
    uint32_t maxkey = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) maxkey = i < CS ? max(maxkey, M.cmax[i]) : maxkey;
    uint16_t* trace = (half == 0 && q == 0 && P.tr.sel) ? P.tr.sel + (size_t)rc * P.k : nullptr;
    select_share(keys, I, P.k, maxkey, hist, M, c0, c1, trace);
    if (half == 0 && q == 0 && tid == 0 && P.tr.sel_count) P.tr.sel_count[rc] = P.k;
  } else {
#pragma unroll 1
    for (int i = tid; i < nmine; i += kFT) M.mysel[i] = (uint16_t)(c0 + i);
    __syncthreads();
  }
  const uint32_t rec_bytes = 6u * d;
  uint16_t* ring = reinterpret_cast<uint16_t*>(big);
  if (warp == 0 && ok) {  // lane i issues the copy into slot i
    fence_proxy_async();
    const int first = min(P.ring, nmine);
    if (lane < first) {
      const int ch = M.mysel[lane];
      mbar_arrive_expect_tx(&M.bar[2 + lane], rec_bytes);
      bulk_g2s(ring + (size_t)lane * P.rs, P.records + ((size_t)e * I + ch) * 3 * d, rec_bytes,
               &M.bar[2 + lane]);
    }
  }
  // A_e z on this CTA's output slice, while the records are in flight
  if (ok && lr_out) {
    if (P.aslice_regs) {
      const int cpr = r / 8;  // register quads per A_e row
#pragma unroll
      for (int u = 0; u < kAregs; ++u) {
        const int j = tid + u * kFT;
        if (j < nachunk) {
          const int row = j / cpr, rho0 = (j - row * cpr) * 8;
          const float* zz = zs + rho0;
          float acc = bf16_lo(areg[u].x) * zz[0];
          acc = fmaf(bf16_hi(areg[u].x), zz[1], acc);
          acc = fmaf(bf16_lo(areg[u].y), zz[2], acc);
          acc = fmaf(bf16_hi(areg[u].y), zz[3], acc);
          acc = fmaf(bf16_lo(areg[u].z), zz[4], acc);
          acc = fmaf(bf16_hi(areg[u].z), zz[5], acc);
          acc = fmaf(bf16_lo(areg[u].w), zz[6], acc);
          acc = fmaf(bf16_hi(areg[u].w), zz[7], acc);
          atomicAdd(&ylr[row], acc);
        }
      }
    } else {
#pragma unroll 1
      for (int i = tid; i < P.slice; i += kFT) {
        const uint16_t* arow = aslice + (size_t)i * r;
        float acc = 0.f;
#pragma unroll 1
        for (int rho = 0; rho < r; ++rho) acc = fmaf(bf16_lo(arow[rho]), zs[rho], acc);
        ylr[i] = acc;
      }
    }
  }

  // Per group: gate . x and up . x of the group's channels on the tensor cores (A =
  // the records' gate/up rows, bf16 straight from the ring via ldmatrix; B = x; warp w
  // takes k-steps [ks0, ks1) and the warps' partials meet in
  // M.red), then h, then y += h_i * down_i with every thread owning 8-element groups.
  const int KS = d / 16;
  const int ks0 = warp * KS / kFW, ks1 = (warp + 1) * KS / kFW;
  const uint32_t* x32 = reinterpret_cast<const uint32_t*>(P.x);
  const int c4 = lane & 3, g8 = lane >> 2;
  // d <= 2048: the x B-fragments of this warp's k-steps sit in registers (loaded while
  // the records are in flight); larger d reads them through L1 at each k-step
  constexpr int KSW = IT == 1 ? 16 : 0;
  uint32_t xb[KSW > 0 ? KSW : 1][2];
#pragma unroll
  for (int i = 0; i < KSW; ++i)
    if (ks0 + i < ks1) {
      xb[i][0] = __ldg(x32 + (ks0 + i) * 8 + c4);
      xb[i][1] = __ldg(x32 + (ks0 + i) * 8 + 4 + c4);
    }
  float y[IT][8];
#pragma unroll
  for (int it = 0; it < IT; ++it)
#pragma unroll
    for (int i = 0; i < 8; ++i) y[it][i] = 0.f;
  // channel g0 + i of a group sits in slot s0 + i (wrapping at the ring size, where the
  // slot's phase parity flips); s0 and its parity par0 advance group by group
  int s0 = 0;
  uint32_t par0 = 0;
#pragma unroll 1
  for (int g0 = 0; g0 < nmine; g0 += P.group) {
    const int ng = min(P.group, nmine - g0);
#pragma unroll 1
    for (int i = 0; i < ng; ++i) {
      const int sl = s0 + i < P.ring ? s0 + i : s0 + i - P.ring;
      ok = ok && wait_phase(&M.bar[2 + sl], s0 + i < P.ring ? par0 : par0 ^ 1u, P.err);
    }
#pragma unroll 1
    for (int tb = 0; tb < ng; tb += 8) {
      // this lane's ldmatrix row: channel tb + lane % 8 (rows past ng repeat channel tb;
      // their results are dropped), gate (lanes 0-7, 16-23) or up, k offset 8 * (lane / 16)
      const int ch = (tb + (lane & 7) < ng) ? tb + (lane & 7) : tb;
      const int csl = s0 + ch < P.ring ? s0 + ch : s0 + ch - P.ring;
      uint32_t a_addr = smem_addr(ring + (size_t)csl * P.rs + ((lane >> 3) & 1) * d +
                                  8 * (lane >> 4)) + 32u * ks0;
      float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
      int ks = ks0;
      if (ok && KSW > 0) {
#pragma unroll
        for (int i = 0; i < KSW; i += 2) {
          if (ks0 + i + 1 < ks1) {
            uint32_t a[2][4];
            ldsm_x4(a_addr + 32u * i, a[0][0], a[0][1], a[0][2], a[0][3]);
            ldsm_x4(a_addr + 32u * (i + 1), a[1][0], a[1][1], a[1][2], a[1][3]);
            mma_bf16(acc0, a[0][0], a[0][1], a[0][2], a[0][3], xb[i][0], xb[i][1]);
            mma_bf16(acc1, a[1][0], a[1][1], a[1][2], a[1][3], xb[i + 1][0], xb[i + 1][1]);
          } else if (ks0 + i < ks1) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(a_addr + 32u * i, a0, a1, a2, a3);
            mma_bf16(acc0, a0, a1, a2, a3, xb[i][0], xb[i][1]);
          }
        }
      } else if (ok) {
#pragma unroll 1
        for (; ks + 4 <= ks1; ks += 4, a_addr += 128u) {
          uint32_t a[4][4], b[4][2];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            ldsm_x4(a_addr + 32u * u, a[u][0], a[u][1], a[u][2], a[u][3]);
            b[u][0] = __ldg(x32 + (ks + u) * 8 + c4);
            b[u][1] = __ldg(x32 + (ks + u) * 8 + 4 + c4);
          }
          mma_bf16(acc0, a[0][0], a[0][1], a[0][2], a[0][3], b[0][0], b[0][1]);
          mma_bf16(acc1, a[1][0], a[1][1], a[1][2], a[1][3], b[1][0], b[1][1]);
          mma_bf16(acc0, a[2][0], a[2][1], a[2][2], a[2][3], b[2][0], b[2][1]);
          mma_bf16(acc1, a[3][0], a[3][1], a[3][2], a[3][3], b[3][0], b[3][1]);
        }
#pragma unroll 1
        for (; ks < ks1; ++ks, a_addr += 32u) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4(a_addr, a0, a1, a2, a3);
          mma_bf16(acc0, a0, a1, a2, a3, __ldg(x32 + ks * 8 + c4), __ldg(x32 + ks * 8 + 4 + c4));
        }
      }
      // column 0 of D: lanes with lane % 4 == 0 hold gate (row g8) and up (row g8 + 8)
      if (c4 == 0 && tb + g8 < ng) {
        M.red[warp][2 * (tb + g8)] = acc0[0] + acc1[0];
        M.red[warp][2 * (tb + g8) + 1] = acc0[2] + acc1[2];
      }
    }
    ok = __syncthreads_and(ok);
    if (tid < ng) {
      float g = 0.f, u = 0.f;
#pragma unroll
      for (int w = 0; w < kFW; ++w) { g += M.red[w][2 * tid]; u += M.red[w][2 * tid + 1]; }
      M.h[tid] = __fdividef(g, 1.0f + __expf(-g)) * u;
    }
    __syncthreads();
    if (ok) {
      // y += h_i * down_i over this thread's elements
#pragma unroll 4
      for (int i = 0; i < ng; ++i) {
        const int sl = s0 + i < P.ring ? s0 + i : s0 + i - P.ring;
        const uint16_t* rec = ring + (size_t)sl * P.rs + 2 * d;
        const float h = M.h[i];
#pragma unroll
        for (int it = 0; it < IT; ++it) {
          const int el = (it * kFT + tid) * 8;
          if (el < d) {
            const uint4 dv = *reinterpret_cast<const uint4*>(rec + el);
            y[it][0] = fmaf(h, bf16_lo(dv.x), y[it][0]);
            y[it][1] = fmaf(h, bf16_hi(dv.x), y[it][1]);
            y[it][2] = fmaf(h, bf16_lo(dv.y), y[it][2]);
            y[it][3] = fmaf(h, bf16_hi(dv.y), y[it][3]);
            y[it][4] = fmaf(h, bf16_lo(dv.z), y[it][4]);
            y[it][5] = fmaf(h, bf16_hi(dv.z), y[it][5]);
            y[it][6] = fmaf(h, bf16_lo(dv.w), y[it][6]);
            y[it][7] = fmaf(h, bf16_hi(dv.w), y[it][7]);
          }
        }
      }
    }
    __syncthreads();
    // refill the slots just consumed
    if (warp == 0 && ok) {  // channel g0 + i + ring goes where g0 + i was; lane i issues it
      fence_proxy_async();
      const int i = lane, nx = g0 + lane + P.ring;
      if (i < ng && nx < nmine) {
        const int ch = M.mysel[nx];
        const int slot = s0 + i < P.ring ? s0 + i : s0 + i - P.ring;
        mbar_arrive_expect_tx(&M.bar[2 + slot], rec_bytes);
        bulk_g2s(ring + (size_t)slot * P.rs, P.records + ((size_t)e * I + ch) * 3 * d, rec_bytes,
                 &M.bar[2 + slot]);
      }
    }
    s0 += ng;
    if (s0 >= P.ring) {
      s0 -= P.ring;
      par0 ^= 1u;
    }
  }

  // ------------------------------------------------------------------ phase D: reduce, combine
  // partial output to this CTA's shared buffer; each owner then sums its slice over
  // the cluster with 16-byte DSMEM loads
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int el = (it * kFT + tid) * 8;
    if (el < d) {
      *reinterpret_cast<float4*>(ybuf + el) = make_float4(y[it][0], y[it][1], y[it][2], y[it][3]);
      *reinterpret_cast<float4*>(ybuf + el + 4) = make_float4(y[it][4], y[it][5], y[it][6], y[it][7]);
    }
  }
  cluster.sync();
  if (ok) {
#pragma unroll 1
    for (int j = tid; j < P.slice / 4; j += kFT) {
      const int el = q * P.slice + 4 * j;
      // all CS remote loads in flight at once
      float4 v[16];
#pragma unroll
      for (int src = 0; src < 16; ++src)
        if (src < CS) v[src] = *reinterpret_cast<const float4*>(cluster.map_shared_rank(ybuf, src) + el);
      float4 acc = v[0];
#pragma unroll
      for (int src = 1; src < 16; ++src)
        if (src < CS) { acc.x += v[src].x; acc.y += v[src].y; acc.z += v[src].z; acc.w += v[src].w; }
      if (lr_out) {
        acc.x += ylr[4 * j]; acc.y += ylr[4 * j + 1]; acc.z += ylr[4 * j + 2]; acc.w += ylr[4 * j + 3];
      }
      red_add_v4(P.y_acc + el, we * acc.x, we * acc.y, we * acc.z, we * acc.w);
    }
  }
  cluster.sync();  // no CTA leaves while its buffer may still be read
  // the barrier orders warp 0's reduction-adds before thread 0's fence, which makes them
  // visible GPU-wide before the slice counter moves
  if (tid == 0) {
    __threadfence();
    M.last = (atomicAdd(P.slice_cnt + q, 1u) == (uint32_t)(K * P.cpe - 1));
    if (M.last) __threadfence();
  }
  __syncthreads();
  if (M.last) {
    // every contribution to this slice has arrived: convert, re-zero, reset
#pragma unroll 1
    for (int i = tid; i < P.slice; i += kFT) {
      const float v = atomicExch(P.y_acc + q * P.slice + i, 0.f);
      P.out[q * P.slice + i] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    }
    if (tid == 0) P.slice_cnt[q] = 0u;
  }
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

KernelFn kernel_for(int d) {
  const int it = (d + 2047) / 2048;
  if (it <= 1) return fused_block_kernel<1>;
  if (it <= 2) return fused_block_kernel<2>;
  return fused_block_kernel<4>;
}

// Fill the carve-up for cluster size cs within `limit` bytes of shared memory.
bool plan(FusedParams& P, const Dims& D, int k, int cs, int cpe, int limit) {
  const int d = D.d, E = D.experts, ipad = D.ipad, r = D.rank;
  if (d % (8 * cs) != 0) return false;
  P.cs = cs;
  P.cpe = cpe;
  P.rpc = (E + cs - 1) / cs;
  P.tpc = (ipad / kRowTile + cs - 1) / cs;
  P.zpc = (r + cs - 1) / cs;
  P.slice = d / cs;
  int o = 0;
  P.o_z = o;      o = align_up(o + 4 * (r > 0 ? r : 1), 128);
  P.o_ylr = o;    o = align_up(o + 4 * P.slice, 128);
  P.o_misc = o;   o = align_up(o + (int)sizeof(Misc), 128);
  P.o_big = o;
  // offsets inside big (see the kernel): phase A and phase B scratch
  const int need_rows = align_up(P.rpc * 2 * d, 128);
  P.o_logits = need_rows;
  P.epad = (E + 63) / 64 * 64;
  const int need_a = need_rows + align_up(4 * P.epad, 128);
  int b = (P.dense ? 0 : P.tpc * (d / kColChunk) * kChunkWords * 4) + P.zpc * 2 * d;
  b = align_up(b, 128);
  P.o_alpha = b;  b = align_up(b + 4 * P.tpc * kRowTile, 128);
  P.o_part = b;   b = align_up(b + 4 * kFW * P.tpc * kRowTile, 128);
  P.o_xperm = b;  b = align_up(b + 2 * d, 128);
  P.o_keys = b;   b = align_up(b + 4 * ipad, 128);
  P.o_hist = b;   b = align_up(b + (P.dense ? 0 : 4 * kSelBins), 128);
  // x lives past both phases' scratch until the ring takes over
  P.o_xbig = align_up(need_a > b ? need_a : b, 128);
  const int need_b = align_up(P.o_xbig + 2 * d, 128);
  const int need_d = 4 * d;
  if ((k + cs * cpe - 1) / (cs * cpe) > kMyselMax) return false;
  P.aslice_regs = (r > 0 && r % 8 == 0 && P.slice * r / 8 <= kAregs * kFT) ? 1 : 0;
  const int aslice_bytes = P.aslice_regs ? 0 : align_up(P.slice * r * 2, 128);
  const int avail = limit - o - aslice_bytes;
  P.rs = 3 * d + 8;
  const int rec = 2 * P.rs;
  int ring = avail / rec;
  if (ring > kRingMax) ring = kRingMax;
  if (ring < 2 || need_a > avail || need_b > avail || need_d > avail) return false;
  const int per_cta = (k + cs * cpe - 1) / (cs * cpe);  // channels a CTA reads
  if (ring > per_cta) ring = per_cta < 2 ? 2 : per_cta;
  P.ring = ring;
  // one group when every record fits the ring, else two groups in flight
  P.group = per_cta <= ring ? ring : (ring + 1) / 2;
  int bigb = ring * rec;
  if (need_a > bigb) bigb = need_a;
  if (need_b > bigb) bigb = need_b;
  if (need_d > bigb) bigb = need_d;
  P.o_aslice_off = bigb;
  P.smem = o + bigb + aslice_bytes;
  return P.smem <= limit;
}

// Prefer plans whose CTAs can pair on an SM (all clusters then fit the GPCs), then
// one 16-CTA cluster per routed expert when all K are resident, then two 8-CTA
// clusters per expert; otherwise any plan (non-resident clusters run later).
bool choose(FusedParams& P, const Dims& D, int k) {
  const int dev = cur_dev();
  if (dev < 0 || dev >= 64 || !g_ready[dev]) return false;
  const int K = D.top_e;
  const int pair = g_pair_smem[dev];
  const bool have16 = g_max_clusters16[dev] >= 1, have8 = g_max_clusters8[dev] >= 1;
  if (have16 && plan(P, D, k, 16, 1, pair)) return true;
  if (have8 && plan(P, D, k, 8, 2, pair)) return true;
  if (have16 && g_max_clusters16[dev] >= K && plan(P, D, k, 16, 1, kSmemMax)) return true;
  if (have8 && g_max_clusters8[dev] >= 2 * K && plan(P, D, k, 8, 2, kSmemMax)) return true;
  if (have16 && plan(P, D, k, 16, 1, kSmemMax)) return true;
  if (have8 && plan(P, D, k, 8, 2, kSmemMax)) return true;
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
  for (KernelFn fn : {fused_block_kernel<1>, fused_block_kernel<2>, fused_block_kernel<4>}) {
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax) !=
        cudaSuccess)
      return MSB_ECUDA;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
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
  g_max_clusters16[dev] = query_clusters(fused_block_kernel<1>, 16, kSmemMax);
  g_max_clusters8[dev] = query_clusters(fused_block_kernel<1>, 8, kSmemMax);
  g_ready[dev] = true;
  return MSB_OK;
}

void fused_plan_info(const Dims& D, int k, int* info) {
  FusedParams P{};
  P.dense = (k == D.inter);
  const int dev = cur_dev();
  #pragma unroll 1
  for (int i = 0; i < 6; ++i) info[i] = 0;
  if (choose(P, D, k)) {
    info[0] = P.cs;
    info[1] = P.cpe;
    info[2] = P.ring;
    info[3] = P.smem;
  }
  if (dev >= 0 && dev < 64) {
    info[4] = g_max_clusters16[dev];
    info[5] = g_max_clusters8[dev];
  }
}

bool fused_supported(const Dims& D, int k) {
  FusedParams P{};
  P.dense = (k == D.inter);
  return choose(P, D, k);
}

int launch_fused(const uint16_t* x, const uint16_t* router_t, const uint16_t* records,
                 const uint32_t* sketch, const float* alpha, int k, const uint16_t* lr_a,
                 const uint16_t* lr_b, uint16_t* out, const Dims& D, uint32_t* err,
                 uint32_t* counters, float* y_acc, const TraceDev& tr, cudaStream_t st) {
  FusedParams P{};
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
  P.tr = tr;
  P.D = D;
  P.k = k;
  P.dense = (k == D.inter);
  if (!choose(P, D, k)) return MSB_ENOTFUSED;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(P.cs * P.cpe * D.top_e, 1, 1);
  cfg.blockDim = dim3(kFT, 1, 1);
  cfg.dynamicSmemBytes = P.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = P.cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel_for(D.d), P);
  return e == cudaSuccess ? MSB_OK : MSB_ECUDA;
}

}  // namespace msb
