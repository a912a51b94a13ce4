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
constexpr int kGroup = 8;       // channels reduced together
constexpr int kSmemMax = 227 * 1024;
constexpr int kSmemPair = 110 * 1024;  // fallback pairing limit if the device cannot be queried
constexpr int kAregs = 8;              // register quads for the slice's A_e rows (8 bf16 each)

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
  int rpc;     // router rows per CTA
  int tpc;     // sketch row tiles per CTA
  int zpc;     // z rows per CTA (max)
  int slice;   // output elements owned per CTA (d / cs)
  int ring;    // record slots
  int group;   // channels per reduction group (<= ring)
  // shared-memory carve-up (byte offsets)
  int o_x, o_z, o_sel, o_ylr, o_misc, o_big;  // shared-memory offsets
  int o_logits, o_xperm, o_keys, o_alpha, o_part, o_hist;  // byte offsets inside big
  int o_aslice_off;  // A_e rows: byte offset inside big, past every other use of big
  int aslice_regs;   // 1: A_e rows of the slice are held in registers instead
  int smem;
};

struct Misc {
  uint64_t bar[2 + kRingMax];
  int ids[MSB_MAX_TOP_E];
  float w[MSB_MAX_TOP_E];
  uint32_t info[2];
  uint32_t scan[kFT / 32 + 1];
  float h[kGroup];
  float maxv;
  float wsum[kFW];
  float pe[MSB_MAX_TOP_E];
  uint32_t sscr[208];  // select scratch (block scan, results, candidates)
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

// Router top-K over the E logits in shared memory, by rank counting:
// rank(e) = #{e' : l_e' > l_e or (l_e' == l_e and e' < e)}, two threads per logit.
// Writes M.ids[0..K) (rank order) and the combine weights M.w[0..K).
__device__ __noinline__ void router_topk(const float* logits, int E, int K, int renorm, Misc& M,
                                         uint32_t* err) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid < K) M.ids[tid] = -1;
  __syncthreads();
  const int halfE = E / 2;
#pragma unroll 1
  for (int base = 0; base < 2 * E; base += kFT) {
    const int item = base + tid, ee = item >> 1, h = item & 1;
    int rank = 0;
    float v = 0.f;
    if (ee < E) {
      v = logits[ee];
      const int j1 = h ? E : halfE;
#pragma unroll 2
      for (int j = h ? halfE : 0; j < j1; ++j) {
        const float u = logits[j];
        rank += (u > v) || (u == v && j < ee);
      }
    }
    rank += __shfl_xor_sync(0xffffffffu, rank, 1);
    if (ee < E && h == 0) {
      if (rank < K) M.ids[rank] = ee;
      if (rank == 0) M.maxv = v;
    }
  }
  __syncthreads();
  if (tid < K && M.ids[tid] < 0) {  // non-finite logits: keep a valid index and flag the call
    M.ids[tid] = tid;
    atomicOr(err, kErrNonFinite);
  }
  const float mx = M.maxv;
  if (!renorm) {  // the softmax denominator over all E experts is only needed without renorm
    float ps = 0.f;
#pragma unroll 1
    for (int ee = tid; ee < E; ee += kFT) ps += __expf(logits[ee] - mx);
    ps = warp_sum(ps);
    if (lane == 0) M.wsum[warp] = ps;
  }
  if (tid < K) M.pe[tid] = __expf(logits[M.ids[tid]] - mx);
  __syncthreads();
  if (tid < K) {
    float denom = 0.f;
    if (renorm) {
      for (int j = 0; j < K; ++j) denom += M.pe[j];
    } else {
      for (int w = 0; w < kFW; ++w) denom += M.wsum[w];
    }
    M.w[tid] = __fdividef(M.pe[tid], denom);
  }
  __syncthreads();
}

// Exact top-k of the I channel scores (keys = float bits) into sel[0..k), ascending.
// hist4096: 4096 zeroed words of shared memory.
__device__ __noinline__ void select_channels(const uint32_t* keys, int I, int k, uint16_t* sel,
                                             uint32_t* hist4096, Misc& M) {
  uint32_t kth, need;
  hist_kth_smem<kFT>(keys, I, k, hist4096, M.sscr, &kth, &need);
  scatter_topk<kFT>(keys, I, kth, need, sel, M.scan);
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

// One warp per channel: h = silu(gate . x) * (up . x) for channel record `rec`.
__device__ __forceinline__ float channel_h(const uint16_t* rec, const uint16_t* xs, int d) {
  const int lane = threadIdx.x & 31;
  const uint4* gr = reinterpret_cast<const uint4*>(rec);
  const uint4* ur = reinterpret_cast<const uint4*>(rec + d);
  const uint4* xr = reinterpret_cast<const uint4*>(xs);
  float g = 0.f, u = 0.f;
#pragma unroll 2
  for (int i = lane; i < d / 8; i += 32) {
    const uint4 xv = xr[i];
    g = dot8(gr[i], xv, g);
    u = dot8(ur[i], xv, u);
  }
  g = warp_sum(g);
  u = warp_sum(u);
  return __fdividef(g, 1.0f + __expf(-g)) * u;
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

  uint16_t* xs = reinterpret_cast<uint16_t*>(sm + P.o_x);
  float* zs = reinterpret_cast<float*>(sm + P.o_z);
  uint16_t* sel = reinterpret_cast<uint16_t*>(sm + P.o_sel);
  float* ylr = reinterpret_cast<float*>(sm + P.o_ylr);     // A_e z on this CTA's slice
  Misc& M = *reinterpret_cast<Misc*>(sm + P.o_misc);
  uint8_t* big = sm + P.o_big;
  // `big` is reused phase by phase (offsets from the plan):
  //   A: router rows at 0, logits (remote-written) after them
  //   B: sketch tiles at 0, B_e rows, alpha, partial sums, x fragments, scores (remote-written)
  //   C: the record ring at 0          D: the partial output at 0
  //   A_e rows sit past all of these (loaded in B, read after the ring drains)
  float* logits = reinterpret_cast<float*>(big + P.o_logits);
  uint32_t* xperm = reinterpret_cast<uint32_t*>(big + P.o_xperm);
  uint32_t* keys = reinterpret_cast<uint32_t*>(big + P.o_keys);  // channel scores (float bits)
  float* alpha_s = reinterpret_cast<float*>(big + P.o_alpha);
  float* part = reinterpret_cast<float*>(big + P.o_part);
  uint32_t* hist4096 = reinterpret_cast<uint32_t*>(big + P.o_hist);  // phase C select
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
  router_topk(logits, E, K, D.renorm, M, P.err);
  const int e = M.ids[rc];
  const float we = M.w[rc];
  if (blockIdx.x == 0) {
    if (tid < K) {
      if (P.tr.expert_ids) P.tr.expert_ids[tid] = M.ids[tid];
      if (P.tr.expert_w) P.tr.expert_w[tid] = M.w[tid];
    }
    if (P.tr.union_count)
#pragma unroll 1
      for (int i = tid; i < E; i += kFT) {
        int c = 0;
        for (int j = 0; j < K; ++j) c = (M.ids[j] == i) ? P.k : c;
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
    for (int i = tid; i < 1024; i += kFT) reinterpret_cast<uint4*>(hist4096)[i] = make_uint4(0u, 0u, 0u, 0u);
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
#pragma unroll 1
  for (int lr = tid; lr < nrows; lr += kFT) {
    float sc = 0.f;
#pragma unroll
    for (int w = 1; w < kFW; ++w) sc += part[w * P.tpc * kRowTile + lr];
    sc = alpha_s[lr] * fabsf(sc + part[lr]) * 0.5f;
    part[lr] = sc;
    if (half == 0 && P.tr.scores) P.tr.scores[(size_t)rc * ipad + lt0 * kRowTile + lr] = sc;
  }
  __syncthreads();
  // ... then broadcast to every CTA of the cluster: item i -> (row i / CS, CTA i % CS)
  const int lg = CS == 16 ? 4 : 3;
#pragma unroll 1
  for (int i = tid; i < nrows * CS; i += kFT)
    cluster.map_shared_rank(keys, i & (CS - 1))[lt0 * kRowTile + (i >> lg)] =
        __float_as_uint(part[i >> lg]);
  cluster.sync();
  pdl_trigger();  // the next launch may start its weight-only prologue

  // ------------------------------------------------------------------ phase C: top-k, records
  if (!P.dense) select_channels(keys, I, P.k, sel, hist4096, M);
  if (!P.dense && half == 0 && q == 0) {
    if (P.tr.sel)
#pragma unroll 1
      for (int i = tid; i < P.k; i += kFT) P.tr.sel[(size_t)rc * P.k + i] = sel[i];
    if (tid == 0 && P.tr.sel_count) P.tr.sel_count[rc] = P.k;
  }
  // this CTA's share of the k channels
  const int NQ = CS * P.cpe, gq = half * CS + q;
  const int c0 = (int)((long)gq * P.k / NQ), c1 = (int)((long)(gq + 1) * P.k / NQ);
  const int nmine = c1 - c0;
  const uint32_t rec_bytes = 6u * d;
  uint16_t* ring = reinterpret_cast<uint16_t*>(big);
  if (tid == 0 && ok) {
    fence_proxy_async();
    const int first = min(P.ring, nmine);
#pragma unroll 1
    for (int i = 0; i < first; ++i) {
      const int ch = P.dense ? c0 + i : (int)sel[c0 + i];
      mbar_arrive_expect_tx(&M.bar[2 + i], rec_bytes);
      bulk_g2s(ring + (size_t)i * 3 * d, P.records + ((size_t)e * I + ch) * 3 * d, rec_bytes,
               &M.bar[2 + i]);
    }
  }
  float y[IT][8];
#pragma unroll
  for (int it = 0; it < IT; ++it)
#pragma unroll
    for (int i = 0; i < 8; ++i) y[it][i] = 0.f;
#pragma unroll 1
  for (int g0 = 0; g0 < nmine; g0 += P.group) {
    const int ng = min(P.group, nmine - g0);
    // warp w computes h of channel g0 + w once its record has landed
    if (warp < ng) {
      const int ci = g0 + warp;
      const bool okw = ok && wait_phase(&M.bar[2 + ci % P.ring], (ci / P.ring) & 1u, P.err);
      float hv = 0.f;
      if (okw) hv = channel_h(ring + (size_t)(ci % P.ring) * 3 * d, xs, d);
      if (lane == 0) M.h[warp] = hv;
      if (!okw && lane == 0) M.h[warp] = 0.f;
    }
    ok = __syncthreads_and(ok);
    if (ok) {
      // y += h_i * down_i over this thread's elements
#pragma unroll 1
      for (int i = 0; i < ng; ++i) {
        const uint16_t* rec = ring + (size_t)((g0 + i) % P.ring) * 3 * d + 2 * d;
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
    if (tid == 0 && ok) {
      fence_proxy_async();
#pragma unroll 1
      for (int i = g0; i < g0 + ng; ++i) {
        const int nx = i + P.ring;
        if (nx < nmine) {
          const int ch = P.dense ? c0 + nx : (int)sel[c0 + nx];
          const int slot = nx % P.ring;
          mbar_arrive_expect_tx(&M.bar[2 + slot], rec_bytes);
          bulk_g2s(ring + (size_t)slot * 3 * d, P.records + ((size_t)e * I + ch) * 3 * d, rec_bytes,
                   &M.bar[2 + slot]);
        }
      }
    }
  }

  // A_e z on this CTA's output slice
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
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
      for (int src = 0; src < CS; ++src) {
        const float4 v = *reinterpret_cast<const float4*>(cluster.map_shared_rank(ybuf, src) + el);
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
      }
      if (lr_out) {
        acc.x += ylr[4 * j]; acc.y += ylr[4 * j + 1]; acc.z += ylr[4 * j + 2]; acc.w += ylr[4 * j + 3];
      }
      red_add_v4(P.y_acc + el, we * acc.x, we * acc.y, we * acc.z, we * acc.w);
    }
  }
  cluster.sync();  // no CTA leaves while its buffer may still be read
  __threadfence();
  __syncthreads();
  if (tid == 0) M.last = (atomicAdd(P.slice_cnt + q, 1u) == (uint32_t)(K * P.cpe - 1));
  __syncthreads();
  if (M.last) {
    // every contribution to this slice has arrived: convert, re-zero, reset
    __threadfence();
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
  P.o_x = o;      o = align_up(o + 2 * d, 128);
  P.o_z = o;      o = align_up(o + 4 * (r > 0 ? r : 1), 128);
  P.o_sel = o;    o = align_up(o + 2 * ipad, 128);
  P.o_ylr = o;    o = align_up(o + 4 * P.slice, 128);
  P.o_misc = o;   o = align_up(o + (int)sizeof(Misc), 128);
  P.o_big = o;
  // offsets inside big (see the kernel): phase A and phase B scratch
  const int need_rows = align_up(P.rpc * 2 * d, 128);
  P.o_logits = need_rows;
  const int need_a = need_rows + align_up(4 * E, 128);
  int b = (P.dense ? 0 : P.tpc * (d / kColChunk) * kChunkWords * 4) + P.zpc * 2 * d;
  b = align_up(b, 128);
  P.o_alpha = b;  b = align_up(b + 4 * P.tpc * kRowTile, 128);
  P.o_part = b;   b = align_up(b + 4 * kFW * P.tpc * kRowTile, 128);
  P.o_xperm = b;  b = align_up(b + 2 * d, 128);
  P.o_keys = b;   b = align_up(b + 4 * ipad, 128);
  P.o_hist = b;   b = align_up(b + (P.dense ? 0 : 4 * 4096), 128);
  const int need_b = b;
  const int need_d = 4 * d;
  P.aslice_regs = (r > 0 && r % 8 == 0 && P.slice * r / 8 <= kAregs * kFT) ? 1 : 0;
  const int aslice_bytes = P.aslice_regs ? 0 : align_up(P.slice * r * 2, 128);
  const int avail = limit - o - aslice_bytes;
  const int rec = 6 * d;
  int ring = avail / rec;
  if (ring > kRingMax) ring = kRingMax;
  if (ring < 2 || need_a > avail || need_b > avail || need_d > avail) return false;
  const int per_cta = (k + cs * cpe - 1) / (cs * cpe);  // channels a CTA reads
  if (ring > per_cta) ring = per_cta < 2 ? 2 : per_cta;
  P.ring = ring;
  P.group = ring < kFW ? ring : kFW;  // one warp per channel of a group
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
