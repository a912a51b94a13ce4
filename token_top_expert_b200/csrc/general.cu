// Multi-kernel sparse-MoE block path, any batch size 1..256 (the default for batches past
// the single launch's crossover), every kernel launched with programmatic stream
// serialization:
//
//   router_kernel   logits (each router and x row read once per CTA), softmax, top-K,
//                   grouping of (token, expert) pairs by expert
//   score_kernel    ternary-sketch channel scores on the tensor cores; z = B_e x on CTAs
//                   of their own in the same grid
//   select_kernel   exact top-k (or threshold) per pair, per-expert union bitmap
//   union_kernel    per-expert union lists, runs of at most 64 channels as work items
//   gather_kernel   persistent: gathered channel records -> SwiGLU -> down on the tensor
//                   cores, outputs held in registers over a run; then A_e z on the tensor
//                   cores from bulk-copied rows of A_e; router-weighted reduction into an
//                   FP32 accumulator
//   finalize_kernel FP32 accumulator -> BF16 output (and re-zeroing)
//
// Each step follows the block definition of "KAIST drops calibration from MoE
// decoding ..." ("Top-k instead of a threshold", "A reader built from weights
// alone"); the batch path reads the union of the tokens' selected channels of
// each expert once.
#include "block_scan.cuh"
#include "common.cuh"
#include "launch.h"

namespace msb {

constexpr int kNT = 256;          // threads per CTA in every general kernel
constexpr int kRouterTok = 8;     // tokens per router CTA
constexpr int kRouterExp = 8;     // experts per router CTA
constexpr int kScoreRows = 64;    // sketch rows per score CTA (4 tensor-core row tiles)
constexpr int kScoreTok = 8;      // tokens per MMA n-tile
constexpr int kLrPass = 4;        // low-rank work item: passes of kNT / qs rows of A_e
static_assert(MSB_MAX_RANK % 8 == 0 && (MSB_MAX_RANK & (MSB_MAX_RANK - 1)) == 0,
              "the low-rank z stride 8 qs must fit 8 * MSB_MAX_RANK floats per token group");
constexpr int kGCh = 8;           // gather: channels per stage at most (one m-tile of gate/up rows)
constexpr int kGBufs = 2;         // gather: stage buffers (kGBufs - 1 stages in flight)
constexpr int kGRunCh = 64;       // gather: channels per work item at most (a multiple of stages)
static_assert(kGCh <= kNT / 32, "gather: one warp issues each channel of a stage");

// Sums of v[0..N) over the warp, transposed: afterwards lane l holds in v[0 .. N/32) the
// totals of the values N/32 l .. N/32 l + N/32 - 1 (N a power of two, N >= 32).  Each round
// halves the values a lane keeps: the lane whose bit o is set keeps the upper half and adds
// its partner's copy of it.
template <int N>
__device__ __forceinline__ void warp_sum_transposed(float (&v)[N], int lane) {
  static_assert(N >= 32 && (N & (N - 1)) == 0, "N: a power of two, at least 32");
#pragma unroll
  for (int s = 0; s < 5; ++s) {
    const int o = 16 >> s, half = N >> (s + 1);
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = up ? v[i] : v[i + half];
      const float keep = up ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
}

// Every kernel of this path is launched with programmatic stream serialization and begins
// here: wait until the kernels before it on the stream have completed and their writes are
// visible, then let the next kernel be scheduled while this one runs (it waits in turn).
__device__ __forceinline__ void pdl_begin() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// =====================================================================================
// router
// =====================================================================================
__global__ void __launch_bounds__(kNT) router_kernel(const uint16_t* __restrict__ x, int B,
                                                     const uint16_t* __restrict__ router_t, Dims D,
                                                     Workspace ws, TraceDev tr) {
  pdl_begin();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = D.d, E = D.experts, K = D.top_e;
  const int t0 = blockIdx.y * kRouterTok;
  const int nt = min(kRouterTok, B - t0);

  // zero this CTA's share of the output accumulator (rows t0.., a column slice)
  {
    const int cols = (d + gridDim.x - 1) / gridDim.x;
    const int c0 = blockIdx.x * cols, c1 = min(d, c0 + cols);
    for (int t = 0; t < nt; ++t)
      for (int c = c0 + threadIdx.x; c < c1; c += kNT) ws.y_acc[(size_t)(t0 + t) * d + c] = 0.f;
  }

  // logits of this CTA's 8 experts for its tokens: thread i takes the 16-byte groups
  // i, i + kNT, ... of d for every (expert, token), so that each row of the router and of
  // x is read once; the 64 partial sums meet across the warp (transposed) and the warps
  {
    const int e0 = blockIdx.x * kRouterExp;
    float acc[kRouterExp * kRouterTok];
#pragma unroll
    for (int i = 0; i < kRouterExp * kRouterTok; ++i) acc[i] = 0.f;
    for (int v = threadIdx.x; v < d / 8; v += kNT) {
      uint4 wv[kRouterExp], xv[kRouterTok];
#pragma unroll
      for (int i = 0; i < kRouterExp; ++i)
        wv[i] = e0 + i < E ? __ldg(reinterpret_cast<const uint4*>(router_t + (size_t)(e0 + i) * d) + v)
                           : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int t = 0; t < kRouterTok; ++t)
        xv[t] = t < nt ? __ldg(reinterpret_cast<const uint4*>(x + (size_t)(t0 + t) * d) + v)
                       : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int i = 0; i < kRouterExp; ++i)
#pragma unroll
        for (int t = 0; t < kRouterTok; ++t) acc[i * kRouterTok + t] = dot8(wv[i], xv[t], acc[i * kRouterTok + t]);
    }
    warp_sum_transposed(acc, lane);  // lane l: totals of (expert, token) 2l and 2l + 1
    __shared__ float2 s_part[kNT / 32][32];
    s_part[warp][lane] = make_float2(acc[0], acc[1]);
    __syncthreads();
    if (threadIdx.x < kRouterExp * kRouterTok) {
      const int q = threadIdx.x, i = q / kRouterTok, t = q % kRouterTok;
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kNT / 32; ++w) {
        const float2 pp = s_part[w][q >> 1];
        sum += (q & 1) ? pp.y : pp.x;
      }
      if (e0 + i < E && t < nt) ws.logits[(size_t)(t0 + t) * E + e0 + i] = sum;
    }
  }

  // ---- last CTA of this token group: softmax + top-K
  __shared__ int s_last;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t old = atomicAdd(&ws.counters[kCntRouterGroup + blockIdx.y], 1u);
    s_last = (old == gridDim.x - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (warp < nt) {
    const int t = t0 + warp;
    constexpr int MAXM = MSB_MAX_EXPERTS / 32;
    float v[MAXM];
    float mx = -INFINITY;
    bool bad = false;
#pragma unroll
    for (int m = 0; m < MAXM; ++m) {
      const int ee = lane + 32 * m;
      v[m] = ee < E ? __ldcg(&ws.logits[(size_t)t * E + ee]) : -INFINITY;
      bad = bad || (ee < E && !isfinite(v[m]));
      mx = fmaxf(mx, v[m]);
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(ws.err, kErrNonFinite);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
#pragma unroll
    for (int m = 0; m < MAXM; ++m)
      if (lane + 32 * m < E) sum += expf(v[m] - mx);
    sum = warp_sum(sum);
    uint32_t taken = 0;
    float pk[MSB_MAX_TOP_E];
    int ik[MSB_MAX_TOP_E];
    float psum = 0.f;
    for (int r = 0; r < K; ++r) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int m = 0; m < MAXM; ++m) {
        const int ee = lane + 32 * m;
        if (ee < E && !((taken >> m) & 1u) && (v[m] > bv || (v[m] == bv && ee < bi))) {
          bv = v[m];
          bi = ee;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
      }
      if (bi >= E) {  // non-finite logits: keep a valid index and flag the call
        bi = r;
        bv = mx;
        if (lane == 0) atomicOr(ws.err, kErrNonFinite);
      }
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
      pk[r] = expf(bv - mx);
      ik[r] = bi;
      psum += pk[r];
    }
    if (lane == 0) {
      const float denom = D.renorm ? psum : sum;
      for (int r = 0; r < K; ++r) {
        const float w = pk[r] / denom;
        ws.ids[t * K + r] = ik[r];
        ws.wts[t * K + r] = w;
        if (tr.expert_ids) tr.expert_ids[t * K + r] = ik[r];
        if (tr.expert_w) tr.expert_w[t * K + r] = w;
      }
    }
  }
  if (threadIdx.x == 0) ws.counters[kCntRouterGroup + blockIdx.y] = 0;

  // ---- last token group overall: group the (token, expert) pairs by expert
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t old = atomicAdd(&ws.counters[kCntRouterAll], 1u);
    s_last = (old == gridDim.y - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  __shared__ uint32_t cnt[MSB_MAX_EXPERTS];
  __shared__ uint32_t tokmask[MSB_MAX_EXPERTS][MSB_MAX_BATCH / 32];
  __shared__ uint32_t offs[MSB_MAX_EXPERTS];
  __shared__ uint32_t slot[MSB_MAX_EXPERTS];
  __shared__ uint32_t scan_tmp[kNT / 32 + 1];
  const int nwords = (B + 31) / 32;
  for (int i = threadIdx.x; i < E; i += kNT) {
    cnt[i] = 0;
    for (int w = 0; w < nwords; ++w) tokmask[i][w] = 0;
  }
  __syncthreads();
  const int P = B * K;
  for (int p = threadIdx.x; p < P; p += kNT) {
    const int t = p / K;
    const int ee = __ldcg(&ws.ids[p]);
    atomicAdd(&cnt[ee], 1u);
    atomicOr(&tokmask[ee][t >> 5], 1u << (t & 31));
  }
  __syncthreads();
  // exclusive scans of counts and of "used" flags over experts (2 experts per thread)
  {
    const int e0 = 2 * threadIdx.x, e1 = e0 + 1;
    const uint32_t c0 = e0 < E ? cnt[e0] : 0, c1 = e1 < E ? cnt[e1] : 0;
    uint32_t tot;
    const uint32_t pc = block_excl_scan<kNT>(c0 + c1, scan_tmp, &tot);
    const uint32_t u0 = c0 > 0, u1 = c1 > 0;
    uint32_t nu;
    const uint32_t pu = block_excl_scan<kNT>(u0 + u1, scan_tmp, &nu);
    if (e0 < E) { offs[e0] = pc; slot[e0] = pu; }
    if (e1 < E) { offs[e1] = pc + c0; slot[e1] = pu + u0; }
    if (e0 < E && c0) { ws.slot_expert[pu] = e0; ws.slot_off[pu] = pc; }
    if (e1 < E && c1) { ws.slot_expert[pu + u0] = e1; ws.slot_off[pu + u0] = pc + c0; }
    if (threadIdx.x == 0) { ws.slot_off[nu] = (int)tot; *ws.nused = (int)nu; }
  }
  __syncthreads();
  for (int p = threadIdx.x; p < P; p += kNT) {
    const int t = p / K;
    const int ee = __ldcg(&ws.ids[p]);
    uint32_t rank = 0;
    for (int w = 0; w < (t >> 5); ++w) rank += __popc(tokmask[ee][w]);
    rank += __popc(tokmask[ee][t >> 5] & ((1u << (t & 31)) - 1u));
    const int pos = (int)(offs[ee] + rank);
    ws.pair_tok[pos] = t;
    ws.pair_w[pos] = __ldcg(&ws.wts[p]);
    ws.pair_slot[pos] = (int)slot[ee];
    ws.pair_of[p] = pos;
  }
  // clear the union bitmaps of every slot
  const int uw = mask_words(D.ipad);
  for (int i = threadIdx.x; i < E * uw; i += kNT) ws.umask[i] = 0u;
  if (threadIdx.x == 0) ws.counters[kCntRouterAll] = 0;
}

// =====================================================================================
// sketch scores (tensor cores) and z = B_e x
// =====================================================================================
// One 64-column chunk of a 16-row tile: the codes pair w (2 bits per weight, placed at
// the sign and exponent bits of a BF16 +-2 or 0) x the staged x fragments, into sum.
__device__ __forceinline__ void score_chunk(uint2 w, const uint32_t* xp, float (&sum)[4]) {
  const uint4 xa = *reinterpret_cast<const uint4*>(xp);
  const uint4 xb = *reinterpret_cast<const uint4*>(xp + 4);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  mma_bf16(acc, w.x & kSketchMask, w.y & kSketchMask, (w.x << 2) & kSketchMask,
           (w.y << 2) & kSketchMask, xa.x, xa.y);
  mma_bf16(acc, (w.x << 4) & kSketchMask, (w.y << 4) & kSketchMask, (w.x << 6) & kSketchMask,
           (w.y << 6) & kSketchMask, xa.z, xa.w);
  mma_bf16(acc, (w.x << 8) & kSketchMask, (w.y << 8) & kSketchMask, (w.x << 10) & kSketchMask,
           (w.y << 10) & kSketchMask, xb.x, xb.y);
  mma_bf16(acc, (w.x << 12) & kSketchMask, (w.y << 12) & kSketchMask,
           (w.x << 14) & kSketchMask, (w.y << 14) & kSketchMask, xb.z, xb.w);
  sum[0] += acc[0];
  sum[1] += acc[1];
  sum[2] += acc[2];
  sum[3] += acc[3];
}

// Dynamic shared memory: xperm [kScoreTok][KC*32 + 4] uint32, then part [4][64] floats.
// xperm holds, per token n, chunk kc and lane column c, the eight bf16 pairs
// (s, p) = B-fragment registers of the four 16-column steps of that chunk.
__global__ void __launch_bounds__(kNT, 3) score_kernel(const uint16_t* __restrict__ x,
                                                    const uint32_t* __restrict__ sketch,
                                                    const float* __restrict__ alpha,
                                                    const uint16_t* __restrict__ lr_b, Dims D,
                                                    Workspace ws, TraceDev tr, int nsb) {
  pdl_begin();
  extern __shared__ __align__(16) uint32_t smem[];
  const int u = blockIdx.y;
  if (u >= *ws.nused) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int d = D.d, KC = d / kColChunk, ipad = D.ipad;
  const int e = ws.slot_expert[u];
  const int off = ws.slot_off[u], cnt = ws.slot_off[u + 1] - off;
  const int xstride = KC * 32 + 4;
  uint32_t* xperm = smem;
  float* part = reinterpret_cast<float*>(smem + kScoreTok * xstride);

  // ---- CTAs nsb.. of a slot: z = B_e x, one row of B_e per warp, 4 tokens at a time (they
  // run beside the score CTAs instead of ahead of them)
  if ((int)blockIdx.x >= nsb) {
    const int rho = ((int)blockIdx.x - nsb) * (kNT / 32) + warp;
    if (rho >= D.rank) return;
    const uint4* brow = reinterpret_cast<const uint4*>(lr_b + ((size_t)e * D.rank + rho) * d);
    for (int tq = 0; tq < cnt; tq += 4) {
      const int n = min(4, cnt - tq);
      const uint4* xr[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        xr[j] = reinterpret_cast<const uint4*>(x + (size_t)ws.pair_tok[off + tq + min(j, n - 1)] * d);
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
      for (int i = lane; i < d / 8; i += 32) {
        const uint4 bv = __ldg(brow + i);
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[j] = dot8(bv, __ldg(xr[j] + i), acc[j]);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float v = warp_sum(acc[j]);
        if (lane == 0 && j < n) ws.z[(size_t)(off + tq + j) * D.rank + rho] = v;
      }
    }
    return;
  }

  const int tile0 = blockIdx.x * (kScoreRows / kRowTile);
  const int ntiles = min(kScoreRows / kRowTile, ipad / kRowTile - tile0);
  if (ntiles <= 0) return;
  const int rt = warp & 3, kh = warp >> 2;
  const int kc0 = kh ? KC / 2 : 0, kc1 = kh ? KC : KC / 2;
  const uint2* codes =
      reinterpret_cast<const uint2*>(sketch) + ((size_t)(e * (ipad / kRowTile) + tile0 + rt) * KC) * 32 + lane;

  // this warp's codes (chunks kc0 .. kc1 of its tile, contiguous) are brought into L2 and
  // its rows' alpha loaded before x is staged, so that the latencies overlap
  if (rt < ntiles && lane == 0)
    prefetch_l2(codes - lane + (size_t)kc0 * 32, (uint32_t)(kc1 - kc0) * 32u * 8u);
  float al[2] = {0.f, 0.f};
  if (kh == 0 && rt < ntiles) {
    const int row0 = (tile0 + rt) * kRowTile + g;
    al[0] = __ldg(alpha + (size_t)e * ipad + row0);
    al[1] = __ldg(alpha + (size_t)e * ipad + row0 + 8);
  }

  __shared__ int s_tk[kScoreTok];
  for (int tt = 0; tt < cnt; tt += kScoreTok) {
    const int ntok = min(kScoreTok, cnt - tt);
    __syncthreads();
    if (threadIdx.x < kScoreTok)
      s_tk[threadIdx.x] = threadIdx.x < ntok ? ws.pair_tok[off + tt + threadIdx.x] : -1;
    __syncthreads();
    // build xperm for tokens pair_tok[off + tt + n]: the 16-byte group v of a row holds
    // columns 8v .. 8v+7 = the pairs cc = 0..3 of (chunk v / 8, step (v / 2) % 4, half v % 2)
#pragma unroll
    for (int n = 0; n < kScoreTok; ++n) {
      const int t = s_tk[n];
      for (int v = threadIdx.x; v < d / 8; v += kNT) {
        uint4 q = make_uint4(0u, 0u, 0u, 0u);
        if (t >= 0) q = __ldg(reinterpret_cast<const uint4*>(x + (size_t)t * d) + v);
        uint32_t* dst = xperm + n * xstride + (v >> 3) * 32 + ((v >> 1) & 3) * 2 + (v & 1);
        dst[0] = q.x;
        dst[8] = q.y;
        dst[16] = q.z;
        dst[24] = q.w;
      }
    }
    __syncthreads();
    float sum[4] = {0.f, 0.f, 0.f, 0.f};
    if (rt < ntiles) {
      const uint32_t* xp = xperm + g * xstride + c * 8;
#pragma unroll 8
      for (int kc = kc0; kc < kc1; ++kc) score_chunk(__ldg(codes + (size_t)kc * 32), xp + kc * 32, sum);
    }
    // combine the two k-halves: kh == 1 writes, kh == 0 adds
    if (kh == 1 && rt < ntiles) {
#pragma unroll
      for (int i = 0; i < 4; ++i) part[(rt * 32 + lane) * 4 + i] = sum[i];
    }
    __syncthreads();
    if (kh == 0 && rt < ntiles) {
#pragma unroll
      for (int i = 0; i < 4; ++i) sum[i] += part[(rt * 32 + lane) * 4 + i];
      const int row0 = (tile0 + rt) * kRowTile + g;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int n = 2 * c + (i & 1);
        const int row = row0 + (i >> 1) * 8;
        if (n < ntok) {
          const int p = off + tt + n;
          const float s = al[i >> 1] * fabsf(sum[i]) * 0.5f;
          ws.scores[(size_t)p * ipad + row] = s;
          if (tr.scores) {
            const int t = ws.pair_tok[p];
            int r = 0;
            while (ws.ids[t * D.top_e + r] != e) ++r;
            tr.scores[((size_t)t * D.top_e + r) * ipad + row] = s;
          }
        }
      }
    }
  }
}

// =====================================================================================
// exact top-k / threshold selection per (token, expert) pair
// =====================================================================================
__global__ void __launch_bounds__(kNT) select_kernel(int k, int mode, float tau, Dims D,
                                                     Workspace ws, TraceDev tr) {
  pdl_begin();
  __shared__ uint32_t keys[MSB_MAX_INTER];
  __shared__ uint16_t sel_s[MSB_MAX_INTER];
  __shared__ uint32_t words[MSB_MAX_INTER / 32];
  __shared__ uint32_t hist4096[4096];
  __shared__ uint32_t sscr[208];
  __shared__ uint32_t scan_tmp[kNT / 32 + 1];
  __shared__ uint32_t s_count;
  const int p = blockIdx.x;
  const int I = D.inter, ipad = D.ipad, mw = mask_words(ipad);
  for (int j = threadIdx.x; j < I; j += kNT)
    keys[j] = __float_as_uint(__ldcg(&ws.scores[(size_t)p * ipad + j]));
  for (int i = threadIdx.x; i < mw; i += kNT) words[i] = 0;
  for (int i = threadIdx.x; i < 4096; i += kNT) hist4096[i] = 0;
  __syncthreads();
  if (mode == 0) {
    uint32_t kth, need;
    hist_kth_smem<kNT>(keys, I, k, hist4096, sscr, &kth, &need);
    scatter_topk<kNT>(keys, I, kth, need, sel_s, scan_tmp);
    if (threadIdx.x == 0) s_count = (uint32_t)k;
  } else {
    const int ept = (I + kNT - 1) / kNT;
    const int j0 = threadIdx.x * ept, j1 = min(I, j0 + ept);
    uint32_t n = 0;
    for (int j = j0; j < j1; ++j) n += __uint_as_float(keys[j]) > tau;
    uint32_t tot;
    uint32_t pos = block_excl_scan<kNT>(n, scan_tmp, &tot);
    for (int j = j0; j < j1; ++j)
      if (__uint_as_float(keys[j]) > tau) sel_s[pos++] = (uint16_t)j;
    if (threadIdx.x == 0) s_count = tot;
  }
  __syncthreads();
  const int count = (int)s_count;
  const int t = ws.pair_tok[p];
  const int slot = ws.pair_slot[p];
  const int e = ws.slot_expert[slot];
  int r = 0;
  while (ws.ids[t * D.top_e + r] != e) ++r;
  const size_t trow = (size_t)t * D.top_e + r;
  const int cap = mode == 0 ? k : I;
  for (int i = threadIdx.x; i < count; i += kNT) {
    const int j = sel_s[i];
    ws.sel[(size_t)p * ipad + i] = (uint16_t)j;
    if (tr.sel) tr.sel[trow * cap + i] = (uint16_t)j;
    atomicOr(&words[j >> 5], 1u << (j & 31));
  }
  __syncthreads();
  for (int i = threadIdx.x; i < mw; i += kNT) {
    const uint32_t wv = words[i];
    ws.selmask[(size_t)p * mw + i] = wv;
    if (wv) atomicOr(&ws.umask[(size_t)slot * mw + i], wv);
  }
  if (threadIdx.x == 0) {
    ws.selcnt[p] = count;
    if (tr.sel_count) tr.sel_count[trow] = count;
  }
}

// =====================================================================================
// union lists: the ascending list of each slot's union bitmap, and the prefix of the
// slots' channel chunks (the gather kernel's work items)
// =====================================================================================
__global__ void __launch_bounds__(kNT) union_kernel(Dims D, Workspace ws, int ch, int ngrid, int dense) {
  pdl_begin();
  __shared__ uint32_t s_tmp[kNT / 32 + 1];
  __shared__ int s_last;
  const int tid = threadIdx.x;
  const int u = blockIdx.x, nu = *ws.nused;
  if (u < nu) {
    int n = D.inter;
    if (!dense) {
      const int nw = mask_words(D.ipad);  // <= 128 words, one per thread
      const uint32_t w = tid < nw ? __ldcg(&ws.umask[(size_t)u * nw + tid]) : 0u;
      uint32_t tot;
      uint32_t rank = block_excl_scan<kNT>((uint32_t)__popc(w), s_tmp, &tot);
      uint16_t* dst = ws.ulist + (size_t)u * D.ipad;
      for (uint32_t b = w; b; b &= b - 1) dst[rank++] = (uint16_t)(tid * 32 + __ffs(b) - 1);
      n = (int)tot;
    }
    if (tid == 0) ws.ucnt[u] = n;
  }
  // the last CTA: chunk prefix over the used slots, and a fresh work counter
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    s_last = atomicAdd(&ws.counters[kCntUnion], 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // run length: a multiple of the stage size ch, about two runs per CTA of the grid,
  // at most kGRunCh channels (longer runs mean fewer reduction-adds per output and less
  // per-item overhead, shorter ones a more even finish)
  uint32_t n2[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 2; ++i)
    if (2 * tid + i < nu) n2[i] = (uint32_t)__ldcg(&ws.ucnt[2 * tid + i]);
  uint32_t all;
  block_excl_scan<kNT>(n2[0] + n2[1], s_tmp, &all);
  int run = (int)((all + 2u * ngrid - 1) / (2u * ngrid));
  run = min(kGRunCh / ch * ch, max(ch, (run + ch - 1) / ch * ch));
  uint32_t c[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 2; ++i) c[i] = (n2[i] + run - 1) / run;
  uint32_t tot;
  const uint32_t pre = block_excl_scan<kNT>(c[0] + c[1], s_tmp, &tot);
  if (2 * tid < nu) ws.coff[2 * tid] = (int)pre;
  if (2 * tid + 1 < nu) ws.coff[2 * tid + 1] = (int)(pre + c[0]);
  if (tid == 0) {
    ws.coff[nu] = (int)tot;
    ws.counters[kCntGatherRun] = (uint32_t)run;
    ws.counters[kCntGatherWork] = 0u;
    ws.counters[kCntUnion] = 0u;
  }
}

// =====================================================================================
// gathered channel records -> SwiGLU -> down; low-rank A_e z; weighted reduction
// =====================================================================================
// Persistent CTAs (one per SM) take work items off a counter: first runs of at most
// kGRunCh channels of one expert's union list, then low-rank row blocks.  A run streams
// through stages of up to kGCh channels for every token routed to the expert, 8 tokens at
// a time, on the tensor cores:
//   gate/up   D[16 rows][8 tokens] = [gate rows | up rows] (ldmatrix from the records
//             in shared memory) x the tokens' x rows (B fragments in registers, or read
//             through L1); warp w takes k-steps [w KS/8, (w+1) KS/8) over four
//             accumulator chains, the warps' partials meet in shared memory;
//   h         silu(g) u, times the pair's selection bit and router weight;
//   down      D[16 columns][8 tokens] += the records' down columns (ldmatrix.trans) x
//             [h_hi ; h_lo]: h split into two bf16 halves laid along k against the same
//             8 channels repeated, so that one MMA keeps ~16 significant bits of h; the
//             run's outputs stay in registers (NACC > 0) and reach the FP32 accumulator
//             once per run, two adjacent columns per 8-byte reduction-add.
// Low-rank items: A_e z for a block of rows of A_e, on the tensor cores the same way
// (z's halves along k), from rows bulk-copied into a stage buffer while the previous item
// is computed.
// Dynamic shared memory: records [ch][3d + 8] bf16 (16 bytes of stagger per slot).
struct GatherCfg {
  int ch;       // channels per work item (<= kGCh)
  int nlr;      // low-rank work items per slot
  int lr_qs;    // low-rank: 8-element pieces per row of A_e, rounded up to a power of two
  int lr_vec;   // low-rank: rows are 16-byte aligned (r % 8 == 0)
  int lr_rows;  // low-rank: rows of A_e per item copied into a stage buffer (0: registers)
  int dense;    // 1: every channel is selected (no sketch)
  uint64_t wait_ns;  // bounded-wait limit
#ifdef MSB_INSTRUMENTED
  uint32_t skip;     // 2: the CTA of work item 0 never issues its first stage (test only)
#endif
};

__device__ __forceinline__ void red_add_v2(float* dst, float a, float b) {
  asm volatile("red.global.add.v2.f32 [%0], {%1,%2};" ::"l"(dst), "f"(a), "f"(b) : "memory");
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
         ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
}

// Reduction-add of one down tile D[16 columns][8 tokens] (columns m0 + row, the mma.sync
// accumulator layout) into the FP32 accumulator y[token][column].  Lanes g and g ^ 1 of a
// column pair swap one value so that each lane adds two adjacent columns of one token;
// `hi`: rows 8-15 are real columns too.
__device__ __forceinline__ void gather_red_tile(float* y, const int* s_tok, int ntg, int d, int m0,
                                                const float (&acc)[4], int lane, bool hi) {
  const int g8 = lane >> 2, c4 = lane & 3;
  const bool odd = g8 & 1;
  const int t = 2 * c4 + (odd ? 1 : 0);  // token of this lane's pair after the swap
  const int col = m0 + (g8 & ~1);
  const float s0 = __shfl_xor_sync(0xffffffffu, odd ? acc[0] : acc[1], 4);
  const float s1 = __shfl_xor_sync(0xffffffffu, odd ? acc[2] : acc[3], 4);
  if (t < ntg) {
    float* row = y + (size_t)s_tok[t] * d + col;
    red_add_v2(row, odd ? s0 : acc[0], odd ? acc[1] : s0);
    if (hi) red_add_v2(row + 8, odd ? s1 : acc[2], odd ? acc[3] : s1);
  }
}

// acc[t] = (8 bf16 of a row of A_e) . z[t][0..8) for the 8 tokens of a group, z at stride zs
__device__ __forceinline__ void gather_lr_dot(uint4 av, const float* z, int zs, float (&acc)[8]) {
  const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const float4 z0 = *reinterpret_cast<const float4*>(z + t * zs);
    const float4 z1 = *reinterpret_cast<const float4*>(z + t * zs + 4);
    const float zz[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      a = fmaf(__uint_as_float(aw[i] << 16), zz[2 * i], a);
      a = fmaf(__uint_as_float(aw[i] & 0xffff0000u), zz[2 * i + 1], a);
    }
    acc[t] = a;
  }
}

// B fragment of the low-rank MMA: z[t][i], z[t][i + 1] (FP32, times the router weight) as
// a BF16 pair (zhi) and the pair of what BF16 rounding left over (zlo)
__device__ __forceinline__ void lr_zfrag(const float* z, uint32_t& zhi, uint32_t& zlo) {
  const float2 v = *reinterpret_cast<const float2*>(z);
  zhi = pack_bf16x2(v.x, v.y);
  zlo = pack_bf16x2(v.x - __uint_as_float(zhi << 16), v.y - __uint_as_float(zhi & 0xffff0000u));
}

// Thread 0 copies rows [row0, row0 + nrow) of A_e (r bf16 each, r % 8 == 0) into `buf`.
__device__ __forceinline__ void gather_lr_issue(uint16_t* buf, const uint16_t* lr_a, int e, int row0,
                                                int nrow, int d, int r, uint64_t* bar) {
  const uint32_t bytes = (uint32_t)nrow * 2u * (uint32_t)r;
  fence_proxy_async();
  mbar_arrive_expect_tx(bar, bytes);
  bulk_g2s(buf, lr_a + ((size_t)e * d + row0) * r, bytes, bar);
}

// Every thread calls, after thread 0 has armed `bar` with the stage's bytes (gather_arm)
// and a barrier of the CTA has ordered that before this call: the channel list of
// run[c0 .. c0 + n) (shared memory) into `list` and (copy) the bulk copies of their
// records into a stage buffer, lane 0 of warp i taking channel i (n <= warps), so that no
// warp waits for all the issues.  The list is always written: the consumer reads it
// whether or not the copies were issued.
__device__ __forceinline__ void gather_issue(uint16_t* buf, const uint16_t* records, const int* run,
                                             int e, int c0, int n, int d, int I, int* list,
                                             uint64_t* bar, bool copy = true) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0 && warp < n) {
    const int j = run[c0 + warp];
    list[warp] = j;
    if (copy) {
      fence_proxy_async();  // the buffer's earlier reads (generic proxy) before the copy
      bulk_g2s(buf + (size_t)warp * (3 * d + 8), records + ((size_t)e * I + j) * 3 * d, 6u * d, bar);
    }
  }
}

// Thread 0: arrive on a stage barrier whose previous phase has completed, expecting the
// bytes of n records (the stage's copies are issued later by gather_issue).
__device__ __forceinline__ void gather_arm(uint64_t* bar, int n, int d) {
  mbar_arrive_expect_tx(bar, 6u * d * n);
}

// NACC > 0: d <= 128 NACC, each warp's outputs (NACC tiles of 16 columns) held in
// registers over a run; 0: reduction-adds after every stage.
// KSW: the x B-fragments of this warp's k-steps held in registers per token group
// (d <= 128 * KSW); 0: read through L1/L2 at every stage.
// Stages of cfg.ch channels stream through kGBufs buffers, kGBufs - 1 of them in flight
// while one is computed.
template <int NACC, int KSW>
__global__ void __launch_bounds__(kNT, 1) gather_kernel(const uint16_t* __restrict__ x,
                                                        const uint16_t* __restrict__ records,
                                                        const uint16_t* __restrict__ lr_a, Dims D,
                                                        Workspace ws, GatherCfg cfg) {
  pdl_begin();
  constexpr bool REGACC = NACC > 0;
  extern __shared__ __align__(128) uint8_t gsm[];
  __shared__ __align__(8) uint64_t bar[kGBufs];
  __shared__ int s_item, s_u;
  __shared__ int s_list[kGBufs][kGCh];
  __shared__ int s_run[kGRunCh];  // channel indices of the current run
  __shared__ int s_tok[8];
  __shared__ float s_w[8];
  __shared__ float s_red[kNT / 32][16][8];
  __shared__ __align__(16) float s_h[8][2 * kGCh];  // [token][channel], channels >= ch zero
  __shared__ __align__(16) float s_lz[8 * MSB_MAX_RANK];  // low-rank: [token][8 qs] z times weight
  __shared__ int s_ltok[8];
  __shared__ int s_lr_next[2];
  // slot tables, copied once: run offsets, union sizes, experts, pair offsets
  __shared__ int s_coff[MSB_MAX_EXPERTS + 1], s_ucnt[MSB_MAX_EXPERTS], s_se[MSB_MAX_EXPERTS],
      s_so[MSB_MAX_EXPERTS + 1];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int d = D.d, I = D.inter, ipad = D.ipad, r = D.rank;
  const int nu = *ws.nused;
  for (int i = tid; i <= nu; i += kNT) {
    s_coff[i] = __ldcg(&ws.coff[i]);
    s_so[i] = __ldcg(&ws.slot_off[i]);
    if (i < nu) {
      s_ucnt[i] = __ldcg(&ws.ucnt[i]);
      s_se[i] = __ldcg(&ws.slot_expert[i]);
    }
  }
  const int nchunks = __ldcg(&ws.coff[nu]);
  const int run = (int)__ldcg(&ws.counters[kCntGatherRun]);
  const int nitems = nchunks + nu * cfg.nlr;
  const int rs = 3 * d + 8;  // slot stride (elements)
  const int CH = cfg.ch;
  uint16_t* const buf0 = reinterpret_cast<uint16_t*>(gsm);
  const size_t bstride = (size_t)CH * rs;  // stage buffer b at buf0 + b * bstride
  if (tid == 0) {
#pragma unroll
    for (int b = 0; b < kGBufs; ++b) mbar_init(&bar[b], 1);
    fence_mbar_init();
  }
  for (int i = tid; i < 8 * 2 * kGCh; i += kNT) (&s_h[0][0])[i] = 0.f;
  uint32_t phases = 0;  // bit b: parity of buffer b's next completion
  const int c4 = lane & 3, g8 = lane >> 2;
  const int KS = d / 16;
  const int ks0 = warp * KS / (kNT / 32), ks1 = (warp + 1) * KS / (kNT / 32);
  // down columns of this warp: [c0w, c0w + d / 8), NT16 tiles of 16 and one of 8 if d / 64 is odd
  const int c0w = warp * (d / 8);
  const int NT16 = d / 128;
  const bool tail8 = (d / 64) & 1;
  const int nmw = mask_words(ipad);
  // h step ownership: thread tid < 8 * CH takes (token tid / CH, channel tid % CH)
  const int hc = tid % CH, ht = tid / CH;
  bool ok = true;
  // work items are claimed one ahead, so the counter's round trip overlaps an item
  int next_item = 0;
  if (tid == 0) next_item = (int)atomicAdd(&ws.counters[kCntGatherWork], 1u);

#pragma unroll 1
  for (;;) {
    __syncthreads();  // the previous item's reads of shared memory are done (and the tables)
    if (tid == 0) {
      const int it = next_item;
      if (it < nitems) next_item = (int)atomicAdd(&ws.counters[kCntGatherWork], 1u);
      int u = 0;
      if (it < nchunks) {  // slot of run `it`: last u with coff[u] <= it
        int lo = 0, hi = nu - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (s_coff[mid] <= it) lo = mid; else hi = mid - 1;
        }
        u = lo;
      }
      s_item = it;
      s_u = u;
    }
    __syncthreads();
    const int item = s_item;
    if (item >= nitems || !ok) break;

    // ----------------------------------------------------------- low-rank items, staged
    // Every later item is a low-rank item too, so the CTA stays here: thread 0 copies the
    // next item's rows of A_e (cfg.lr_rows rows of r bf16, contiguous) into the other stage
    // buffer while the current item is computed from shared memory.
    if (item >= nchunks && cfg.lr_rows > 0) {
      const int zs = 8 * cfg.lr_qs;  // z stride: r rounded up to 8 times a power of two
      const int R = cfg.lr_rows;
      const uint32_t rowb = 2u * (uint32_t)r;
      int cur = item, bsel = 0, par = 0;
      if (tid == 0) {
        const int q = cur - nchunks, u = q / cfg.nlr, row0 = (q - u * cfg.nlr) * R;
        gather_lr_issue(buf0, lr_a, s_se[u], row0, min(R, d - row0), d, r, &bar[0]);
      }
      for (;;) {
        if (tid == 0) {  // claim the item after next and start the next one's copy
          const int nx = next_item;
          if (nx < nitems) {
            next_item = (int)atomicAdd(&ws.counters[kCntGatherWork], 1u);
            const int q = nx - nchunks, u = q / cfg.nlr, row0 = (q - u * cfg.nlr) * R;
            gather_lr_issue(buf0 + (bsel ^ 1) * bstride, lr_a, s_se[u], row0, min(R, d - row0), d, r,
                            &bar[bsel ^ 1]);
          }
          s_lr_next[par] = nx;
        }
        const int q = cur - nchunks, u = q / cfg.nlr;
        const int off = s_so[u], cnt = s_so[u + 1] - off;
        const int row0 = (q - u * cfg.nlr) * R, nrow = min(R, d - row0);
        const uint8_t* abuf = reinterpret_cast<const uint8_t*>(buf0 + bsel * bstride);
        for (int tg = 0; tg < cnt; tg += 8) {
          const int ntg = min(8, cnt - tg);
          if (tg > 0) __syncthreads();  // the previous group's reads of s_lz
          for (int i = tid; i < 8 * zs; i += kNT) {
            const int t = i / zs, c = i - t * zs;
            float v = 0.f;
            if (t < ntg && c < r) v = __ldcg(ws.z + (size_t)(off + tg + t) * r + c) * ws.pair_w[off + tg + t];
            s_lz[i] = v;
          }
          if (tid < 8) s_ltok[tid] = tid < ntg ? ws.pair_tok[off + tg + tid] : 0;
          if (tg == 0) {  // the rows' copy, and s_lz / s_ltok / s_lr_next visible
            const bool okw = mbar_wait(&bar[bsel], (phases >> bsel) & 1u, ws.err, cfg.wait_ns);
            if (!__syncthreads_and(okw)) {  // sticky error set; let the copies in flight land
              mbar_wait(&bar[bsel], (phases >> bsel) & 1u, ws.err, cfg.wait_ns);
              if (s_lr_next[par] < nitems)
                mbar_wait(&bar[bsel ^ 1], (phases >> (bsel ^ 1)) & 1u, ws.err, cfg.wait_ns);
              ok = false;
              break;
            }
            phases ^= 1u << bsel;
          } else {
            __syncthreads();
          }
          // D[16 rows][8 tokens] += rows of A_e x [z_hi ; z_lo]: the two BF16 halves of z lie
          // along k against the same 8 values of r repeated, 8 values of r per MMA; a warp
          // takes every (kNT / 32)-th tile of 16 rows (nrow is a multiple of 16)
          for (int tl = warp; tl < nrow / 16; tl += kNT / 32) {
            const uint8_t* tb = abuf + (size_t)tl * 16 * rowb + (size_t)(lane & 15) * rowb;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            int rc = 0;
            for (; rc + 16 <= r; rc += 16) {  // lanes 16-31 address the next 8 values of r
              uint32_t a0, a1, a2, a3, z0, z1, z2, z3;
              ldsm_x4(smem_addr(tb + 2 * (rc + 8 * (lane >> 4))), a0, a1, a2, a3);
              lr_zfrag(s_lz + g8 * zs + rc + 2 * c4, z0, z1);
              lr_zfrag(s_lz + g8 * zs + rc + 8 + 2 * c4, z2, z3);
              mma_bf16(acc, a0, a1, a0, a1, z0, z1);
              mma_bf16(acc, a2, a3, a2, a3, z2, z3);
            }
            if (rc < r) {  // 8 values of r left
              uint32_t a0, a1, z0, z1;
              ldsm_x2(smem_addr(tb + 2 * rc), a0, a1);
              lr_zfrag(s_lz + g8 * zs + rc + 2 * c4, z0, z1);
              mma_bf16(acc, a0, a1, a0, a1, z0, z1);
            }
            gather_red_tile(ws.y_acc, s_ltok, ntg, d, row0 + 16 * tl, acc, lane, true);
          }
        }
        if (!ok) break;
        __syncthreads();  // buffer bsel and s_lz are free
        cur = s_lr_next[par];
        par ^= 1;
        bsel ^= 1;
        if (cur >= nitems) break;
      }
      break;
    }

    // ----------------------------------------------------------- low-rank item
    // (rows not 16-byte aligned) kLrPass passes of kNT / qs rows of A_e: thread (row, piece) holds 8 elements of the
    // row per pass (one 16-byte load when r % 8 == 0), all loads issued before the
    // tokens' z (times the router weight) are staged in shared memory 8 tokens at a time;
    // the row's pieces meet by shuffles and lane `piece` adds tokens piece, piece + qs, ...
    if (item >= nchunks) {
      const int q = item - nchunks, u = q / cfg.nlr;
      const int e = s_se[u];
      const int off = s_so[u], cnt = s_so[u + 1] - off;
      const int qs = cfg.lr_qs, zs = 8 * qs;  // pieces per row (a power of two), z stride
      const int rpp = kNT / qs;               // rows per pass
      const int lrow = tid / qs, piece = tid - lrow * qs;
      const int row0 = (q - u * cfg.nlr) * (kLrPass * rpp);
      uint4 av[kLrPass];
#pragma unroll
      for (int ps = 0; ps < kLrPass; ++ps) {
        const int row = row0 + ps * rpp + lrow;
        av[ps] = make_uint4(0u, 0u, 0u, 0u);
        if (row < d && piece * 8 < r) {
          const uint16_t* src = lr_a + ((size_t)e * d + row) * r + piece * 8;
          if (cfg.lr_vec) {
            av[ps] = __ldg(reinterpret_cast<const uint4*>(src));
          } else {
            uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int i = 0; i < 8; ++i)
              if (piece * 8 + i < r) w[i >> 1] |= (uint32_t)__ldg(src + i) << (16 * (i & 1));
            av[ps] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      for (int tg = 0; tg < cnt; tg += 8) {
        const int ntg = min(8, cnt - tg);
        if (tg > 0) __syncthreads();  // the previous group's reads of s_lz
        for (int i = tid; i < 8 * zs; i += kNT) {
          const int t = i / zs, c = i - t * zs;
          float v = 0.f;
          if (t < ntg && c < r) v = __ldcg(ws.z + (size_t)(off + tg + t) * r + c) * ws.pair_w[off + tg + t];
          s_lz[i] = v;
        }
        if (tid < 8) s_ltok[tid] = tid < ntg ? ws.pair_tok[off + tg + tid] : 0;
        __syncthreads();
#pragma unroll
        for (int ps = 0; ps < kLrPass; ++ps) {
          const int row = row0 + ps * rpp + lrow;
          float acc[8];
          gather_lr_dot(av[ps], s_lz + piece * 8, zs, acc);
          for (int o = 1; o < qs; o <<= 1)
#pragma unroll
            for (int t = 0; t < 8; ++t) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
          if (row < d)
#pragma unroll
            for (int t = 0; t < 8; ++t)
              if ((t & (qs - 1)) == piece && t < ntg) atomicAdd(&ws.y_acc[(size_t)s_ltok[t] * d + row], acc[t]);
        }
      }
      continue;
    }

    // ----------------------------------------------------------- a run of union channels
    const int u = s_u;
    const int e = s_se[u];
    const int off = s_so[u], cnt = s_so[u + 1] - off;
    const int rb = (item - s_coff[u]) * run;
    const int nrun = min(run, s_ucnt[u] - rb);
    const int nst = (nrun + CH - 1) / CH;
    for (int i = tid; i < nrun; i += kNT)
      s_run[i] = cfg.dense ? rb + i : (int)__ldcg(&ws.ulist[(size_t)u * ipad + rb + i]);

    for (int tg0 = 0; tg0 < cnt && ok; tg0 += 8) {  // (records are streamed again per 8 tokens)
      const int ntg = min(8, cnt - tg0);
      // every stage barrier's last phase has completed: thread 0 arms those of stages
      // 0 .. kGBufs - 1 (the fill's, and the one iteration 0 issues)
      if (tid == 0)
        for (int st = 0; st < min(kGBufs, nst); ++st) {
          bool copy = true;
#ifdef MSB_INSTRUMENTED
          copy = !(cfg.skip == 2u && item == 0 && tg0 == 0 && st == 0);  // withhold the stage
#endif
          if (copy) gather_arm(&bar[st], min(CH, nrun - st * CH), d);
        }
      __syncthreads();  // s_run; s_tok, s_w, s_h and every stage buffer are free
      if (tid < 8) {
        const int p = off + tg0 + min(tid, ntg - 1);
        s_tok[tid] = ws.pair_tok[p];
        s_w[tid] = tid < ntg ? ws.pair_w[p] : 0.f;
      }
      for (int st = 0; st < min(kGBufs - 1, nst); ++st) {  // fill: stages 0 .. kGBufs - 2
        bool copy = true;
#ifdef MSB_INSTRUMENTED
        copy = !(cfg.skip == 2u && item == 0 && tg0 == 0 && st == 0);  // withhold the stage
#endif
        gather_issue(buf0 + st * bstride, records, s_run, e, st * CH, min(CH, nrun - st * CH), d, I,
                     s_list[st], &bar[st], copy);
      }
      __syncthreads();  // s_tok, the fill's lists
      // B fragments (x of this lane's token g8) of this warp's k-steps
      uint32_t xb[KSW > 0 ? KSW : 1][2];
      const uint32_t* xrow = reinterpret_cast<const uint32_t*>(x + (size_t)s_tok[g8] * d);
#pragma unroll
      for (int i = 0; i < KSW; ++i)
        if (ks0 + i < ks1) {
          xb[i][0] = __ldg(xrow + (ks0 + i) * 8 + c4);
          xb[i][1] = __ldg(xrow + (ks0 + i) * 8 + 4 + c4);
        }
      float yacc[REGACC ? NACC : 1][4];
#pragma unroll
      for (int i = 0; i < (REGACC ? NACC : 1); ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) yacc[i][j] = 0.f;

#pragma unroll 1
      for (int stg = 0; stg < nst; ++stg) {
        const int b = stg % kGBufs;
        const int nch = min(CH, nrun - stg * CH);
        // keep kGBufs - 1 stages in flight: stage stg + kGBufs - 1 goes into the buffer
        // that stage stg - 1 has just released (its barrier armed before that release)
        if (stg + kGBufs - 1 < nst) {
          const int sn = stg + kGBufs - 1, bn = sn % kGBufs;
          gather_issue(buf0 + bn * bstride, records, s_run, e, sn * CH, min(CH, nrun - sn * CH), d, I,
                       s_list[bn], &bar[bn]);
        }
        const bool okw = mbar_wait(&bar[b], (phases >> b) & 1u, ws.err, cfg.wait_ns);
        if (!__syncthreads_and(okw)) {  // sticky error set; let copies in flight land
          for (int q = stg; q < min(nst, stg + kGBufs); ++q)
            mbar_wait(&bar[q % kGBufs], (phases >> (q % kGBufs)) & 1u, ws.err, cfg.wait_ns);
          ok = false;
          break;
        }
        phases ^= 1u << b;
        // selection bit of this thread's (token, channel), loaded here so that its latency
        // overlaps gate/up (the stage's list was written before the barrier above)
        uint32_t selw = 1u;
        if (!cfg.dense && tid < 8 * CH && ht < ntg && hc < nch) {
          const int j = s_list[b][hc];
          selw = __ldcg(&ws.selmask[(size_t)(off + tg0 + ht) * nmw + (j >> 5)]) >> (j & 31);
        }
        const uint16_t* rec = buf0 + b * bstride;
        // gate/up ldmatrix row: channel lane % 8 (channels past nch read channel 0;
        // their rows are dropped), gate (lanes 0-7, 16-23) or up, k offset 8 (lane / 16)
        const int gch = (lane & 7) < nch ? (lane & 7) : 0;
        uint32_t a_addr =
            smem_addr(rec + (size_t)gch * rs + ((lane >> 3) & 1) * d + 8 * (lane >> 4)) + 32u * ks0;
        // down ldmatrix.trans row: channel lane % 8 (channels past nch read channel 0;
        // their h is zero); lane / 8 picks the 8-column block
        const uint32_t b_base = smem_addr(rec + (size_t)gch * rs + 2 * d);
        // ---- gate/up partials over this warp's k-steps (four accumulator chains)
        {
          float acc[4][4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
          int ks = ks0;
          if (KSW > 0) {
#pragma unroll
            for (int i = 0; i < KSW; ++i)
              if (ks0 + i < ks1) {
                uint32_t a0, a1, a2, a3;
                ldsm_x4(a_addr + 32u * i, a0, a1, a2, a3);
                mma_bf16(acc[i & 3], a0, a1, a2, a3, xb[i][0], xb[i][1]);
              }
            ks = ks1;
          }
          for (; ks + 4 <= ks1; ks += 4, a_addr += 128u) {
            uint32_t a[4][4], bb[4][2];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              ldsm_x4(a_addr + 32u * i, a[i][0], a[i][1], a[i][2], a[i][3]);
              bb[i][0] = __ldg(xrow + (ks + i) * 8 + c4);
              bb[i][1] = __ldg(xrow + (ks + i) * 8 + 4 + c4);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) mma_bf16(acc[i], a[i][0], a[i][1], a[i][2], a[i][3], bb[i][0], bb[i][1]);
          }
          for (; ks < ks1; ++ks, a_addr += 32u) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(a_addr, a0, a1, a2, a3);
            mma_bf16(acc[0], a0, a1, a2, a3, __ldg(xrow + ks * 8 + c4), __ldg(xrow + ks * 8 + 4 + c4));
          }
          s_red[warp][g8][2 * c4] = (acc[0][0] + acc[1][0]) + (acc[2][0] + acc[3][0]);
          s_red[warp][g8][2 * c4 + 1] = (acc[0][1] + acc[1][1]) + (acc[2][1] + acc[3][1]);
          s_red[warp][g8 + 8][2 * c4] = (acc[0][2] + acc[1][2]) + (acc[2][2] + acc[3][2]);
          s_red[warp][g8 + 8][2 * c4 + 1] = (acc[0][3] + acc[1][3]) + (acc[2][3] + acc[3][3]);
        }
        __syncthreads();
        // ---- h[token][channel] = silu(g) u, times the selection bit and the router weight
        if (tid < 8 * CH) {
          float h = 0.f;
          if (hc < nch && ht < ntg && (selw & 1u)) {
            float g = 0.f, uu = 0.f;
#pragma unroll
            for (int w = 0; w < kNT / 32; ++w) { g += s_red[w][hc][ht]; uu += s_red[w][8 + hc][ht]; }
            h = silu(g) * uu * s_w[ht];
          }
          s_h[ht][hc] = h;
        }
        __syncthreads();
        // ---- down: D[16 columns][8 tokens] += A x B with A = this warp's down columns
        // (rows) over k = [channels 0-7 | channels 0-7 again] and B = [h_hi ; h_lo] of the
        // tokens, so that one MMA carries both halves of h
        const float2 hp = *reinterpret_cast<const float2*>(&s_h[g8][2 * c4]);
        const uint32_t hhi = pack_bf16x2(hp.x, hp.y);
        const float hx = __uint_as_float(hhi << 16), hy = __uint_as_float(hhi & 0xffff0000u);
        const uint32_t hlo = pack_bf16x2(hp.x - hx, hp.y - hy);
        if (REGACC) {
          // (register indices stay compile-time: the tile loop is unrolled)
#pragma unroll
          for (int t = 0; t < NACC; t += 2) {
            const int m0 = c0w + 16 * t;
            if (t + 1 < NT16) {
              uint32_t a0, a1, a2, a3;
              ldsm_x4_t(b_base + 2u * (m0 + 8 * (lane >> 3)), a0, a1, a2, a3);
              mma_bf16(yacc[t], a0, a1, a0, a1, hhi, hlo);
              mma_bf16(yacc[t + 1], a2, a3, a2, a3, hhi, hlo);
            } else if (t < NT16) {  // one 16-column tile, then perhaps 8 columns
              uint32_t a0, a1;
              ldsm_x2_t(b_base + 2u * (m0 + 8 * ((lane >> 3) & 1)), a0, a1);
              mma_bf16(yacc[t], a0, a1, a0, a1, hhi, hlo);
              if (tail8) {
                ldsm_x2_t(b_base + 2u * (m0 + 16), a0, a1);
                mma_bf16(yacc[t + 1], a0, a0, a0, a0, hhi, hlo);
              }
            } else if (t == NT16 && tail8) {  // 8 columns: rows 8-15 repeat rows 0-7, dropped
              uint32_t a0, a1;
              ldsm_x2_t(b_base + 2u * m0, a0, a1);
              mma_bf16(yacc[t], a0, a0, a0, a0, hhi, hlo);
            }
          }
        } else {
          int t = 0;
          for (; t + 2 <= NT16; t += 2) {
            const int m0 = c0w + 16 * t;
            uint32_t a0, a1, a2, a3;
            ldsm_x4_t(b_base + 2u * (m0 + 8 * (lane >> 3)), a0, a1, a2, a3);
            float dA[4] = {0.f, 0.f, 0.f, 0.f}, dB[4] = {0.f, 0.f, 0.f, 0.f};
            mma_bf16(dA, a0, a1, a0, a1, hhi, hlo);
            mma_bf16(dB, a2, a3, a2, a3, hhi, hlo);
            gather_red_tile(ws.y_acc, s_tok, ntg, d, m0, dA, lane, true);
            gather_red_tile(ws.y_acc, s_tok, ntg, d, m0 + 16, dB, lane, true);
          }
          if (t < NT16) {
            const int m0 = c0w + 16 * t;
            uint32_t a0, a1;
            ldsm_x2_t(b_base + 2u * (m0 + 8 * ((lane >> 3) & 1)), a0, a1);
            float dA[4] = {0.f, 0.f, 0.f, 0.f};
            mma_bf16(dA, a0, a1, a0, a1, hhi, hlo);
            gather_red_tile(ws.y_acc, s_tok, ntg, d, m0, dA, lane, true);
          }
          if (tail8) {
            uint32_t a0, a1;
            ldsm_x2_t(b_base + 2u * (c0w + 16 * NT16), a0, a1);
            float dA[4] = {0.f, 0.f, 0.f, 0.f};
            mma_bf16(dA, a0, a0, a0, a0, hhi, hlo);
            gather_red_tile(ws.y_acc, s_tok, ntg, d, c0w + 16 * NT16, dA, lane, false);
          }
        }
        // the stage that reuses this buffer: arm its barrier (this phase has completed)
        if (tid == 0 && stg + kGBufs < nst) gather_arm(&bar[b], min(CH, nrun - (stg + kGBufs) * CH), d);
        __syncthreads();  // this stage's buffer, s_red and s_h are free
      }
      if (REGACC && ok) {  // one reduction-add per output of the run
#pragma unroll
        for (int t = 0; t < NACC; ++t)
          if (t < NT16 + (tail8 ? 1 : 0))
            gather_red_tile(ws.y_acc, s_tok, ntg, d, c0w + 16 * t, yacc[t], lane, t < NT16);
      }
    }
  }
}

// =====================================================================================
// FP32 accumulator -> BF16 output; union sizes for the trace
// =====================================================================================
__global__ void __launch_bounds__(kNT) finalize_kernel(uint16_t* __restrict__ out, int B, Dims D,
                                                       Workspace ws, TraceDev tr, int dense) {
  pdl_begin();
  const size_t n8 = (size_t)B * D.d / 8;
  for (size_t i = blockIdx.x * (size_t)kNT + threadIdx.x; i < n8; i += (size_t)gridDim.x * kNT) {
    float4* src = reinterpret_cast<float4*>(ws.y_acc) + 2 * i;
    const float4 a = __ldcg(src), b = __ldcg(src + 1);
    src[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    src[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    uint4 o;
    o.x = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(a.x)) |
          ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(a.y)) << 16);
    o.y = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(a.z)) |
          ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(a.w)) << 16);
    o.z = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(b.x)) |
          ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(b.y)) << 16);
    o.w = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(b.z)) |
          ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(b.w)) << 16);
    reinterpret_cast<uint4*>(out)[i] = o;
  }
  if (blockIdx.x == 0 && tr.union_count) {
    const int nu = *ws.nused;
    for (int e = threadIdx.x; e < D.experts; e += kNT) tr.union_count[e] = 0;
    __syncthreads();
    for (int u = threadIdx.x; u < nu; u += kNT) {
      int c = 0;
      if (dense) {
        c = D.inter;
      } else {
        for (int w = 0; w < mask_words(D.ipad); ++w) c += __popc(ws.umask[(size_t)u * mask_words(D.ipad) + w]);
      }
      tr.union_count[ws.slot_expert[u]] = c;
    }
  }
}

// =====================================================================================
// host-side launcher
// =====================================================================================
int sm_count() {
  static int n[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (n[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    n[dev] = v;
  }
  return n[dev];
}

// Launch one kernel of this path, kNT threads per CTA, with programmatic stream
// serialization (the kernel begins with pdl_begin()).
template <typename... KArgs, typename... Args>
bool launch_pdl(void (*kernel)(KArgs...), dim3 grid, size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kNT, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...) == cudaSuccess;
}

int launch_general(const uint16_t* x, int B, const uint16_t* router_t, const uint16_t* records,
                   const uint32_t* sketch, const float* alpha, int k, int mode, float tau,
                   const uint16_t* lr_a, const uint16_t* lr_b, uint16_t* out, const Dims& D,
                   const Workspace& ws, const TraceDev& tr, cudaStream_t st) {
  const int E = D.experts, K = D.top_e, d = D.d;
  const int dense = (mode == 0 && k == D.inter);
  const int maxslots = min(E, B * K);
  bool ok = true;
  {
    dim3 grid((E + kRouterExp - 1) / kRouterExp, (B + kRouterTok - 1) / kRouterTok);
    ok = ok && launch_pdl(router_kernel, grid, 0, st, x, B, router_t, D, ws, tr);
  }
  const int KC = d / kColChunk;
  const size_t score_smem = (size_t)kScoreTok * (KC * 32 + 4) * 4 + 4 * 32 * 4 * 4;
  if (!dense || D.rank > 0) {
    // per slot: nsb score CTAs of kScoreRows rows, then the z CTAs of kNT / 32 rows of B_e
    const int nsb = dense ? 0 : (D.ipad + kScoreRows - 1) / kScoreRows;
    const int nzb = (D.rank + kNT / 32 - 1) / (kNT / 32);
    dim3 grid(nsb + nzb, maxslots);
    ok = ok && launch_pdl(score_kernel, grid, score_smem, st, x, sketch, alpha, lr_b, D, ws, tr, nsb);
  }
  if (!dense) ok = ok && launch_pdl(select_kernel, dim3(B * K), 0, st, k, mode, tau, D, ws, tr);
  GatherCfg cfg;
  cfg.ch = max(1, min(kGCh, (196 * 1024 / kGBufs) / (6 * d + 16)));
  cfg.lr_qs = 1;
  while (cfg.lr_qs * 8 < D.rank) cfg.lr_qs *= 2;
  cfg.lr_vec = D.rank % 8 == 0;
  {
    // staged items: about 64 KB of A_e each, within one stage buffer, a multiple of the
    // rows one pass covers; otherwise kLrPass passes from registers
    const int rpp = kNT / cfg.lr_qs;
    int rows = 0;
    if (D.rank > 0 && cfg.lr_vec) {
      const int fit = (int)(((size_t)cfg.ch * (6 * d + 16)) / (2 * D.rank));
      rows = min(fit, max(rpp, 65536 / (2 * D.rank)));
      rows = min(rows, (d + rpp - 1) / rpp * rpp) / rpp * rpp;
    }
    cfg.lr_rows = rows;
    if (rows == 0) rows = kLrPass * rpp;
    cfg.nlr = D.rank > 0 ? (d + rows - 1) / rows : 0;
  }
  cfg.dense = dense;
  cfg.wait_ns = kWaitLimitNs;
#ifdef MSB_INSTRUMENTED
  cfg.skip = debug_ctl().skip;
  if (debug_ctl().wait_ns) cfg.wait_ns = debug_ctl().wait_ns;
#endif
  // persistent CTAs, one per SM, taking work items (runs of union channels, then
  // low-rank row blocks) off a counter
  const int ngrid = sm_count();
  ok = ok && launch_pdl(union_kernel, dim3(maxslots), 0, st, D, ws, cfg.ch, ngrid, dense);
  const size_t gsmem = (size_t)kGBufs * cfg.ch * (6 * d + 16);
  if (d <= 2048)  // outputs and x fragments in registers
    ok = ok && launch_pdl(gather_kernel<16, 16>, dim3(ngrid), gsmem, st, x, records, lr_a, D, ws, cfg);
  else if (d <= 4096)  // outputs in registers, x fragments through L1
    ok = ok && launch_pdl(gather_kernel<32, 0>, dim3(ngrid), gsmem, st, x, records, lr_a, D, ws, cfg);
  else
    ok = ok && launch_pdl(gather_kernel<0, 0>, dim3(ngrid), gsmem, st, x, records, lr_a, D, ws, cfg);
  {
    const size_t n8 = (size_t)B * d / 8;
    const size_t nb = (n8 + kNT - 1) / kNT;
    const int blocks = (int)(nb < 148 * 4 ? nb : 148 * 4);
    ok = ok && launch_pdl(finalize_kernel, dim3(blocks), 0, st, out, B, D, ws, tr, dense);
  }
  return ok && cudaGetLastError() == cudaSuccess ? MSB_OK : MSB_ECUDA;
}

int general_set_smem_limits() {
  const int big = 200 * 1024;
  cudaError_t e = cudaSuccess;
  e = cudaFuncSetAttribute(score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, big);
  if (e != cudaSuccess) return MSB_ECUDA;
  e = cudaFuncSetAttribute(gather_kernel<16, 16>, cudaFuncAttributeMaxDynamicSharedMemorySize, big);
  if (e != cudaSuccess) return MSB_ECUDA;
  e = cudaFuncSetAttribute(gather_kernel<32, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, big);
  if (e != cudaSuccess) return MSB_ECUDA;
  e = cudaFuncSetAttribute(gather_kernel<0, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, big);
  return e == cudaSuccess ? MSB_OK : MSB_ECUDA;
}

}  // namespace msb
