// Single-launch batch-1 sparse-MoE block (the decode hot path).
//
// One thread-block cluster per routed expert (or two clusters of 8 when 16-CTA
// clusters cannot all be resident).  All exchange inside a cluster goes through
// distributed shared memory and hardware cluster barriers; the only global
// synchronisation is the last-arriving CTA that converts the FP32 accumulator
// to BF16.  Phases:
//
//  A  router: the cluster's CTAs each score E/CS experts (x . W_router rows
//     staged by 1-D bulk copies), broadcast the logits over DSMEM; every CTA then
//     runs softmax + top-K and cluster c takes the c-th ranked expert.
//  B  sketch scores: each CTA stages its 16-row tiles of the packed 2-bit sketch,
//     scores them on the tensor cores (the packed codes are the bf16 A fragment),
//     broadcasts alpha*|T.x| to the cluster; z = B_e x rows are computed alongside.
//  C  exact top-k: every CTA selects the same k channels (radix select, ties to the
//     lower index); each CTA streams its share of the 6d-byte channel records
//     through a shared-memory ring and accumulates SwiGLU(gate.x, up.x) * down.
//  D  the cluster reduces its partial outputs over DSMEM (CTA q owns a d/CS
//     slice), adds A_e z, scales by the router weight and adds into the FP32
//     accumulator; the last CTA of the grid writes the BF16 output.
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
  uint32_t* counter;
  float* y_acc;
  TraceDev tr;
  Dims D;
  int k, dense, cs, cpe;
  int rpc;     // router rows per CTA
  int tpc;     // sketch row tiles per CTA
  int zpc;     // z rows per CTA (max)
  int slice;   // output elements owned per CTA in the cluster reduction (d / cs)
  int ring;    // record slots
  int group;   // channels per reduction group (<= ring)
  // shared-memory carve-up (byte offsets)
  int o_x, o_logits, o_scores, o_alpha, o_z, o_sel, o_part, o_ybuf, o_aslice, o_misc, o_big;
  int smem;
};

struct Misc {
  uint64_t bar[2 + kRingMax];
  int ids[MSB_MAX_TOP_E];
  float w[MSB_MAX_TOP_E];
  uint32_t hist[256];
  uint32_t info[4];
  uint32_t scan[kFT / 32 + 1];
  float red[kFW][2 * kGroup];
  float h[kGroup];
  int last;
  int ok;
};

__device__ __forceinline__ void store_cluster(cg::cluster_group& cl, float* local, int idx, float v,
                                              int lane, int cs) {
  // lanes 0..cs-1 each write one destination CTA
  if (lane < cs) cl.map_shared_rank(local, lane)[idx] = v;
}

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
  float* logits = reinterpret_cast<float*>(sm + P.o_logits);
  float* scores = reinterpret_cast<float*>(sm + P.o_scores);
  float* alpha_s = reinterpret_cast<float*>(sm + P.o_alpha);
  float* zs = reinterpret_cast<float*>(sm + P.o_z);
  uint16_t* sel = reinterpret_cast<uint16_t*>(sm + P.o_sel);
  float* part = reinterpret_cast<float*>(sm + P.o_part);
  float* ybuf = reinterpret_cast<float*>(sm + P.o_ybuf);
  uint16_t* aslice = reinterpret_cast<uint16_t*>(sm + P.o_aslice);
  Misc& M = *reinterpret_cast<Misc*>(sm + P.o_misc);
  uint8_t* big = sm + P.o_big;

  // Every CTA of the cluster must be running before any DSMEM store targets it:
  // arrive now, wait just before the first remote store (overlaps the loads).
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");

  // ------------------------------------------------------------------ phase A: router
  const int e_lo = min(E, q * P.rpc), e_hi = min(E, e_lo + P.rpc);
  if (tid == 0) {
    for (int i = 0; i < 2 + P.ring; ++i) mbar_init(&M.bar[i], 1);
    fence_mbar_init();
    const uint32_t rbytes = (uint32_t)(e_hi - e_lo) * 2u * d;
    mbar_arrive_expect_tx(&M.bar[0], 2u * d + rbytes);
    bulk_g2s(xs, P.x, 2u * d, &M.bar[0]);
    if (rbytes) bulk_g2s(big, P.router_t + (size_t)e_lo * d, rbytes, &M.bar[0]);
    M.ok = 1;
  }
  __syncthreads();
  bool ok = mbar_wait(&M.bar[0], 0, P.err);
  ok = __syncthreads_and(ok);
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  if (ok) {
    const uint16_t* rows = reinterpret_cast<const uint16_t*>(big);
    for (int row = warp; row < e_hi - e_lo; row += kFW) {
      const uint4* wr = reinterpret_cast<const uint4*>(rows + (size_t)row * d);
      const uint4* xr = reinterpret_cast<const uint4*>(xs);
      float acc = 0.f;
      for (int i = lane; i < d / 8; i += 32) acc = dot8(wr[i], xr[i], acc);
      acc = warp_sum(acc);
      store_cluster(cluster, logits, e_lo + row, acc, lane, CS);
    }
  }
  cluster.sync();
  if (warp == 0) {
    constexpr int MAXM = MSB_MAX_EXPERTS / 32;
    float v[MAXM];
    float mx = -INFINITY;
#pragma unroll
    for (int m = 0; m < MAXM; ++m) {
      const int ee = lane + 32 * m;
      v[m] = ee < E ? logits[ee] : -INFINITY;
      mx = fmaxf(mx, v[m]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
#pragma unroll
    for (int m = 0; m < MAXM; ++m)
      if (lane + 32 * m < E) sum += expf(v[m] - mx);
    sum = warp_sum(sum);
    uint32_t taken = 0;
    float psum = 0.f;
    for (int rr = 0; rr < K; ++rr) {
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
        bi = rr;
        bv = mx;
        if (lane == 0) atomicOr(P.err, kErrNonFinite);
      }
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
      const float pe = expf(bv - mx);
      psum += pe;
      if (lane == 0) { M.ids[rr] = bi; M.w[rr] = pe; }
    }
    __syncwarp();
    if (lane < K) M.w[lane] = M.w[lane] / (D.renorm ? psum : sum);
  }
  __syncthreads();
  const int e = M.ids[rc];
  const float we = M.w[rc];
  if (blockIdx.x == 0 && tid < K) {
    if (P.tr.expert_ids) P.tr.expert_ids[tid] = M.ids[tid];
    if (P.tr.expert_w) P.tr.expert_w[tid] = M.w[tid];
  }

  // ------------------------------------------------------------------ phase B: scores, z
  const int ntile_all = ipad / kRowTile;
  const int lt0 = min(ntile_all, q * P.tpc), lt1 = min(ntile_all, lt0 + P.tpc);
  const int nt = lt1 - lt0;
  const uint32_t code_bytes = P.dense ? 0u : (uint32_t)nt * KC * kChunkWords * 4u;
  int nz = 0;
  for (int rho = q; rho < r; rho += CS) ++nz;
  if (tid == 0 && ok) {
    uint32_t bytes = code_bytes + (P.dense ? 0u : (uint32_t)nt * kRowTile * 4u) + (uint32_t)nz * 2u * d;
    const bool lr_out = (half == 0 && r > 0);
    if (lr_out) bytes += (uint32_t)P.slice * r * 2u;
    fence_proxy_async();
    mbar_arrive_expect_tx(&M.bar[1], bytes);
    if (code_bytes) {
      bulk_g2s(big, P.sketch + ((size_t)e * ntile_all + lt0) * KC * kChunkWords, code_bytes, &M.bar[1]);
      bulk_g2s(alpha_s, P.alpha + (size_t)e * ipad + (size_t)lt0 * kRowTile, nt * kRowTile * 4u,
               &M.bar[1]);
    }
    uint16_t* brows = reinterpret_cast<uint16_t*>(big + code_bytes);
    int i = 0;
    for (int rho = q; rho < r; rho += CS, ++i)
      bulk_g2s(brows + (size_t)i * d, P.lr_b + ((size_t)e * r + rho) * d, 2u * d, &M.bar[1]);
    if (lr_out)
      bulk_g2s(aslice, P.lr_a + ((size_t)e * d + (size_t)q * P.slice) * r, (uint32_t)P.slice * r * 2u,
               &M.bar[1]);
  }
  for (int i = tid; i < kFW * P.tpc * kRowTile; i += kFT) part[i] = 0.f;
  __syncthreads();
  ok = ok && mbar_wait(&M.bar[1], 0, P.err);
  ok = __syncthreads_and(ok);
  if (ok && !P.dense && nt > 0) {
    // items (tile, chunk) in tile-major order; warp w takes a contiguous range
    const int nitems = nt * KC;
    const int i0 = warp * nitems / kFW, i1 = (warp + 1) * nitems / kFW;
    const uint2* codes = reinterpret_cast<const uint2*>(big);
    const uint32_t* x32 = reinterpret_cast<const uint32_t*>(xs);
    const int g = lane >> 2, c = lane & 3;
    int cur = -1;
    float acc0 = 0.f, acc1 = 0.f;
    for (int it = i0; it < i1; ++it) {
      const int tl = it / KC, kc = it - tl * KC;
      if (tl != cur) {
        if (cur >= 0 && c == 0) {
          part[warp * P.tpc * kRowTile + cur * kRowTile + g] = acc0;
          part[warp * P.tpc * kRowTile + cur * kRowTile + g + 8] = acc1;
        }
        cur = tl;
        acc0 = acc1 = 0.f;
      }
      const uint2 w = codes[(size_t)it * 32 + lane];
      uint32_t b[8];
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        b[2 * s] = g == 0 ? x32[kc * 32 + 8 * s + c] : 0u;
        b[2 * s + 1] = g == 0 ? x32[kc * 32 + 8 * s + c + 4] : 0u;
      }
      float a4[4] = {0.f, 0.f, 0.f, 0.f};
      mma_bf16(a4, w.x & kSketchMask, w.y & kSketchMask, (w.x << 2) & kSketchMask,
               (w.y << 2) & kSketchMask, b[0], b[1]);
      mma_bf16(a4, (w.x << 4) & kSketchMask, (w.y << 4) & kSketchMask, (w.x << 6) & kSketchMask,
               (w.y << 6) & kSketchMask, b[2], b[3]);
      mma_bf16(a4, (w.x << 8) & kSketchMask, (w.y << 8) & kSketchMask, (w.x << 10) & kSketchMask,
               (w.y << 10) & kSketchMask, b[4], b[5]);
      mma_bf16(a4, (w.x << 12) & kSketchMask, (w.y << 12) & kSketchMask, (w.x << 14) & kSketchMask,
               (w.y << 14) & kSketchMask, b[6], b[7]);
      acc0 += a4[0];
      acc1 += a4[2];
    }
    if (cur >= 0 && c == 0) {
      part[warp * P.tpc * kRowTile + cur * kRowTile + g] = acc0;
      part[warp * P.tpc * kRowTile + cur * kRowTile + g + 8] = acc1;
    }
  }
  // z rows: z[rho] = B_e[rho] . x, broadcast to the cluster
  if (ok && r > 0) {
    const uint16_t* brows = reinterpret_cast<const uint16_t*>(big + code_bytes);
    for (int i = warp; i < nz; i += kFW) {
      const uint4* br = reinterpret_cast<const uint4*>(brows + (size_t)i * d);
      const uint4* xr = reinterpret_cast<const uint4*>(xs);
      float acc = 0.f;
      for (int j = lane; j < d / 8; j += 32) acc = dot8(br[j], xr[j], acc);
      acc = warp_sum(acc);
      store_cluster(cluster, zs, q + i * CS, acc, lane, CS);
    }
  }
  __syncthreads();
  if (ok && !P.dense) {
    for (int lr = tid; lr < nt * kRowTile; lr += kFT) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < kFW; ++w) s += part[w * P.tpc * kRowTile + lr];
      s = alpha_s[lr] * fabsf(s) * 0.5f;
      const int row = lt0 * kRowTile + lr;
      for (int dst = 0; dst < CS; ++dst) cluster.map_shared_rank(scores, dst)[row] = s;
      if (half == 0 && P.tr.scores) P.tr.scores[(size_t)rc * ipad + row] = s;
    }
  }
  cluster.sync();

  // ------------------------------------------------------------------ phase C: top-k, records
  if (!P.dense) {
    constexpr int EPT = MSB_MAX_INTER / kFT;
    const int ept = (I + kFT - 1) / kFT;
    const int j0 = tid * ept;
    uint32_t key[EPT];
    uint32_t valid = 0;
#pragma unroll
    for (int m = 0; m < EPT; ++m) {
      key[m] = 0;
      if (m < ept && j0 + m < I) { key[m] = __float_as_uint(scores[j0 + m]); valid |= 1u << m; }
    }
    uint32_t kth, need;
    radix_kth<kFT, EPT>(key, valid, P.k, M.hist, M.info, &kth, &need);
    uint32_t ngt = 0, neq = 0;
#pragma unroll
    for (int m = 0; m < EPT; ++m)
      if ((valid >> m) & 1u) { ngt += key[m] > kth; neq += key[m] == kth; }
    uint32_t tot;
    const uint32_t pre = block_excl_scan<kFT>(ngt | (neq << 16), M.scan, &tot);
    uint32_t gtb = pre & 0xffffu, eqb = pre >> 16;
#pragma unroll
    for (int m = 0; m < EPT; ++m) {
      if (!((valid >> m) & 1u)) continue;
      const bool gt = key[m] > kth, eq = key[m] == kth;
      if (gt || (eq && eqb < need)) sel[gtb + min(eqb, need)] = (uint16_t)(j0 + m);
      gtb += gt;
      eqb += eq;
    }
    __syncthreads();
    if (half == 0 && q == 0) {
      for (int i = tid; i < P.k; i += kFT)
        if (P.tr.sel) P.tr.sel[(size_t)rc * P.k + i] = sel[i];
      if (tid == 0 && P.tr.sel_count) P.tr.sel_count[rc] = P.k;
    }
  }
  // this CTA's share of the k channels
  const int NQ = CS * P.cpe, gq = half * CS + q;
  const int c0 = (int)((long)gq * P.k / NQ), c1 = (int)((long)(gq + 1) * P.k / NQ);
  const int nmine = c1 - c0;
  const uint32_t rec_bytes = 6u * d;
  uint16_t* ring = reinterpret_cast<uint16_t*>(big);
  if (tid == 0 && ok) {
    fence_proxy_async();
    for (int i = 0; i < min(P.ring, nmine); ++i) {
      const int ch = P.dense ? c0 + i : (int)sel[c0 + i];
      mbar_arrive_expect_tx(&M.bar[2 + i], rec_bytes);
      bulk_g2s(ring + (size_t)i * 3 * d, P.records + ((size_t)e * I + ch) * 3 * d, rec_bytes,
               &M.bar[2 + i]);
    }
  }
  // x in registers: thread owns elements (it*kFT + tid)*8 .. +8
  constexpr int ITM = MSB_MAX_D / (kFT * 8);
  const int IT = (d + kFT * 8 - 1) / (kFT * 8);
  float y[ITM][8];
  float xf[ITM][8];
#pragma unroll
  for (int it = 0; it < ITM; ++it) {
    const int el = (it * kFT + tid) * 8;
#pragma unroll
    for (int i = 0; i < 8; ++i) { y[it][i] = 0.f; xf[it][i] = 0.f; }
    if (it < IT && el < d) {
      const uint4 xv = *reinterpret_cast<const uint4*>(xs + el);
      xf[it][0] = bf16_lo(xv.x); xf[it][1] = bf16_hi(xv.x);
      xf[it][2] = bf16_lo(xv.y); xf[it][3] = bf16_hi(xv.y);
      xf[it][4] = bf16_lo(xv.z); xf[it][5] = bf16_hi(xv.z);
      xf[it][6] = bf16_lo(xv.w); xf[it][7] = bf16_hi(xv.w);
    }
  }
  __syncthreads();
  for (int g0 = 0; g0 < nmine; g0 += P.group) {
    const int ng = min(P.group, nmine - g0);
    bool okw = true;
    for (int i = 0; i < ng; ++i) {
      const int ci = g0 + i;
      okw = okw && (!ok || mbar_wait(&M.bar[2 + ci % P.ring], (ci / P.ring) & 1u, P.err));
    }
    ok = __syncthreads_and(ok && okw);
    float v[2 * kGroup];
#pragma unroll
    for (int i = 0; i < 2 * kGroup; ++i) v[i] = 0.f;
    if (ok) {
#pragma unroll
      for (int i = 0; i < kGroup; ++i) {
        if (i < ng) {
          const uint16_t* rec = ring + (size_t)((g0 + i) % P.ring) * 3 * d;
#pragma unroll
          for (int it = 0; it < ITM; ++it) {
            const int el = (it * kFT + tid) * 8;
            if (it < IT && el < d) {
              v[i] = dot8f(*reinterpret_cast<const uint4*>(rec + el), xf[it], v[i]);
              v[kGroup + i] = dot8f(*reinterpret_cast<const uint4*>(rec + d + el), xf[it], v[kGroup + i]);
            }
          }
        }
      }
    }
    // transpose-reduce 16 values across the warp: lane pair (2m, 2m+1) ends with value m
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const bool up = lane & 16;
      const float send = up ? v[i] : v[i + 8];
      const float keep = up ? v[i + 8] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const bool up = lane & 8;
      const float send = up ? v[i] : v[i + 4];
      const float keep = up ? v[i + 4] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const bool up = lane & 4;
      const float send = up ? v[i] : v[i + 2];
      const float keep = up ? v[i + 2] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    {
      const bool up = lane & 2;
      const float send = up ? v[0] : v[1];
      const float keep = up ? v[1] : v[0];
      v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
    if ((lane & 1) == 0) M.red[warp][lane >> 1] = v[0];
    __syncthreads();
    if (tid < ng) {
      float gs = 0.f, us = 0.f;
#pragma unroll
      for (int w = 0; w < kFW; ++w) { gs += M.red[w][tid]; us += M.red[w][kGroup + tid]; }
      M.h[tid] = silu(gs) * us;
    }
    __syncthreads();
    if (ok) {
      for (int i = 0; i < ng; ++i) {
        const uint16_t* rec = ring + (size_t)((g0 + i) % P.ring) * 3 * d + 2 * d;
        const float h = M.h[i];
#pragma unroll
        for (int it = 0; it < ITM; ++it) {
          const int el = (it * kFT + tid) * 8;
          if (it < IT && el < d) {
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

  // ------------------------------------------------------------------ phase D: reduce, combine
#pragma unroll
  for (int it = 0; it < ITM; ++it) {
    const int el = (it * kFT + tid) * 8;
    if (it < IT && el < d) {
      *reinterpret_cast<float4*>(ybuf + el) = make_float4(y[it][0], y[it][1], y[it][2], y[it][3]);
      *reinterpret_cast<float4*>(ybuf + el + 4) = make_float4(y[it][4], y[it][5], y[it][6], y[it][7]);
    }
  }
  cluster.sync();
  if (ok) {
    for (int i = tid; i < P.slice; i += kFT) {
      const int el = q * P.slice + i;
      float acc = 0.f;
      for (int j = 0; j < CS; ++j) acc += cluster.map_shared_rank(ybuf, j)[el];
      if (half == 0 && r > 0) {
        const uint16_t* ar = aslice + (size_t)i * r;
        for (int rho = 0; rho < r; ++rho) acc = fmaf(bf16_lo(ar[rho]), zs[rho], acc);
      }
      atomicAdd(P.y_acc + el, we * acc);
    }
  }
  __threadfence();
  cluster.sync();
  if (tid == 0) M.last = (atomicAdd(P.counter, 1u) == gridDim.x - 1);
  __syncthreads();
  if (M.last) {
    __threadfence();
    for (int i = tid; i < d; i += kFT) {
      const float v = atomicExch(P.y_acc + i, 0.f);
      P.out[i] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    }
    if (P.tr.union_count) {
      for (int i = tid; i < E; i += kFT) P.tr.union_count[i] = 0;
      __syncthreads();
      if (tid < K) P.tr.union_count[M.ids[tid]] = P.k;
    }
    if (tid == 0) *P.counter = 0u;
  }
}

// =====================================================================================
// host side
// =====================================================================================
namespace {
int g_max_clusters16[64];
int g_max_clusters8[64];
bool g_ready[64];

int cur_dev() {
  int d = 0;
  cudaGetDevice(&d);
  return d;
}

int align_up(int v, int a) { return (v + a - 1) / a * a; }

// Fill the carve-up for cluster size cs; returns false if it does not fit.
bool plan(FusedParams& P, const Dims& D, int k, int cs, int cpe) {
  const int d = D.d, E = D.experts, ipad = D.ipad, r = D.rank;
  P.cs = cs;
  P.cpe = cpe;
  P.rpc = (E + cs - 1) / cs;
  P.tpc = (ipad / kRowTile + cs - 1) / cs;
  P.zpc = (r + cs - 1) / cs;
  P.slice = d / cs;
  int o = 0;
  P.o_x = o;      o = align_up(o + 2 * d, 128);
  P.o_logits = o; o = align_up(o + 4 * E, 128);
  P.o_scores = o; o = align_up(o + 4 * ipad, 128);
  P.o_alpha = o;  o = align_up(o + 4 * P.tpc * kRowTile, 128);
  P.o_z = o;      o = align_up(o + 4 * (r > 0 ? r : 1), 128);
  P.o_sel = o;    o = align_up(o + 2 * ipad, 128);
  P.o_part = o;   o = align_up(o + 4 * kFW * P.tpc * kRowTile, 128);
  P.o_ybuf = o;   o = align_up(o + 4 * d, 128);
  P.o_aslice = o; o = align_up(o + 2 * P.slice * (r > 0 ? r : 0), 128);
  P.o_misc = o;   o = align_up(o + (int)sizeof(Misc), 128);
  P.o_big = o;
  const int avail = kSmemMax - o;
  const int need_a = P.rpc * 2 * d;
  const int need_b = (P.dense ? 0 : P.tpc * (d / kColChunk) * kChunkWords * 4) + P.zpc * 2 * d;
  const int rec = 6 * d;
  int ring = avail / rec;
  if (ring > kRingMax) ring = kRingMax;
  if (ring < 2 || need_a > avail || need_b > avail) return false;
  P.ring = ring;
  P.group = ring < kGroup ? ring : kGroup;
  int big = ring * rec;
  if (need_a > big) big = need_a;
  if (need_b > big) big = need_b;
  P.smem = o + big;
  return P.smem <= kSmemMax;
}

// Prefer one 16-CTA cluster per routed expert when K of them are resident at once,
// else two 8-CTA clusters per expert when 2K are; otherwise whichever shape can be
// resident at all (clusters that do not fit wait for a free GPC: correct, slower).
bool choose(FusedParams& P, const Dims& D, int k) {
  const int dev = cur_dev();
  if (dev < 0 || dev >= 64 || !g_ready[dev]) return false;
  const bool ok16 = D.d % (8 * 16) == 0 && g_max_clusters16[dev] >= 1;
  const bool ok8 = D.d % (8 * 8) == 0 && g_max_clusters8[dev] >= 1;
  if (ok16 && g_max_clusters16[dev] >= D.top_e && plan(P, D, k, 16, 1)) return true;
  if (ok8 && g_max_clusters8[dev] >= 2 * D.top_e && plan(P, D, k, 8, 2)) return true;
  if (ok16 && plan(P, D, k, 16, 1)) return true;
  if (ok8 && plan(P, D, k, 8, 2)) return true;
  return false;
}
}  // namespace

int fused_setup() {
  const int dev = cur_dev();
  if (dev < 0 || dev >= 64) return MSB_ECUDA;
  if (cudaFuncSetAttribute(fused_block_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kSmemMax) != cudaSuccess)
    return MSB_ECUDA;
  if (cudaFuncSetAttribute(fused_block_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
      cudaSuccess) {
    cudaGetLastError();
  }
  for (int cs : {16, 8}) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cs * 16, 1, 1);
    cfg.blockDim = dim3(kFT, 1, 1);
    cfg.dynamicSmemBytes = kSmemMax;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, fused_block_kernel, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    (cs == 16 ? g_max_clusters16 : g_max_clusters8)[dev] = n;
  }
  g_ready[dev] = true;
  return MSB_OK;
}

void fused_plan_info(const Dims& D, int k, int* info) {
  FusedParams P{};
  P.dense = (k == D.inter);
  const int dev = cur_dev();
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
  P.counter = counters + kCntFused;
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
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = P.cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, fused_block_kernel, P);
  return e == cudaSuccess ? MSB_OK : MSB_ECUDA;
}

}  // namespace msb
