// Single-launch batch-1 path (internal to libmsb).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace msb {

constexpr int MSB_ENOTFUSED = 1;  // internal: the fused path declines, use the general path
// The single-launch kernel takes batches up to this size, one cluster per (token, routed
// expert) pair, each pair reading its own channels; the multi-kernel path reads each
// expert's union of channels once.
constexpr int kFusedMaxBatch = 16;

// Largest batch that runs on the single launch by default.  Its records traffic grows
// with every (token, expert) pair while the union's saturates, so the crossover falls
// as d grows: measured on B200, the single launch is ahead up to 12 tokens and behind
// at 16 at d = 2048, ahead at 2 and behind from 4 at d = 4096; the limit is
// 12 (2048 / d)^2 tokens, 1..kFusedMaxBatch.  `single` (the caller asked for the
// single launch) and 4-bit records (the single launch only) raise it to kFusedMaxBatch.
inline int single_launch_max_batch(const Dims& D, bool single, bool q4) {
  if (single || q4) return kFusedMaxBatch;
  const long long v = 12LL * 2048 * 2048 / ((long long)D.d * D.d);
  return v < 1 ? 1 : (v > kFusedMaxBatch ? kFusedMaxBatch : (int)v);
}

bool fused_supported(const Dims& D, int k, bool q4 = false);
// {cluster size, clusters per expert, ring slots, smem bytes, max 16-clusters, max 8-clusters}
void fused_plan_info(const Dims& D, int k, int batch, int* info6);
int fused_setup();
int launch_fused(const uint16_t* x, const uint16_t* router_t, const uint16_t* records,
                 const uint32_t* sketch, const float* alpha, int k, const uint16_t* lr_a,
                 const uint16_t* lr_b, uint16_t* out, const Dims& D, uint32_t* err,
                 uint32_t* counters, float* y_acc, const TraceDev& tr, cudaStream_t st,
                 bool x_mapped = false, bool x_ready = false, int batch = 1, bool q4 = false);

}  // namespace msb
