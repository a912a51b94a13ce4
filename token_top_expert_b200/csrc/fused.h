// Single-launch batch-1 path (internal to libmsb).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace msb {

constexpr int MSB_ENOTFUSED = 1;  // internal: the fused path declines, use the general path
// Batches up to this size run on the single-launch kernel, one cluster per (token,
// routed expert) pair, each pair reading its own channels; larger ones take the
// multi-kernel path, which reads each expert's union of channels once.  (Measured on
// B200 with d = 2048 and 4096: the single launch is ahead up to 16 tokens, behind at 32.)
constexpr int kFusedMaxBatch = 16;

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
