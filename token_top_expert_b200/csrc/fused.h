// Single-launch batch-1 path (internal to libmsb).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace msb {

constexpr int MSB_ENOTFUSED = 1;  // internal: the fused path declines, use the general path

bool fused_supported(const Dims& D, int k);
int fused_setup();
int launch_fused(const uint16_t* x, const uint16_t* router_t, const uint16_t* records,
                 const uint32_t* sketch, const float* alpha, int k, const uint16_t* lr_a,
                 const uint16_t* lr_b, uint16_t* out, const Dims& D, uint32_t* err,
                 uint32_t* counters, float* y_acc, const TraceDev& tr, cudaStream_t st);

}  // namespace msb
