// Host-side launch entry points of the kernels (internal to libmsb).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace msb {

// Multi-kernel path (any batch).  mode 0 = top-k (k == I: dense), 1 = threshold tau.
int launch_general(const uint16_t* x, int B, const uint16_t* router_t, const uint16_t* records,
                   const uint32_t* sketch, const float* alpha, int k, int mode, float tau,
                   const uint16_t* lr_a, const uint16_t* lr_b, uint16_t* out, const Dims& D,
                   const Workspace& ws, const TraceDev& tr, cudaStream_t st);
int general_set_smem_limits();

#ifdef MSB_INSTRUMENTED
// Test and profiling controls of the instrumented build (libmsb_instr.so); the product
// library is compiled without them.
struct DebugCtl {
  unsigned long long* marks;  // phase marks of the single-launch kernel ([grid][16]), or null
  uint32_t skip;              // 1: the single-launch kernel's first CTA never issues its first
                              //    record copy; 2: the gather CTA of work item 0 never issues
                              //    its first stage -- so that a bounded wait runs out
  uint64_t wait_ns;           // bounded-wait limit (0: the product's)
};
DebugCtl& debug_ctl();
#endif

// Residual add + RMSNorm glue between stacked layers.
int launch_residual_rmsnorm(float* h, const uint16_t* y, uint16_t* x_next, int B, int d, float eps,
                            cudaStream_t st);

}  // namespace msb
