// Single-launch batch-1 path: not built yet; the general path serves batch 1.
#include "fused.h"

namespace msb {

bool fused_supported(const Dims&, int) { return false; }
int fused_setup() { return MSB_OK; }
int launch_fused(const uint16_t*, const uint16_t*, const uint16_t*, const uint32_t*, const float*,
                 int, const uint16_t*, const uint16_t*, uint16_t*, const Dims&, uint32_t*,
                 uint32_t*, float*, const TraceDev&, cudaStream_t) {
  return MSB_ENOTFUSED;
}

}  // namespace msb
