// moe_sparse_block_noalloc: the batch-1 block with its scratch in a static device
// array, for callers that cannot allocate device memory.
//
// Some callers own no device allocator: a plugin that its host framework hands
// only input and output buffers, or code running where a cudaMalloc would
// synchronise the device or is not permitted at all.  This entry point needs
// nothing from them but the inputs and the output.
//
// The scratch the single-launch kernel needs (a sticky error word, per-slice
// arrival counters and a d-float FP32 accumulator) lives in the file-scope array
// below.  Every GPU that loads this library holds it (kStaticBytes) until the
// process exits.  Every call shares it and it keeps the last call's contents, so
// each call clears it on its stream before the launch; calls that overlap on the
// GPU (different streams without ordering) race on it.
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "fused.h"
#include "msb.h"

namespace msb {
namespace {

constexpr size_t kHeaderBytes = 256;                           // error word
constexpr size_t kCounterBytes = 4 * (size_t)kCounters;        // arrival counters
constexpr size_t kStaticBytes = kHeaderBytes + kCounterBytes + 4 * (size_t)MSB_NOALLOC_MAX_D;

static __device__ __align__(256) unsigned char g_scratch[kStaticBytes];

// Device address of g_scratch for the current device, looked up once per device.
void* scratch_address(int* status) {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    *status = MSB_ECUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      *status = MSB_ECUDA;
      return nullptr;
    }
    if (fused_setup() != MSB_OK) {
      *status = MSB_ECUDA;
      return nullptr;
    }
    addr[dev] = p;
  }
  *status = MSB_OK;
  return addr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace msb

using namespace msb;

extern "C" int32_t moe_sparse_block_noalloc(const void* x, const void* router_t,
                                            const void* records, const uint32_t* sketch,
                                            const float* alpha, int32_t k, const void* lr_a,
                                            const void* lr_b, void* out, const msb_dims* dims,
                                            const msb_trace* trace, void* stream) {
  if (!dims || !x || !router_t || !records || !out) return MSB_EINVAL;
  const msb_dims m = *dims;
  if (m.d < 64 || m.d % 64 != 0 || m.inter < 1 || m.experts < 1 || m.top_e < 1 ||
      m.top_e > m.experts || m.rank < 0 || (m.renorm != 0 && m.renorm != 1) || k < 1 ||
      k > m.inter)
    return MSB_EINVAL;
  if (m.d > MSB_NOALLOC_MAX_D || m.inter > MSB_MAX_INTER || m.experts > MSB_MAX_EXPERTS ||
      m.top_e > MSB_MAX_TOP_E || m.rank > MSB_MAX_RANK)
    return MSB_EUNSUPPORTED;
  const bool dense = (k == m.inter);
  if (!dense && (!sketch || !alpha)) return MSB_EINVAL;
  if (m.rank > 0 && (!lr_a || !lr_b)) return MSB_EINVAL;
  if (!aligned16(x) || !aligned16(router_t) || !aligned16(records) || !aligned16(out) ||
      (sketch && !aligned16(sketch)) || (alpha && !aligned16(alpha)) ||
      (lr_a && !aligned16(lr_a)) || (lr_b && !aligned16(lr_b)))
    return MSB_EINVAL;
  const uintptr_t xa = reinterpret_cast<uintptr_t>(x), oa = reinterpret_cast<uintptr_t>(out);
  const size_t nb = 2 * (size_t)m.d;
  if (xa < oa + nb && oa < xa + nb) return MSB_EINVAL;

  int status = MSB_OK;
  unsigned char* base = static_cast<unsigned char*>(scratch_address(&status));
  if (!base) return status;

  Dims D;
  D.d = m.d;
  D.inter = m.inter;
  D.ipad = pad16(m.inter);
  D.experts = m.experts;
  D.top_e = m.top_e;
  D.rank = m.rank;
  D.renorm = m.renorm;
  if (!fused_supported(D, k)) return MSB_EUNSUPPORTED;

  TraceDev tr = {nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
  if (trace) {
    tr.expert_ids = trace->expert_ids;
    tr.expert_w = trace->expert_w;
    tr.sel = trace->sel;
    tr.sel_count = trace->sel_count;
    tr.union_count = trace->union_count;
    tr.scores = trace->scores;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the kernel needs the error word, the counters and the accumulator zeroed
  const size_t used = kHeaderBytes + kCounterBytes + 4 * (size_t)m.d;
  if (cudaMemsetAsync(base, 0, used, st) != cudaSuccess) return MSB_ECUDA;
  uint32_t* err = reinterpret_cast<uint32_t*>(base);
  uint32_t* counters = reinterpret_cast<uint32_t*>(base + kHeaderBytes);
  float* y_acc = reinterpret_cast<float*>(base + kHeaderBytes + kCounterBytes);
  const int rc = launch_fused(static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(router_t),
                              static_cast<const uint16_t*>(records), sketch, alpha, k,
                              static_cast<const uint16_t*>(lr_a), static_cast<const uint16_t*>(lr_b),
                              static_cast<uint16_t*>(out), D, err, counters, y_acc, tr, st);
  return rc == MSB_ENOTFUSED ? MSB_EUNSUPPORTED : rc;
}

// The kernel records a non-finite router logit, an expired bounded wait or a failed
// consistency check in the array's first word; this reads it (and clears it) for the
// caller, who has no workspace for msb_check to read.
extern "C" int32_t msb_noalloc_check(void* stream) {
  int status = MSB_OK;
  unsigned char* base = static_cast<unsigned char*>(scratch_address(&status));
  if (!base) return status;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t err = 0;
  if (cudaMemcpyAsync(&err, base, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess) return MSB_ECUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MSB_ECUDA;
  if (err == 0) return MSB_OK;
  if (cudaMemsetAsync(base, 0, 4, st) != cudaSuccess) return MSB_ECUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MSB_ECUDA;
  if (err & kErrInternal) return MSB_EINTERNAL;
  return (err & kErrTimeout) ? MSB_ETIMEOUT : MSB_ENONFINITE;
}
