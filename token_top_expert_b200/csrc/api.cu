// C ABI entry points of libmsb: argument checks, workspace layout, dispatch.
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "common.cuh"
#include "fused.h"
#include "launch.h"
#include "msb.h"
#include "msb_q4.h"

namespace msb {

#ifdef MSB_INSTRUMENTED
DebugCtl& debug_ctl() {
  static DebugCtl ctl = {nullptr, 0u, 0u};
  return ctl;
}
#endif

namespace {

constexpr size_t kAlign = 256;
size_t up(size_t v) { return (v + kAlign - 1) & ~(kAlign - 1); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_dims(const msb_dims* dims) {
  if (!dims) return MSB_EINVAL;
  const msb_dims& m = *dims;
  if (m.d < 64 || m.d % 64 != 0 || m.inter < 1 || m.experts < 1 || m.top_e < 1 ||
      m.top_e > m.experts || m.rank < 0 || (m.renorm != 0 && m.renorm != 1))
    return MSB_EINVAL;
  if (m.d > MSB_MAX_D || m.inter > MSB_MAX_INTER || m.experts > MSB_MAX_EXPERTS ||
      m.top_e > MSB_MAX_TOP_E || m.rank > MSB_MAX_RANK)
    return MSB_EUNSUPPORTED;
  return MSB_OK;
}

Dims to_dims(const msb_dims& m) {
  Dims D;
  D.d = m.d;
  D.inter = m.inter;
  D.ipad = pad16(m.inter);
  D.experts = m.experts;
  D.top_e = m.top_e;
  D.rank = m.rank;
  D.renorm = m.renorm;
  return D;
}

// Byte offsets of every workspace array for a batch of B tokens.
struct Layout {
  size_t err, counters, y_acc, logits, ids, wts, slot_expert, slot_off, nused, pair_tok, pair_w,
      pair_slot, pair_of, scores, selmask, sel, selcnt, umask, z, ulist, ucnt, coff, total;
};

Layout layout(const Dims& D, int B) {
  Layout L;
  const size_t P = (size_t)B * D.top_e, E = D.experts;
  size_t o = 0;
  L.err = o;           o = up(o + 4);
  L.counters = o;      o = up(o + 4 * (size_t)kCounters);
  L.y_acc = o;         o = up(o + 4 * (size_t)B * D.d);
  L.logits = o;        o = up(o + 4 * (size_t)B * E);
  L.ids = o;           o = up(o + 4 * P);
  L.wts = o;           o = up(o + 4 * P);
  L.slot_expert = o;   o = up(o + 4 * E);
  L.slot_off = o;      o = up(o + 4 * (E + 1));
  L.nused = o;         o = up(o + 4);
  L.pair_tok = o;      o = up(o + 4 * P);
  L.pair_w = o;        o = up(o + 4 * P);
  L.pair_slot = o;     o = up(o + 4 * P);
  L.pair_of = o;       o = up(o + 4 * P);
  L.scores = o;        o = up(o + 4 * P * D.ipad);
  L.selmask = o;       o = up(o + 4 * P * mask_words(D.ipad));
  L.sel = o;           o = up(o + 2 * P * D.ipad);
  L.selcnt = o;        o = up(o + 4 * P);
  L.umask = o;         o = up(o + 4 * E * mask_words(D.ipad));
  L.z = o;             o = up(o + 4 * P * (size_t)(D.rank > 0 ? D.rank : 1));
  L.ulist = o;         o = up(o + 2 * E * D.ipad);
  L.ucnt = o;          o = up(o + 4 * E);
  L.coff = o;          o = up(o + 4 * (E + 1));
  L.total = o;
  return L;
}

Workspace bind(void* base, const Layout& L) {
  uint8_t* b = static_cast<uint8_t*>(base);
  Workspace w;
  w.err = reinterpret_cast<uint32_t*>(b + L.err);
  w.counters = reinterpret_cast<uint32_t*>(b + L.counters);
  w.y_acc = reinterpret_cast<float*>(b + L.y_acc);
  w.logits = reinterpret_cast<float*>(b + L.logits);
  w.ids = reinterpret_cast<int32_t*>(b + L.ids);
  w.wts = reinterpret_cast<float*>(b + L.wts);
  w.slot_expert = reinterpret_cast<int32_t*>(b + L.slot_expert);
  w.slot_off = reinterpret_cast<int32_t*>(b + L.slot_off);
  w.nused = reinterpret_cast<int32_t*>(b + L.nused);
  w.pair_tok = reinterpret_cast<int32_t*>(b + L.pair_tok);
  w.pair_w = reinterpret_cast<float*>(b + L.pair_w);
  w.pair_slot = reinterpret_cast<int32_t*>(b + L.pair_slot);
  w.pair_of = reinterpret_cast<int32_t*>(b + L.pair_of);
  w.scores = reinterpret_cast<float*>(b + L.scores);
  w.selmask = reinterpret_cast<uint32_t*>(b + L.selmask);
  w.sel = reinterpret_cast<uint16_t*>(b + L.sel);
  w.selcnt = reinterpret_cast<int32_t*>(b + L.selcnt);
  w.umask = reinterpret_cast<uint32_t*>(b + L.umask);
  w.z = reinterpret_cast<float*>(b + L.z);
  w.ulist = reinterpret_cast<uint16_t*>(b + L.ulist);
  w.ucnt = reinterpret_cast<int32_t*>(b + L.ucnt);
  w.coff = reinterpret_cast<int32_t*>(b + L.coff);
  return w;
}

TraceDev to_trace(const msb_trace* t) {
  TraceDev d;
  std::memset(&d, 0, sizeof(d));
  if (t) {
    d.expert_ids = t->expert_ids;
    d.expert_w = t->expert_w;
    d.sel = t->sel;
    d.sel_count = t->sel_count;
    d.union_count = t->union_count;
    d.scores = t->scores;
  }
  return d;
}

// One-time per-device attribute setup (dynamic shared memory limits).
int ensure_setup() {
  static std::mutex mu;
  static bool done[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MSB_ECUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (done[dev]) return MSB_OK;
  int rc = general_set_smem_limits();
  if (rc != MSB_OK) return rc;
  rc = fused_setup();
  if (rc != MSB_OK) return rc;
  done[dev] = true;
  return MSB_OK;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// Argument checks of a block call (no CUDA call): MSB_OK or the error to return.
int block_check(const void* x, int32_t batch, const void* router_t, const void* records,
                const uint32_t* sketch, const float* alpha, int32_t k, int mode, float tau,
                const void* lr_a, const void* lr_b, const void* out, const msb_dims* dims,
                const void* workspace, size_t workspace_bytes) {
  int rc = check_dims(dims);
  if (rc != MSB_OK) return rc;
  if (batch < 1) return MSB_EINVAL;
  if (batch > MSB_MAX_BATCH) return MSB_EUNSUPPORTED;
  const Dims D = to_dims(*dims);
  const bool dense = (mode == 0 && k == D.inter);
  if (mode == 0 && (k < 1 || k > D.inter)) return MSB_EINVAL;
  if (mode == 1 && !(tau == tau)) return MSB_EINVAL;
  if (!x || !router_t || !records || !out || !workspace) return MSB_EINVAL;
  if (!dense && (!sketch || !alpha)) return MSB_EINVAL;
  if (D.rank > 0 && (!lr_a || !lr_b)) return MSB_EINVAL;
  if (!aligned16(x) || !aligned16(router_t) || !aligned16(records) || !aligned16(out) ||
      !aligned16(workspace) || (sketch && !aligned16(sketch)) || (alpha && !aligned16(alpha)))
    return MSB_EINVAL;
  if ((lr_a && !aligned16(lr_a)) || (lr_b && !aligned16(lr_b))) return MSB_EINVAL;
  const size_t act_bytes = (size_t)batch * D.d * 2;
  if (overlaps(x, act_bytes, out, act_bytes)) return MSB_EINVAL;
  if (workspace_bytes < layout(D, batch).total) return MSB_EINVAL;
  return MSB_OK;
}

int block_common(const void* x, int32_t batch, const void* router_t, const void* records,
                 const uint32_t* sketch, const float* alpha, int32_t k, int mode, float tau,
                 const void* lr_a, const void* lr_b, void* out, const msb_dims* dims,
                 void* workspace, size_t workspace_bytes, const msb_trace* trace, uint32_t flags,
                 void* stream, bool x_mapped = false, bool q4 = false) {
  int rc = check_dims(dims);
  if (rc != MSB_OK) return rc;
  if (batch < 1) return MSB_EINVAL;
  if (batch > MSB_MAX_BATCH) return MSB_EUNSUPPORTED;
  const Dims D = to_dims(*dims);
  const bool dense = (mode == 0 && k == D.inter);
  if (mode == 0 && (k < 1 || k > D.inter)) return MSB_EINVAL;
  if (mode == 1 && !(tau == tau)) return MSB_EINVAL;
  if (!x || !router_t || !records || !out || !workspace) return MSB_EINVAL;
  if (!dense && (!sketch || !alpha)) return MSB_EINVAL;
  if (D.rank > 0 && (!lr_a || !lr_b)) return MSB_EINVAL;
  if (!aligned16(x) || !aligned16(router_t) || !aligned16(records) || !aligned16(out) ||
      !aligned16(workspace) || (sketch && !aligned16(sketch)) || (alpha && !aligned16(alpha)))
    return MSB_EINVAL;
  if ((lr_a && !aligned16(lr_a)) || (lr_b && !aligned16(lr_b))) return MSB_EINVAL;
  const size_t act_bytes = (size_t)batch * D.d * 2;
  if (overlaps(x, act_bytes, out, act_bytes)) return MSB_EINVAL;
  const Layout L = layout(D, batch);
  if (workspace_bytes < L.total) return MSB_EINVAL;
  rc = ensure_setup();
  if (rc != MSB_OK) return rc;
  const Workspace ws = bind(workspace, L);
  const TraceDev tr = to_trace(trace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  const uint16_t* rt = static_cast<const uint16_t*>(router_t);
  const uint16_t* rec = static_cast<const uint16_t*>(records);
  const uint16_t* la = static_cast<const uint16_t*>(lr_a);
  const uint16_t* lb = static_cast<const uint16_t*>(lr_b);
  uint16_t* o = static_cast<uint16_t*>(out);
  if (mode == 0 && batch <= single_launch_max_batch(D, (flags & MSB_FLAG_SINGLE) != 0, q4) &&
      !(flags & MSB_FLAG_GENERAL) && fused_supported(D, k, q4)) {
    rc = launch_fused(xb, rt, rec, sketch, alpha, k, la, lb, o, D, ws.err, ws.counters, ws.y_acc,
                      tr, st, x_mapped, (flags & MSB_FLAG_X_READY) != 0, batch, q4);
    if (rc != MSB_ENOTFUSED) return rc;
  }
  if (x_mapped) return MSB_ENOTFUSED;  // the multi-kernel path takes device buffers only
  if (q4) return MSB_EUNSUPPORTED;     // 4-bit records: the single-launch kernel only
  return launch_general(xb, batch, rt, rec, sketch, alpha, k, mode, tau, la, lb, o, D, ws, tr, st);
}

}  // namespace
}  // namespace msb

using namespace msb;

extern "C" {

size_t msb_sketch_words(const msb_dims* dims) {
  if (check_dims(dims) != MSB_OK) return 0;
  return (size_t)dims->experts * pad16(dims->inter) * dims->d / 16;
}

size_t msb_alpha_count(const msb_dims* dims) {
  if (check_dims(dims) != MSB_OK) return 0;
  return (size_t)dims->experts * pad16(dims->inter);
}

size_t msb_workspace_size(const msb_dims* dims, int32_t max_batch) {
  if (check_dims(dims) != MSB_OK || max_batch < 1 || max_batch > MSB_MAX_BATCH) return 0;
  return layout(to_dims(*dims), max_batch).total;
}

int32_t msb_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
  if (!workspace || workspace_bytes == 0) return MSB_EINVAL;
  return cudaMemsetAsync(workspace, 0, workspace_bytes, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? MSB_OK
             : MSB_ECUDA;
}

int32_t msb_check(void* workspace, void* stream) {
  if (!workspace) return MSB_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t err = 0;
  if (cudaMemcpyAsync(&err, workspace, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return MSB_ECUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MSB_ECUDA;
  if (err == 0) return MSB_OK;
  const uint32_t zero = 0;
  if (cudaMemcpyAsync(workspace, &zero, 4, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return MSB_ECUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MSB_ECUDA;
  if (err & kErrInternal) return MSB_EINTERNAL;
  return (err & kErrTimeout) ? MSB_ETIMEOUT : MSB_ENONFINITE;
}

const char* msb_strerror(int32_t status) {
  switch (status) {
    case MSB_OK: return "ok";
    case MSB_EINVAL: return "invalid argument (null pointer, size out of range, misaligned "
                            "pointer, workspace too small or out overlapping x)";
    case MSB_EUNSUPPORTED: return "size beyond the compiled limits";
    case MSB_ECUDA: return "CUDA launch or runtime error";
    case MSB_ETIMEOUT: return "a kernel's bounded wait ran out";
    case MSB_ENONFINITE: return "non-finite router logits (x or W_router has NaN/Inf)";
    case MSB_EINTERNAL: return "a kernel's internal consistency check failed";
    default: return "unknown status";
  }
}

int32_t moe_sparse_block(const void* x, int32_t batch, const void* router_t, const void* records,
                         const uint32_t* sketch, const float* alpha, int32_t k, const void* lr_a,
                         const void* lr_b, void* out, const msb_dims* dims, void* workspace,
                         size_t workspace_bytes, const msb_trace* trace, uint32_t flags,
                         void* stream) {
  return block_common(x, batch, router_t, records, sketch, alpha, k, 0, 0.f, lr_a, lr_b, out, dims,
                      workspace, workspace_bytes, trace, flags, stream);
}

int32_t moe_sparse_block_q4(const void* x, int32_t batch, const void* router_t, const void* records_q4,
                            const uint32_t* sketch, const float* alpha, int32_t k, const void* lr_a,
                            const void* lr_b, void* out, const msb_dims* dims, void* workspace,
                            size_t workspace_bytes, const msb_trace* trace, uint32_t flags,
                            void* stream) {
  if (flags & MSB_FLAG_GENERAL) return MSB_EUNSUPPORTED;
  return block_common(x, batch, router_t, records_q4, sketch, alpha, k, 0, 0.f, lr_a, lr_b, out, dims,
                      workspace, workspace_bytes, trace, flags, stream, false, true);
}

int32_t moe_sparse_block_top_e(const void* x, int32_t batch, const void* router_t,
                               const void* records, const uint32_t* sketch, const float* alpha,
                               int32_t k, int32_t top_e, const void* lr_a, const void* lr_b,
                               void* out, const msb_dims* dims, void* workspace,
                               size_t workspace_bytes, const msb_trace* trace, uint32_t flags,
                               void* stream) {
  // "MoE top_k override (--moe-top-k)", "Ce que ca fait": fewer experts than trained only
  if (!dims || top_e < 1 || top_e > dims->top_e) return MSB_EINVAL;
  msb_dims m = *dims;
  m.top_e = top_e;
  return block_common(x, batch, router_t, records, sketch, alpha, k, 0, 0.f, lr_a, lr_b, out, &m,
                      workspace, workspace_bytes, trace, flags, stream);
}

// Device address of pinned host memory that is mapped into the current device's address
// space, or null (pageable memory, or not mapped).
const void* mapped_address(const void* h) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, h) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return a.type == cudaMemoryTypeHost ? a.devicePointer : nullptr;
}

int32_t moe_sparse_block_host(const void* x_host, void* x_dev, int32_t batch, const void* router_t,
                              const void* records, const uint32_t* sketch, const float* alpha,
                              int32_t k, const void* lr_a, const void* lr_b, void* out_dev,
                              void* out_host, const msb_dims* dims, void* workspace,
                              size_t workspace_bytes, uint32_t flags, void* stream) {
  // every check before the first copy, so that a rejected call enqueues nothing
  int rc = block_check(x_dev, batch, router_t, records, sketch, alpha, k, 0, 0.f, lr_a, lr_b, out_dev,
                       dims, workspace, workspace_bytes);
  if (rc != MSB_OK) return rc;
  if (!x_host || !out_host) return MSB_EINVAL;
  const size_t bytes = (size_t)batch * dims->d * 2;
  if (overlaps(x_host, bytes, out_host, bytes)) return MSB_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // pinned, mapped host buffers on the single-launch path: the kernel itself reads x and
  // writes the result across the host link (no copy-engine round trip between launches)
  if (batch <= single_launch_max_batch(to_dims(*dims), (flags & MSB_FLAG_SINGLE) != 0, false) &&
      !(flags & MSB_FLAG_GENERAL)) {
    const void* xm = mapped_address(x_host);
    void* om = const_cast<void*>(mapped_address(out_host));
    if (xm && om && aligned16(xm) && aligned16(om)) {
      rc = block_common(xm, batch, router_t, records, sketch, alpha, k, 0, 0.f, lr_a, lr_b, om, dims,
                        workspace, workspace_bytes, nullptr, flags, stream, true);
      if (rc != MSB_ENOTFUSED) return rc;
    }
  }
  if (cudaMemcpyAsync(x_dev, x_host, bytes, cudaMemcpyHostToDevice, st) != cudaSuccess) return MSB_ECUDA;
  rc = block_common(x_dev, batch, router_t, records, sketch, alpha, k, 0, 0.f, lr_a, lr_b, out_dev,
                    dims, workspace, workspace_bytes, nullptr, flags, stream);
  if (rc != MSB_OK) return rc;
  if (cudaMemcpyAsync(out_host, out_dev, bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return MSB_ECUDA;
  return MSB_OK;
}

int32_t moe_sparse_block_threshold(const void* x, int32_t batch, const void* router_t,
                                   const void* records, const uint32_t* sketch,
                                   const float* alpha, float tau, const void* lr_a,
                                   const void* lr_b, void* out, const msb_dims* dims,
                                   void* workspace, size_t workspace_bytes,
                                   const msb_trace* trace, void* stream) {
  if (!sketch || !alpha) return MSB_EINVAL;
  return block_common(x, batch, router_t, records, sketch, alpha, 1, 1, tau, lr_a, lr_b, out,
                      dims, workspace, workspace_bytes, trace, MSB_FLAG_GENERAL, stream);
}

int32_t msb_path_info(const msb_dims* dims, int32_t batch, int32_t k, uint32_t flags,
                      int32_t* info) {
  int rc = check_dims(dims);
  if (rc != MSB_OK) return rc;
  if (!info || batch < 1 || k < 1 || k > dims->inter) return MSB_EINVAL;
  if (batch > MSB_MAX_BATCH) return MSB_EUNSUPPORTED;
  rc = ensure_setup();
  if (rc != MSB_OK) return rc;
  const Dims D = to_dims(*dims);
  int p[6];
  fused_plan_info(D, k, batch, p);
  const bool fused = batch <= single_launch_max_batch(D, (flags & MSB_FLAG_SINGLE) != 0, false) &&
                     !(flags & MSB_FLAG_GENERAL) && fused_supported(D, k);
  info[0] = fused ? 1 : 2;
  for (int i = 0; i < 6; ++i) info[1 + i] = p[i];
  info[7] = 0;
  return MSB_OK;
}

#ifdef MSB_INSTRUMENTED
// Instrumented build only (libmsb_instr.so): per-CTA %globaltimer marks of the
// single-launch kernel's phases go to `marks` (device, [grid][16] u64; slot 15 = the
// SM the CTA ran on), or nowhere when NULL.
int32_t msb_debug_set_marks(void* marks) {
  debug_ctl().marks = static_cast<unsigned long long*>(marks);
  return MSB_OK;
}

// Instrumented build only: skip = 1 makes the single-launch kernel's first CTA withhold
// its first record copy, skip = 2 makes the gather CTA of work item 0 withhold its first stage
// (0: neither); wait_ns replaces the 2-second limit of the bounded waits (0: restore it).
// A withheld copy is never issued, so the wait for it runs out: the call is flagged
// (msb_check: MSB_ETIMEOUT) and its output is undefined.
int32_t msb_debug_inject(uint32_t skip, uint64_t wait_ns) {
  if (skip > 2u) return MSB_EINVAL;
  debug_ctl().skip = skip;
  debug_ctl().wait_ns = wait_ns;
  return MSB_OK;
}
#endif

int32_t msb_residual_rmsnorm(float* h, const void* y, void* x_next, int32_t batch, int32_t d,
                             float eps, void* stream) {
  if (!h || !x_next || batch < 1 || d < 64 || d % 64 != 0 || !(eps >= 0.f)) return MSB_EINVAL;
  if (batch > MSB_MAX_BATCH || d > MSB_MAX_D) return MSB_EUNSUPPORTED;
  if (!aligned16(h) || !aligned16(x_next) || (y && !aligned16(y))) return MSB_EINVAL;
  return launch_residual_rmsnorm(h, static_cast<const uint16_t*>(y),
                                 static_cast<uint16_t*>(x_next), batch, d, eps,
                                 static_cast<cudaStream_t>(stream));
}

}  // extern "C"
