// Offline packer (host only): model-layout BF16 weights -> the layout the kernels read.
//
// Built from the weights alone, with no calibration data ("KAIST drops
// calibration from MoE decoding ...", "A reader built from weights alone"):
//  * the ternary sketch of every W_gate row at 2 bits per weight, with the
//    ternarisation of Ternary Weight Networks (Li, Zhang, Liu 2016):
//    T_i = sign(W_i) * [|W_i| > 0.7 * mean|W|], alpha = mean |W_i| over kept i;
//  * one contiguous channel record per (expert, channel): gate row | up row |
//    down column, so a selected channel is one 6d-byte read;
//  * the router transposed to one contiguous row per expert.
// The 4-bit variant (msb_pack_q4, format in msb_q4.h) stores each record's three
// vectors as group-wise affine 4-bit codes ("MoE top_k override (--moe-top-k)",
// "Combinaison avec d'autres optimisations": the override composes with 4-bit
// checkpoints) and sketches the dequantised gate rows.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <functional>
#include <thread>
#include <vector>

#include "msb.h"
#include "msb_prep.h"
#include "msb_q4.h"

namespace {

inline float bf16_value(uint16_t b) {
  const uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// 2-bit code of a ternary value: bit 1 = sign, bit 0 = magnitude.
inline uint32_t code_of(int t) { return t > 0 ? 1u : (t < 0 ? 3u : 0u); }

// Ternary sketch of one row w[0..d): writes T (-1/0/1) and returns alpha.
// |w| > 0.7 * sum|w| / d is evaluated as 10 * d * |w| > 7 * sum|w| in double; for
// BF16 rows (and dequantised 4-bit rows of ordinary range) both sides are exact.
float ternary_row(const double* w, int d, int8_t* t) {
  double sum = 0.0;
  for (int i = 0; i < d; ++i) sum += std::fabs(w[i]);
  const double rhs = 7.0 * sum;
  double kept_sum = 0.0;
  int n_kept = 0;
  for (int i = 0; i < d; ++i) {
    const double a = std::fabs(w[i]);
    t[i] = 0;
    if (10.0 * (double)d * a > rhs) {
      t[i] = w[i] > 0 ? 1 : -1;
      kept_sum += a;
      ++n_kept;
    }
  }
  return n_kept ? (float)(kept_sum / (double)n_kept) : 0.0f;
}

// Sketch and alpha of expert e from its gate rows (row(j, buf) fills buf[0..d) with
// row j as doubles): tensor-core tile order [tile][chunk][lane][h], 8 column pairs
// per word; rows I..Ipad-1 are zero codes with alpha 0.
void pack_sketch(int e, const msb_dims& m, const std::function<void(int, double*)>& row,
                 uint32_t* sketch, float* alpha) {
  const int d = m.d, I = m.inter;
  const int ipad = (I + 15) & ~15;
  const int KC = d / 64;
  std::vector<int8_t> t((size_t)ipad * d, 0);
  std::vector<double> w(d);
  for (int j = 0; j < I; ++j) {
    row(j, w.data());
    alpha[(size_t)e * ipad + j] = ternary_row(w.data(), d, t.data() + (size_t)j * d);
  }
  for (int j = I; j < ipad; ++j) alpha[(size_t)e * ipad + j] = 0.0f;

  const int ntiles = ipad / 16;
  for (int rt = 0; rt < ntiles; ++rt)
    for (int kc = 0; kc < KC; ++kc) {
      uint32_t* out = sketch + (((size_t)e * ntiles + rt) * KC + kc) * 64;
      for (int lane = 0; lane < 32; ++lane) {
        const int gg = lane >> 2, c = lane & 3;
        for (int h = 0; h < 2; ++h) {
          const int r = rt * 16 + gg + 8 * h;
          const int8_t* tr = t.data() + (size_t)r * d;
          uint32_t word = 0;
          for (int q = 0; q < 8; ++q) {
            const int sq = q >> 1, p = q & 1;
            const int col = kc * 64 + 16 * sq + 2 * c + 8 * p;
            word |= code_of(tr[col]) << (14 - 2 * q);
            word |= code_of(tr[col + 1]) << (30 - 2 * q);
          }
          out[lane * 2 + h] = word;
        }
      }
    }
}

void pack_expert(int e, const uint16_t* gate, const uint16_t* up, const uint16_t* down,
                 const msb_dims& m, uint16_t* records, uint32_t* sketch, float* alpha) {
  const int d = m.d, I = m.inter;
  const uint16_t* g = gate + (size_t)e * I * d;
  const uint16_t* u = up + (size_t)e * I * d;
  const uint16_t* dn = down + (size_t)e * d * I;

  // channel records
  for (int j = 0; j < I; ++j) {
    uint16_t* rec = records + ((size_t)e * I + j) * 3 * d;
    std::memcpy(rec, g + (size_t)j * d, 2 * (size_t)d);
    std::memcpy(rec + d, u + (size_t)j * d, 2 * (size_t)d);
    for (int i = 0; i < d; ++i) rec[2 * d + i] = dn[(size_t)i * I + j];
  }
  pack_sketch(e, m, [&](int j, double* w) {
    for (int i = 0; i < d; ++i) w[i] = (double)bf16_value(g[(size_t)j * d + i]);
  }, sketch, alpha);
}

// ---------------------------------------------------------------- 4-bit records

// Nearest BF16 of a double (ties to even), as its bit pattern.  Finite values in
// BF16's normal range: the value is rounded to 8 significant bits, which a float
// holds exactly, so the pattern is the float's upper half.
uint16_t bf16_nearest(double v) {
  if (v == 0.0) return 0;
  int ex;
  const double m = std::frexp(v, &ex);  // v = m * 2^ex, 0.5 <= |m| < 1
  const float f = (float)std::ldexp(std::nearbyint(m * 256.0) / 256.0, ex);
  uint32_t bits;
  std::memcpy(&bits, &f, 4);
  return (uint16_t)(bits >> 16);
}

size_t q4_record_bytes(int d) {
  const size_t raw = (size_t)3 * d / 2 + (size_t)3 * (d / MSB_Q4_GROUP) * 4;
  return (raw + 15) / 16 * 16;
}

// Quantise w[0..d) group by group (rule in msb_q4.h): nibble codes into codes[0..d/2),
// (scale, bias) BF16 pairs into params[0..2*d/64), the dequantised weights into deq.
void quantize_vector(const double* w, int d, uint8_t* codes, uint16_t* params, double* deq) {
  constexpr int G = MSB_Q4_GROUP;
  for (int g0 = 0; g0 < d; g0 += G) {
    double lo = w[g0], hi = w[g0];
    for (int i = g0 + 1; i < g0 + G; ++i) {
      lo = std::min(lo, w[i]);
      hi = std::max(hi, w[i]);
    }
    const uint16_t b_bits = bf16_nearest(lo), s_bits = bf16_nearest((hi - lo) / 15.0);
    const double b = (double)bf16_value(b_bits), s = (double)bf16_value(s_bits);
    params[2 * (g0 / G)] = s_bits;
    params[2 * (g0 / G) + 1] = b_bits;
    for (int i = g0; i < g0 + G; ++i) {
      const double t = s > 0.0 ? (w[i] - b) / s : 0.0;
      const int q = (int)std::min(15.0, std::max(0.0, std::nearbyint(t)));
      deq[i] = s * q + b;
      if (i & 1)
        codes[i >> 1] = (uint8_t)(codes[i >> 1] | (q << 4));
      else
        codes[i >> 1] = (uint8_t)q;
    }
  }
}

void pack_expert_q4(int e, const uint16_t* gate, const uint16_t* up, const uint16_t* down,
                    const msb_dims& m, uint8_t* records, uint32_t* sketch, float* alpha) {
  const int d = m.d, I = m.inter;
  const size_t rb = q4_record_bytes(d);
  const int npar = 2 * (d / MSB_Q4_GROUP);  // BF16 values per vector's (scale, bias) list
  const uint16_t* g = gate + (size_t)e * I * d;
  const uint16_t* u = up + (size_t)e * I * d;
  const uint16_t* dn = down + (size_t)e * d * I;
  std::vector<double> w(d), deq(d), gate_deq((size_t)I * d);
  std::vector<uint16_t> params(3 * (size_t)npar);

  for (int j = 0; j < I; ++j) {
    uint8_t* rec = records + ((size_t)e * I + j) * rb;
    std::memset(rec, 0, rb);
    for (int i = 0; i < d; ++i) w[i] = (double)bf16_value(g[(size_t)j * d + i]);
    quantize_vector(w.data(), d, rec, params.data(), gate_deq.data() + (size_t)j * d);
    for (int i = 0; i < d; ++i) w[i] = (double)bf16_value(u[(size_t)j * d + i]);
    quantize_vector(w.data(), d, rec + d / 2, params.data() + npar, deq.data());
    for (int i = 0; i < d; ++i) w[i] = (double)bf16_value(dn[(size_t)i * I + j]);
    quantize_vector(w.data(), d, rec + d, params.data() + 2 * npar, deq.data());
    std::memcpy(rec + (size_t)3 * d / 2, params.data(), params.size() * 2);
  }
  pack_sketch(e, m, [&](int j, double* out) {
    std::memcpy(out, gate_deq.data() + (size_t)j * d, (size_t)d * sizeof(double));
  }, sketch, alpha);
}

// Sizes the packers accept: those for which msb_sketch_words / msb_alpha_count give the
// output sizes (a 0 there would leave the caller with empty buffers).
int32_t check_pack_dims(const msb_dims* dims) {
  const msb_dims& m = *dims;
  if (m.d < 64 || m.d % 64 != 0 || m.inter < 1 || m.experts < 1) return MSB_EINVAL;
  if (m.d > MSB_MAX_D || m.inter > MSB_MAX_INTER || m.experts > MSB_MAX_EXPERTS)
    return MSB_EUNSUPPORTED;
  if (msb_sketch_words(dims) == 0 || msb_alpha_count(dims) == 0) return MSB_EINVAL;
  return MSB_OK;
}

void transpose_router(const uint16_t* router_host, const msb_dims& m, uint16_t* router_t_host) {
  for (int e = 0; e < m.experts; ++e)
    for (int i = 0; i < m.d; ++i) router_t_host[(size_t)e * m.d + i] = router_host[(size_t)i * m.experts + e];
}

// Runs fn(e) for every expert on up to `threads` host threads (<= 0: all).
void for_each_expert(int experts, int threads, const std::function<void(int)>& fn) {
  int nt = threads > 0 ? threads : (int)std::thread::hardware_concurrency();
  nt = std::max(1, std::min(nt, experts));
  std::vector<std::thread> pool;
  for (int w = 0; w < nt; ++w)
    pool.emplace_back([&, w]() {
      for (int e = w; e < experts; e += nt) fn(e);
    });
  for (auto& th : pool) th.join();
}

}  // namespace

extern "C" int32_t msb_pack(const uint16_t* gate_host, const uint16_t* up_host,
                            const uint16_t* down_host, const uint16_t* router_host,
                            const msb_dims* dims, uint16_t* records_host, uint32_t* sketch_host,
                            float* alpha_host, uint16_t* router_t_host, int32_t threads) {
  if (!dims || !gate_host || !up_host || !down_host || !router_host || !records_host ||
      !sketch_host || !alpha_host || !router_t_host)
    return MSB_EINVAL;
  if (const int32_t rc = check_pack_dims(dims)) return rc;
  const msb_dims m = *dims;
  transpose_router(router_host, m, router_t_host);
  for_each_expert(m.experts, threads, [&](int e) {
    pack_expert(e, gate_host, up_host, down_host, m, records_host, sketch_host, alpha_host);
  });
  return MSB_OK;
}

extern "C" int32_t msb_ternary_rows(const float* w_host, int32_t rows, int32_t d, int8_t* t_host,
                                    float* alpha_host) {
  if (!w_host || !t_host || !alpha_host || rows < 1 || d < 1) return MSB_EINVAL;
  std::vector<double> w((size_t)d);
  for (int j = 0; j < rows; ++j) {
    for (int i = 0; i < d; ++i) w[i] = w_host[(size_t)j * d + i];
    alpha_host[j] = ternary_row(w.data(), d, t_host + (size_t)j * d);
  }
  return MSB_OK;
}

extern "C" size_t msb_q4_record_bytes(const msb_dims* dims) {
  if (!dims || dims->d < 64 || dims->d % 64 != 0 || dims->d > MSB_MAX_D) return 0;
  return q4_record_bytes(dims->d);
}

extern "C" int32_t msb_pack_q4(const uint16_t* gate_host, const uint16_t* up_host,
                               const uint16_t* down_host, const uint16_t* router_host,
                               const msb_dims* dims, uint8_t* records_host, uint32_t* sketch_host,
                               float* alpha_host, uint16_t* router_t_host, int32_t threads) {
  if (!dims || !gate_host || !up_host || !down_host || !router_host || !records_host ||
      !sketch_host || !alpha_host || !router_t_host)
    return MSB_EINVAL;
  if (const int32_t rc = check_pack_dims(dims)) return rc;
  const msb_dims m = *dims;
  transpose_router(router_host, m, router_t_host);
  for_each_expert(m.experts, threads, [&](int e) {
    pack_expert_q4(e, gate_host, up_host, down_host, m, records_host, sketch_host, alpha_host);
  });
  return MSB_OK;
}
