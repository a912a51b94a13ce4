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
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

#include "msb.h"

namespace {

inline float bf16_value(uint16_t b) {
  const uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// 2-bit code of a ternary value: bit 1 = sign, bit 0 = magnitude.
inline uint32_t code_of(int t) { return t > 0 ? 1u : (t < 0 ? 3u : 0u); }

void pack_expert(int e, const uint16_t* gate, const uint16_t* up, const uint16_t* down,
                 const msb_dims& m, uint16_t* records, uint32_t* sketch, float* alpha) {
  const int d = m.d, I = m.inter;
  const int ipad = (I + 15) & ~15;
  const int KC = d / 64;
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

  // ternary sketch, row by row
  std::vector<int8_t> t((size_t)ipad * d, 0);
  for (int j = 0; j < I; ++j) {
    const uint16_t* row = g + (size_t)j * d;
    double sum = 0.0;
    for (int i = 0; i < d; ++i) sum += std::fabs((double)bf16_value(row[i]));
    const double rhs = 7.0 * sum;
    double kept_sum = 0.0;
    int n_kept = 0;
    for (int i = 0; i < d; ++i) {
      const double w = (double)bf16_value(row[i]);
      const double a = std::fabs(w);
      // |w| > 0.7 * sum / d, evaluated exactly as 10 * d * |w| > 7 * sum
      if (10.0 * (double)d * a > rhs) {
        t[(size_t)j * d + i] = w > 0 ? 1 : -1;
        kept_sum += a;
        ++n_kept;
      }
    }
    alpha[(size_t)e * ipad + j] = n_kept ? (float)(kept_sum / (double)n_kept) : 0.0f;
  }
  for (int j = I; j < ipad; ++j) alpha[(size_t)e * ipad + j] = 0.0f;

  // tensor-core tile order: [tile][chunk][lane][h], 8 column pairs per word
  const int ntiles = ipad / 16;
  for (int rt = 0; rt < ntiles; ++rt)
    for (int kc = 0; kc < KC; ++kc) {
      uint32_t* out = sketch + (((size_t)e * ntiles + rt) * KC + kc) * 64;
      for (int lane = 0; lane < 32; ++lane) {
        const int gg = lane >> 2, c = lane & 3;
        for (int h = 0; h < 2; ++h) {
          const int row = rt * 16 + gg + 8 * h;
          const int8_t* tr = t.data() + (size_t)row * d;
          uint32_t w = 0;
          for (int q = 0; q < 8; ++q) {
            const int s = q >> 1, p = q & 1;
            const int col = kc * 64 + 16 * s + 2 * c + 8 * p;
            w |= code_of(tr[col]) << (14 - 2 * q);
            w |= code_of(tr[col + 1]) << (30 - 2 * q);
          }
          out[lane * 2 + h] = w;
        }
      }
    }
}

}  // namespace

extern "C" int32_t msb_pack(const uint16_t* gate_host, const uint16_t* up_host,
                            const uint16_t* down_host, const uint16_t* router_host,
                            const msb_dims* dims, uint16_t* records_host, uint32_t* sketch_host,
                            float* alpha_host, uint16_t* router_t_host, int32_t threads) {
  if (!dims || !gate_host || !up_host || !down_host || !router_host || !records_host ||
      !sketch_host || !alpha_host || !router_t_host)
    return MSB_EINVAL;
  const msb_dims m = *dims;
  if (m.d < 64 || m.d % 64 != 0 || m.inter < 1 || m.experts < 1) return MSB_EINVAL;
  if (m.d > MSB_MAX_D || m.inter > MSB_MAX_INTER || m.experts > MSB_MAX_EXPERTS)
    return MSB_EUNSUPPORTED;
  for (int e = 0; e < m.experts; ++e)
    for (int i = 0; i < m.d; ++i) router_t_host[(size_t)e * m.d + i] = router_host[(size_t)i * m.experts + e];
  int nt = threads > 0 ? threads : (int)std::thread::hardware_concurrency();
  nt = std::max(1, std::min(nt, m.experts));
  std::vector<std::thread> pool;
  for (int w = 0; w < nt; ++w)
    pool.emplace_back([&, w]() {
      for (int e = w; e < m.experts; e += nt)
        pack_expert(e, gate_host, up_host, down_host, m, records_host, sketch_host, alpha_host);
    });
  for (auto& th : pool) th.join();
  return MSB_OK;
}
