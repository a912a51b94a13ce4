/* The C ABI from plain C (C99): both headers compile as C, the library links, and the
 * host-only entry points behave as the headers state.  No CUDA call is made: argument
 * errors are detected before anything is enqueued, and the packers are host code.
 * Exit status 0 on success; the first failed check is printed. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "msb.h"
#include "msb_prep.h"
#include "msb_q4.h"

#define CHECK(cond)                                                  \
  do {                                                               \
    if (!(cond)) {                                                   \
      fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__, __LINE__, #cond); \
      return 1;                                                      \
    }                                                                \
  } while (0)

static uint16_t bf16_of(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

int main(void) {
  const msb_dims dims = {64, 40, 4, 2, 0, 1};
  const msb_dims bad_k = {64, 40, 2, 3, 0, 1}; /* more routed experts than experts */
  const msb_dims bad_d = {96, 40, 4, 2, 0, 1}; /* d not a multiple of 64 */

  /* sizes */
  CHECK(msb_sketch_words(&dims) == (size_t)4 * 48 * 64 / 16);
  CHECK(msb_alpha_count(&dims) == (size_t)4 * 48);
  CHECK(msb_sketch_words(&bad_k) == 0 && msb_sketch_words(&bad_d) == 0);
  CHECK(msb_q4_record_bytes(&dims) == 112 && msb_q4_record_bytes(&bad_d) == 0);
  CHECK(msb_workspace_size(&dims, 1) > 0 && msb_workspace_size(&dims, 0) == 0 &&
        msb_workspace_size(&dims, MSB_MAX_BATCH + 1) == 0);
  CHECK(strcmp(msb_strerror(MSB_OK), "ok") == 0);
  CHECK(strcmp(msb_strerror(12345), "unknown status") == 0);

  /* the packers on a small deterministic layer */
  const size_t ne = (size_t)4 * 40 * 64;
  uint16_t* gate = malloc(ne * 2);
  uint16_t* up = malloc(ne * 2);
  uint16_t* down = malloc(ne * 2);
  uint16_t* router = malloc((size_t)64 * 4 * 2);
  uint16_t* rec = malloc(ne * 3 * 2);
  uint8_t* rec4 = malloc((size_t)4 * 40 * 112);
  uint32_t* sketch = malloc(msb_sketch_words(&dims) * 4);
  float* alpha = malloc(msb_alpha_count(&dims) * 4);
  uint16_t* router_t = malloc((size_t)4 * 64 * 2);
  CHECK(gate && up && down && router && rec && rec4 && sketch && alpha && router_t);
  for (size_t i = 0; i < ne; ++i) {
    gate[i] = bf16_of((float)((int)(i * 7919u % 201u) - 100) / 1000.0f);
    up[i] = bf16_of((float)((int)(i * 104729u % 199u) - 99) / 1000.0f);
    down[i] = bf16_of((float)((int)(i * 1299709u % 197u) - 98) / 1000.0f);
  }
  for (size_t i = 0; i < (size_t)64 * 4; ++i) router[i] = bf16_of((float)i / 256.0f);

  CHECK(msb_pack(gate, up, down, router, &dims, rec, sketch, alpha, router_t, 2) == MSB_OK);
  /* record of (e, j) = gate row j | up row j | down column j */
  for (int e = 0; e < 4; ++e)
    for (int j = 0; j < 40; ++j) {
      const uint16_t* r = rec + ((size_t)e * 40 + j) * 192;
      CHECK(memcmp(r, gate + ((size_t)e * 40 + j) * 64, 128) == 0);
      CHECK(memcmp(r + 64, up + ((size_t)e * 40 + j) * 64, 128) == 0);
      for (int i = 0; i < 64; ++i) CHECK(r[128 + i] == down[(size_t)e * 64 * 40 + (size_t)i * 40 + j]);
    }
  for (int e = 0; e < 4; ++e)
    for (int i = 0; i < 64; ++i) CHECK(router_t[e * 64 + i] == router[i * 4 + e]);
  for (int e = 0; e < 4; ++e)
    for (int j = 40; j < 48; ++j) CHECK(alpha[e * 48 + j] == 0.0f);

  CHECK(msb_pack_q4(gate, up, down, router, &dims, rec4, sketch, alpha, router_t, 1) == MSB_OK);
  for (size_t i = 0; i < (size_t)4 * 40; ++i)
    for (int b = 3 * 64 / 2 + 3 * 4; b < 112; ++b) CHECK(rec4[i * 112 + b] == 0); /* padding */

  /* argument errors, before anything is written or enqueued */
  CHECK(msb_pack(NULL, up, down, router, &dims, rec, sketch, alpha, router_t, 1) == MSB_EINVAL);
  CHECK(msb_pack(gate, up, down, router, &bad_k, rec, sketch, alpha, router_t, 1) == MSB_EINVAL);
  CHECK(msb_pack_q4(gate, up, down, router, &bad_d, rec4, sketch, alpha, router_t, 1) == MSB_EINVAL);
  CHECK(moe_sparse_block(NULL, 1, NULL, NULL, NULL, NULL, 8, NULL, NULL, NULL, &dims, NULL, 0,
                         NULL, 0, NULL) == MSB_EINVAL);
  CHECK(msb_check(NULL, NULL) == MSB_EINVAL);

  free(gate); free(up); free(down); free(router); free(rec); free(rec4);
  free(sketch); free(alpha); free(router_t);
  {  /* the packer's ternarisation on its own: |w| > 0.7 mean|w| keeps 1 and -1 (2 and -2) */
    const float w[8] = {1.0f, -1.0f, 0.1f, 0.0f, 2.0f, -2.0f, 0.2f, 0.0f};
    int8_t t[8];
    float a[2];
    CHECK(msb_ternary_rows(w, 2, 4, t, a) == MSB_OK);
    CHECK(t[0] == 1 && t[1] == -1 && t[2] == 0 && t[3] == 0 && a[0] == 1.0f);
    CHECK(t[4] == 1 && t[5] == -1 && t[6] == 0 && t[7] == 0 && a[1] == 2.0f);
    CHECK(msb_ternary_rows(NULL, 2, 4, t, a) == MSB_EINVAL);
    CHECK(msb_ternary_rows(w, 0, 4, t, a) == MSB_EINVAL);
  }
  printf("c abi ok\n");
  return 0;
}
