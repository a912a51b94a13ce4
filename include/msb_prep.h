/*
 * msb_prep.h -- host-side weight-preparation helpers of libmsb (no CUDA).
 *
 * "KAIST drops calibration from MoE decoding ...", section "A reader built from
 * weights alone": everything the block reads is derived from the weights.  The
 * packer's sketch rule is exported on its own here so that offline preparation
 * (the weight-derived low-rank compensation factors, which estimate what the
 * top-k selection leaves out) selects channels with exactly the block's sketch.
 */
#ifndef MSB_PREP_H_
#define MSB_PREP_H_

#include <stdint.h>

#include "msb.h"

#ifdef __cplusplus
extern "C" {
#endif

/* The ternary sketch of `rows` rows of length d, by the rule msb_pack applies to each
 * W_gate row: T_i = sign(W_i) * [|W_i| > 0.7 * mean|W|] (strict; evaluated exactly as
 * 10*d*|W_i| > 7*sum|W| in double precision) and alpha = mean |W_i| over the kept
 * entries (0 if none), rounded to float.
 *  w_host      float32 [rows][d], row-major, host memory.
 *  t_host      int8 [rows][d] out: -1, 0 or 1.
 *  alpha_host  float32 [rows] out.
 * Returns MSB_OK, or MSB_EINVAL for a null pointer, rows < 1 or d < 1 (nothing
 * written). */
int32_t msb_ternary_rows(const float* w_host, int32_t rows, int32_t d, int8_t* t_host,
                         float* alpha_host);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* MSB_PREP_H_ */
