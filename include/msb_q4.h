/*
 * msb_q4.h -- 4-bit channel records for libmsb (host packer).
 *
 * "MoE top_k override (--moe-top-k)", section "Combinaison avec d'autres
 * optimisations": the expert-count override composes with 4-bit (and 3-bit)
 * quantised checkpoints of the same model, so the channels the block gathers may
 * be held at 4 bits instead of BF16 (3.56x fewer record bytes at d = 2048).  The
 * page does not give the checkpoints' format; the one packed here is group-wise
 * affine 4-bit:
 *
 *   every run of MSB_Q4_GROUP = 64 consecutive weights of a gate row, an up row or
 *   a down column has a BF16 scale s and a BF16 bias b, every weight a code q in
 *   0..15, and the weight the block computes with is s * q + b.
 *
 * Quantisation of one group of BF16 weights w (all arithmetic in double):
 *   b = min w;  s = (max w - min w) / 15 rounded to the nearest BF16 (ties to even);
 *   q = (w - b) / s rounded to the nearest integer (ties to even), clamped to 0..15;
 *   q = 0 for every weight of a constant group (s = 0).
 * Down columns are grouped along d, so that one channel's record is self-contained
 * (a checkpoint grouped along I is re-quantised from its dequantised values).
 *
 * Record of channel (e, j), msb_q4_record_bytes(dims) bytes, 16-byte aligned:
 *   bytes [0, d/2)      codes of gate row j: byte i holds element 2i in bits 0-3 and
 *                       element 2i+1 in bits 4-7
 *   bytes [d/2, d)      codes of up row j, same order
 *   bytes [d, 3d/2)     codes of down column j (element i = W_down[i][j]), same order
 *   then 3 * d/64 (scale, bias) pairs of BF16 bit patterns, 4 bytes per pair: the gate
 *   row's groups 0 .. d/64 - 1, then the up row's, then the down column's;
 *   zero bytes up to the record size (a multiple of 16).
 * records [E][I][msb_q4_record_bytes(dims)] bytes.
 *
 * The sketch of a 4-bit layer is the ternary sketch of its dequantised gate rows, in
 * the format and with the rule of msb_pack (msb.h); router_t as msb_pack.
 *
 * moe_sparse_block_q4 runs the block on such records; the weights it computes with are
 * the dequantised s * q + b (scores from the sketch of the dequantised gate rows).
 */
#ifndef MSB_Q4_H_
#define MSB_Q4_H_

#include <stddef.h>
#include <stdint.h>

#include "msb.h"

#ifdef __cplusplus
extern "C" {
#endif

#define MSB_Q4_GROUP 64

/* Bytes of one 4-bit channel record for dims->d; 0 if dims is NULL or d is not a
 * multiple of 64 in 64..MSB_MAX_D. */
size_t msb_q4_record_bytes(const msb_dims* dims);

/* Offline 4-bit packer, host memory only (no CUDA).  Inputs in model layout, as
 * msb_pack: gate_host, up_host bf16 [E][I][d]; down_host bf16 [E][d][I];
 * router_host bf16 [d][E].  Outputs (caller-allocated host buffers): records_host
 * E * I * msb_q4_record_bytes(dims) bytes; sketch_host (msb_sketch_words) and
 * alpha_host (msb_alpha_count) of the dequantised gate rows; router_t_host [E][d].
 * Uses up to `threads` host threads (<= 0: all hardware threads).
 * Returns MSB_OK, MSB_EINVAL (null pointer, d not a multiple of 64, I or E < 1) or
 * MSB_EUNSUPPORTED (sizes above MSB_MAX_D / MSB_MAX_INTER / MSB_MAX_EXPERTS). */
int32_t msb_pack_q4(const uint16_t* gate_host, const uint16_t* up_host, const uint16_t* down_host,
                    const uint16_t* router_host, const msb_dims* dims, uint8_t* records_host,
                    uint32_t* sketch_host, float* alpha_host, uint16_t* router_t_host,
                    int32_t threads);

/* The block of moe_sparse_block (msb.h: same arguments, same result, same workspace)
 * on 4-bit channel records: records_q4 is the records array of msb_pack_q4 (device,
 * 16-byte aligned), sketch and alpha those msb_pack_q4 wrote for the dequantised gate
 * rows; router_t and the low-rank factors as msb_pack / moe_sparse_block.  Runs on the
 * single-launch kernel only (batches up to 16 tokens whose shapes fit its plan): it
 * gathers 3 d / 2 + 12 d / 64 bytes per channel (rounded up to 16) instead of 6 d, and
 * forms gate.x per group of 64 weights as s * (q . x) + b * sum(x) in FP32.  Returns
 * MSB_EUNSUPPORTED where the single launch declines (more than 16 tokens, a batch trace
 * that asks for union counts, MSB_FLAG_GENERAL, shapes beyond its plan); other errors
 * as moe_sparse_block. */
int32_t moe_sparse_block_q4(const void* x, int32_t batch, const void* router_t, const void* records_q4,
                            const uint32_t* sketch, const float* alpha, int32_t k, const void* lr_a,
                            const void* lr_b, void* out, const msb_dims* dims, void* workspace,
                            size_t workspace_bytes, const msb_trace* trace, uint32_t flags,
                            void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MSB_Q4_H_ */
