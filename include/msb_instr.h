/*
 * msb_instr.h -- entry points of the instrumented build of the library only
 * (libmsb_instr.so: the same sources compiled with MSB_INSTRUMENTED).  The product
 * library libmsb.so does not export them.  They have no counterpart on the source
 * pages: they serve profiling and the tests of the kernels' failure handling.
 */
#ifndef MSB_INSTR_H_
#define MSB_INSTR_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Phase timeline of the single-launch (batch-1) kernel: every launch made after this
 * call writes, per CTA, the %globaltimer value (ns) at each phase boundary into
 * `marks` (device memory, uint64 [grid][16]; slot 15 holds the SM the CTA ran on).
 * The pointer is captured at launch time (also into CUDA graphs).  NULL: no marks.
 * Returns MSB_OK. */
int32_t msb_debug_set_marks(void* marks);

/* Failure injection for tests.  skip = 1: the single-launch kernel's first CTA never
 * issues its first record copy; skip = 2: the multi-kernel gather's CTA that takes
 * work item 0 never issues its first stage; 0: neither.  The copy is simply not
 * issued (no bad address, no fault), so the bounded wait for it runs out: the call is
 * flagged (msb_check: MSB_ETIMEOUT), its output is undefined, and the workspace is
 * ready for the next call.  wait_ns replaces the 2-second limit of the bounded waits
 * (0: the product's limit).  Applies to launches made after the call.  Returns
 * MSB_OK, or MSB_EINVAL for skip > 2. */
int32_t msb_debug_inject(uint32_t skip, uint64_t wait_ns);

#ifdef __cplusplus
}
#endif

#endif /* MSB_INSTR_H_ */
