/*
 * fa_profiling.h — a profiling hook of libfa.so, kept out of fa.h: nothing in
 * the attention API needs it. It times the backward's main kernel alone, for
 * benchmarks that report that kernel against the tensor-core roofline.
 */
#ifndef FA_PROFILING_H_
#define FA_PROFILING_H_

#include "fa.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * fa_bwd_time_main_pass — ev_begin and ev_end are cudaEvent_t handles created
 * by the caller (both non-NULL, or both NULL to cancel). The next fa_bwd,
 * fa_bwd_dropout or fa_bwd_varlen call made by this host thread records
 * ev_begin on its stream right before its main pass (the kernel that runs the
 * five products) and ev_end right after it, so cudaEventElapsedTime gives that
 * kernel's duration without the amax, conversion and D/L passes. The pair is
 * used by one call only; the state is per host thread.
 * Errors: FA_ERR_INVALID_ARG when exactly one handle is NULL.
 */
FA_API fa_status fa_bwd_time_main_pass(void* ev_begin, void* ev_end);

#ifdef __cplusplus
}
#endif

#endif /* FA_PROFILING_H_ */
