/*
 * blasst_measure.h -- measurement-only entry points of libblasst.so.  They are
 * not part of the attention API in blasst.h and exist to take apart what a
 * production call costs.  Conventions (pointers, layouts, streams, errors) are
 * those of blasst.h.
 */
#ifndef BLASST_MEASURE_H
#define BLASST_MEASURE_H

#include "blasst.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * blasst_prefill with the skip decision compiled out: the same kernel, tiles,
 * pipeline and epilogue, but no per-warp vote, no tile-wide AND and no
 * published decision; every visited block is kept (lambda is checked as in
 * blasst_prefill and then not used; the mask reads all zeros and the count 0).
 * Timed against blasst_prefill at lambda = 0, where both compute the same
 * dense result, it gives the cost of taking the decision.  The pages put that
 * cost at 0.96-1.00x of the dense kernel's speed (xllm-io paper review, section
 * 4 "core innovations" and the key findings under Table 5).
 */
BLASST_API blasst_status blasst_measure_prefill_novote(const void *q, const void *k, const void *v, void *o,
                                                       float *lse, int B, int Hq, int Hkv, int Lq, int Lk, int d,
                                                       float scale, float lambda, int causal, uint32_t *skip_mask,
                                                       unsigned long long *skip_count, void *stream,
                                                       const blasst_opts *opts);

#ifdef __cplusplus
}
#endif

#endif /* BLASST_MEASURE_H */
