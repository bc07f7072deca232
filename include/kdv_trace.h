/*
 * kdv_trace.h -- stage timeline of the tensor-core verify kernel (tracing
 * build only).
 *
 * libkdv_trace.so is libkdv.so compiled with -DKDV_TRACE: it exports the
 * same entry points, computes the same bits, and in addition every CTA of
 * the verify kernel writes the GPU's global nanosecond timer
 * (%globaltimer) at fixed pipeline stages into a device array of
 * KDV_TRACE_CTAS x KDV_TRACE_SLOTS 64-bit words (CTA c, stage s at word
 * c * KDV_TRACE_SLOTS + s; CTA c belongs to work item c / 4, and CTAs 0-1 of
 * an item are its S pair, 2-3 its O pair). A stage a CTA does not reach, and
 * every CTA of a launch past KDV_TRACE_CTAS, leaves its word untouched. The
 * stamps cost a few global stores per CTA; the product library has none of
 * this code. For studying the pipeline, not for production.
 */
#ifndef KDV_TRACE_H_
#define KDV_TRACE_H_

#include "kdv.h"

#ifdef __cplusplus
extern "C" {
#endif

#define KDV_TRACE_CTAS 1024
#define KDV_TRACE_SLOTS 16

/* Stages (slot numbers). S = S-pair CTA, O = O-pair CTA. */
enum {
  KDV_TRACE_SETUP = 0,         /* all: barriers, TMEM and cluster set up     */
  KDV_TRACE_S_MMA_T0 = 1,      /* S leader: QK^T MMAs of S tile 0 issued      */
  KDV_TRACE_S_MMA_T1 = 2,      /* S leader: QK^T MMAs of S tile 1 issued      */
  KDV_TRACE_S_MMA_LAST = 3,    /* S leader: QK^T MMAs of the last tile issued */
  KDV_TRACE_SM0_T0_READY = 4,  /* S: softmax warpgroup 0 sees S tile 0        */
  KDV_TRACE_SM0_T0_DONE = 5,   /* S: warpgroup 0 has pushed tile 0's P        */
  KDV_TRACE_SM0_DONE = 6,      /* S: warpgroup 0 has pushed its last P        */
  KDV_TRACE_SM1_DONE = 7,      /* S: warpgroup 1 has pushed its last P        */
  KDV_TRACE_V_READY = 8,       /* O: V producer may read the fp16 rows        */
  KDV_TRACE_PV_T0 = 9,         /* O leader: P.V MMAs of P tile 0 issued       */
  KDV_TRACE_PV_LAST = 10,      /* O leader: P.V MMAs of the last P tile issued */
  KDV_TRACE_O_P0 = 11,         /* O: rescale warps see P tile 0               */
  KDV_TRACE_EPILOGUE = 12,     /* O: the last P.V is done, epilogue starts    */
  KDV_TRACE_STORED = 13,       /* O: every epilogue store issued              */
  KDV_TRACE_TEARDOWN = 14      /* all: teardown starts                        */
};

/* Zero the stamp array (asynchronously on `stream`). */
KDV_API kdv_status kdv_trace_clear(void* stream);

/* Copy the first n_words words of the stamp array to host memory
 * (synchronous; n_words in [0, KDV_TRACE_CTAS * KDV_TRACE_SLOTS]). */
KDV_API kdv_status kdv_trace_read(uint64_t* host_dst, int64_t n_words);

#ifdef __cplusplus
}
#endif

#endif  /* KDV_TRACE_H_ */
