/*
 * thrift_debug.h -- test-only entry point of libthrift.  Not needed to use the library.
 */
#ifndef THRIFT_DEBUG_H
#define THRIFT_DEBUG_H

#include "thrift.h"

#ifdef __cplusplus
extern "C" {
#endif

/* thrift_attn_fwd, plus a dump of one entry (key block visit) of the first unit processed by
 * CTA 0 (batch 0, query head 0, last query tile) into `dbg` (device float):
 *   [0, 128*block_k)                        raw S = Q K^T of the entry as the MMA left it in TMEM
 *                                           (no softmax scale, no tensor scales), row-major
 *   [128*block_k, 128*block_k + 64*block_k) per row, block_k*2 bytes: the PV operand row as
 *                                           written to shared memory (FP16 probabilities, or
 *                                           NVFP4 codes followed by the row's E4M3 scale bytes)
 *   then 128*d floats                       raw PV product of the entry, row-major
 * `dbg_entry` is the entry index within the unit (NVFP4 entries first, then FP16 entries). */
thrift_status thrift_debug_attn_dump(const void* q, const void* k, const void* v,
                                     const thrift_nvfp4* q4, const thrift_nvfp4* k4,
                                     const thrift_nvfp4* v4, const uint32_t* mask, void* out,
                                     float* lse, const thrift_cfg* cfg, void* ws,
                                     size_t ws_bytes, float* dbg, int32_t dbg_entry,
                                     void* stream);

#ifdef __cplusplus
}
#endif

#endif /* THRIFT_DEBUG_H */
