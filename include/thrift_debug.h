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

/* The attention kernel's 2^x on device, for accuracy tests: y[i] = 2^x[i] for n elements by the
 * FMA-pipe polynomial the softmax uses for part of its exponentials (which = 0) or by the MUFU
 * approximation (which = 1).  x, y: device float arrays. */
thrift_status thrift_debug_ex2(const float* x, float* y, int64_t n, int32_t which, void* stream);

/* Measured pipe rates for the attention kernel's elementwise bound (bench and tests only):
 * out (device double[2]) receives the lanes of ex2.approx.f32 (MUFU) and of fma.rn.f32 (FMA pipe)
 * completed per SM clock, measured by one 512-thread CTA per SM running eight independent
 * dependency chains per thread.  ws: 256-byte aligned device workspace of at least
 * thrift_debug_pipe_rates_ws_bytes() bytes (its status header is left alone).  Three launches
 * on `stream`; nothing is synchronised. */
size_t thrift_debug_pipe_rates_ws_bytes(void);
thrift_status thrift_debug_pipe_rates(void* ws, size_t ws_bytes, double* out, void* stream);

/* 1 when the library was built with in-kernel bounds checks (libthrift_checked.so: every index
 * that selects a tile, list entry or mask word is checked before use), else 0. */
int32_t thrift_debug_checks_enabled(void);

/* Runs one in-kernel check that fails when `fail` is non-zero.  In the checked build a failing
 * check records THRIFT_ERR_CHECK in the workspace status word (and skips nothing else); in the
 * regular build checks are compiled out and the status stays 0. */
thrift_status thrift_debug_check(void* ws, int32_t fail, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* THRIFT_DEBUG_H */
