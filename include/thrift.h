/*
 * thrift.h -- C ABI of libthrift: selective mixed-precision (NVFP4 + FP16) attention
 * forward on NVIDIA B200 (sm_100a).
 *
 * The method (ThriftAttention technical summary, gist.science 2605.23081, section
 * "Methodologie"; the same text in the French version, "Méthodologie : ThriftAttention"):
 *   1. Q, K and V are split into blocks; every (query block i, key block j) pair gets the
 *      importance score S^_ij = qbar_i . kbar_j, the dot product of the blocks' token means.
 *   2. The k highest-scoring pairs (per batch and query head here) run in FP16; all other
 *      pairs run in NVFP4 (E2M1 values, one E4M3 scale per 16 elements, one FP32 tensor
 *      scale).
 *   3. Both paths merge through one online softmax; the FP4 path quantises its probability
 *      blocks with a two-level scheme (a per-row scale per key block, then the 16-element
 *      E4M3 micro-scale).
 *
 * Conventions for every entry point:
 *   - Pointers named "device" point to GPU memory; all such memory is owned by the caller.
 *     The library never allocates, never frees and never synchronises the device, except
 *     thrift_get_device_status, which copies one word to the host and waits for it.
 *   - `stream` is a cudaStream_t passed as void*; NULL is the legacy default stream.  All
 *     work is enqueued on it, in call order.
 *   - Argument errors are detected on the host, return a status and launch nothing.
 *     Errors that only the device can see (a bounded wait that ran out) are recorded in a
 *     status word inside the workspace and read with thrift_get_device_status.
 *   - Tensors are dense and row-major.  FP16 means IEEE binary16.
 *   - Every tensor pointer (FP16 inputs and outputs, NVFP4 buffers) must be 16-byte aligned;
 *     a misaligned one is rejected with THRIFT_ERR_INVALID_ARG.
 */
#ifndef THRIFT_H
#define THRIFT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  THRIFT_OK = 0,
  THRIFT_ERR_INVALID_ARG = 1,  /* null pointer, bad size or inconsistent configuration */
  THRIFT_ERR_UNSUPPORTED = 2,  /* valid but outside what the kernels implement */
  THRIFT_ERR_CUDA = 3,         /* a CUDA runtime call or kernel launch failed */
  THRIFT_ERR_TIMEOUT = 4,      /* device status only: a bounded wait inside a kernel ran out */
  THRIFT_ERR_WORKSPACE = 5,    /* workspace pointer null, misaligned or too small */
  THRIFT_ERR_CHECK = 8         /* device status only, checked build (libthrift_checked): an in-kernel
                                  bounds check failed; the access was skipped and the kernel unwound.
                                  The device status word is the bitwise OR of the device-side errors
                                  seen (THRIFT_ERR_TIMEOUT, THRIFT_ERR_CHECK). */
} thrift_status;

/* Problem description, passed by value-pointer; the library keeps no copy. */
typedef struct {
  int32_t B, Hq, Hkv, N, d;  /* batch, query heads, key/value heads (Hq % Hkv == 0),
                                sequence length (queries = keys), head dim (64 or 128) */
  int32_t causal;            /* 0 or 1: key t is visible to query r when t <= r */
  int32_t block_q, block_k;  /* selection block sizes: block_q in {64,128}, block_k in {64,128};
                                N must be a multiple of 128 and of block_k */
  int32_t topk_abs;          /* >= 0: number of FP16 pairs per (batch, query head);
                                -1: use topk_bp */
  int32_t topk_bp;           /* budget in basis points of the valid pairs: k = ceil(bp*V/10000)
                                (0 = uniform NVFP4 attention, 10000 = all pairs in FP16) */
  float softmax_scale;       /* tau; 0 selects 1/sqrt(d) rounded to FP32 */
} thrift_cfg;

/* Strides of an FP16 tensor viewed as [B, H, N, d] (batch, head, token, channel), in elements;
 * the d channels of a token row are contiguous.  The dense layout is {H*N*d, N*d, d}; a tensor
 * stored token-major as [B, N, H, d] (the usual output of a fused QKV projection) has
 * {N*H*d, d, H*d}.  Every stride must be a non-negative multiple of 8 (16 bytes: the rows are
 * moved by tensor copies) and n >= d; an output's rows must not overlap.  Entry points that take
 * strides accept NULL for the dense layout.  NVFP4 copies, masks, lists, scores and lse are
 * always dense. */
typedef struct {
  int64_t b, h, n;
} thrift_strides;

/* NVFP4 tensor view.  All pointers are device pointers owned by the caller.
 * For an FP16 tensor viewed as [outer, N, d]:
 *   group_axis 0 (Q, K): 16-element groups along d.
 *       codes  [outer*N, d/2]   E2M1 nibbles, element 2t in the low nibble of byte t
 *       scales [outer*N, d/16]  E4M3 bytes, one per group (canonical layout)
 *   group_axis 1 (V):    16-element groups along N (tokens), stored transposed.
 *       codes  [outer*d, N/2], scales [outer*d, N/16]
 *   scales_mma: the same scale bytes in the layout the tensor cores read (rows in blocks of
 *       128, groups in blocks of 4 = 64 elements; each 128x4 block is 512 contiguous bytes,
 *       row r, group g at (r%32)*16 + ((r%128)/32)*4 + g%4; blocks ordered row-block major).
 *       Size: thrift_nvfp4_scales_mma_bytes().
 *   tensor_scale: one device float = amax|X| / 2688 (1 for an all-zero tensor). */
typedef struct {
  uint8_t* codes;
  uint8_t* scales;
  uint8_t* scales_mma;
  float* tensor_scale;
  int32_t group_axis;
} thrift_nvfp4;

/* Bytes of the scales_mma buffer of a tensor viewed as [outer, N, d] with this group axis. */
size_t thrift_nvfp4_scales_mma_bytes(int64_t outer, int32_t N, int32_t d, int32_t group_axis);

/* Workspace bytes the calls below need for this configuration (the maximum over
 * thrift_quantize_nvfp4, thrift_block_select, thrift_attn_fwd).  thrift_attn_fwd_auto needs
 * thrift_auto_workspace_bytes() instead.  The workspace must be 256-byte aligned device
 * memory; its first 256 bytes hold the device status word and must be zeroed once before
 * first use (thrift_reset_device_status does that). */
size_t thrift_workspace_bytes(const thrift_cfg* cfg);

/* NVFP4 quantisation (ThriftAttention "FP4-pad": the NVFP4 microscaling format).
 * x: device FP16 [outer, N, d].  Writes codes, scales, scales_mma and tensor_scale of *out
 * (group_axis taken from out->group_axis).  Per 16-element group: s_b = E4M3(amax16/6/s_t),
 * codes = E2M1(x / (s_b * s_t)), all roundings to nearest even with saturation.
 * Requirements: d in {64,128}; N % 128 == 0; outer >= 1.  Two kernels: a grid amax
 * reduction into the workspace, then the encode pass. */
thrift_status thrift_quantize_nvfp4(const void* x, int64_t outer, int32_t N, int32_t d,
                                    const thrift_nvfp4* out, void* ws, size_t ws_bytes,
                                    void* stream);

/* thrift_quantize_nvfp4 of a strided [B, H, N, d] tensor (outer = B * H); the codes and scales
 * are written in the dense layouts above.  Errors as thrift_quantize_nvfp4, plus
 * THRIFT_ERR_INVALID_ARG for bad strides and THRIFT_ERR_UNSUPPORTED for B * H > 65535. */
thrift_status thrift_quantize_nvfp4_strided(const void* x, const thrift_strides* xs, int32_t B,
                                            int32_t H, int32_t N, int32_t d,
                                            const thrift_nvfp4* out, void* ws, size_t ws_bytes,
                                            void* stream);

/* Block selection (ThriftAttention "Heuristische Blokkenselectie").
 * q: device FP16 [B,Hq,N,d]; k: device FP16 [B,Hkv,N,d].
 * Outputs (device):
 *   mask   [B,Hq,nQb,ceil(nKb/32)] u32: bit j%32 of word j/32 set when pair (i,j) is FP16
 *   counts [B,Hq,nQb] i32: selected pairs in query block i
 *   lists  [B,Hq,nQb,nKb] i16: the selected key blocks of query block i in ascending order
 *          (entries past counts[i] are -1)
 *   scores [B,Hq,nQb,nKb] float64 (may be NULL): S^_ij, -inf for causal-invalid pairs.
 * nQb = N/block_q, nKb = N/block_k.  The means are exact FP16 sums in float64 divided by the
 * block size; S^ has no softmax scale; ties in S^ go to the smaller index i*nKb + j. */
thrift_status thrift_block_select(const void* q, const void* k, const thrift_cfg* cfg,
                                  uint32_t* mask, int32_t* counts, int16_t* lists,
                                  double* scores, void* ws, size_t ws_bytes, void* stream);

/* Block selection without any allocation, for callers that cannot allocate device memory:
 * hosts that own every byte of device memory through their own allocator and hand the library
 * only input and output buffers, or latency-bound callers that must not allocate (or grow a
 * workspace) while a request is in flight.  The paper has no counterpart of this entry point.
 * Same inputs, outputs and results as thrift_block_select, but the scratch (block means and the
 * score matrix) lives in a fixed device array inside the library: 16 MiB, held by every GPU that
 * loads the library until the process exits.  A configuration whose thrift_workspace_bytes()
 * exceeds 16 MiB + 256 needs more scratch than that and is rejected with THRIFT_ERR_WORKSPACE
 * before anything is launched.  The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call before any stream
 * capture.  It calls no cudaMalloc or cudaFree and no allocating library routine.  All calls
 * share the one array and the scratch contents of a call are overwritten by the next; calls
 * that overlap on the GPU (different streams, different host threads) race on it. */
thrift_status thrift_block_select_noalloc(const void* q, const void* k, const thrift_cfg* cfg,
                                          uint32_t* mask, int32_t* counts, int16_t* lists,
                                          double* scores, void* stream);

/* thrift_block_select with strided q [B,Hq,N,d] and k [B,Hkv,N,d] views (qs, ks; NULL = dense). */
thrift_status thrift_block_select_strided(const void* q, const thrift_strides* qs, const void* k,
                                          const thrift_strides* ks, const thrift_cfg* cfg,
                                          uint32_t* mask, int32_t* counts, int16_t* lists,
                                          double* scores, void* ws, size_t ws_bytes, void* stream);

/* Attention forward (ThriftAttention "Gemengd-Precisie Berekening & Samenvoeging").
 * q, k, v: device FP16 [B,Hq,N,d], [B,Hkv,N,d], [B,Hkv,N,d] (used for the FP16 pairs);
 * q4, k4 (group_axis 0) and v4 (group_axis 1): NVFP4 copies (used for the other pairs);
 * mask: the selection bitmask of thrift_block_select.  Only the mask is read: the kernel builds
 * each query tile's key-block list from it.  counts and lists are accepted for symmetry with
 * thrift_block_select's outputs, are not read, and may be NULL.
 * out: device FP16 [B,Hq,N,d]; lse: device float [B,Hq,N] (natural log of the softmax
 * denominator of the tau-scaled scores; may be NULL).
 * topk_bp == 0 (or topk_abs == 0): uniform NVFP4; q, k, v, mask, counts, lists may be NULL.
 * topk_bp == 10000: every valid pair in FP16; q4, k4, v4 may be NULL.
 * One persistent kernel: tcgen05 block-scaled FP4 and FP16 MMAs with TMEM accumulators,
 * TMA-staged tiles, the probability blocks re-quantised per row and key block. */
thrift_status thrift_attn_fwd(const void* q, const void* k, const void* v,
                              const thrift_nvfp4* q4, const thrift_nvfp4* k4,
                              const thrift_nvfp4* v4, const uint32_t* mask,
                              const int32_t* counts, const int16_t* lists, void* out,
                              float* lse, const thrift_cfg* cfg, void* ws, size_t ws_bytes,
                              void* stream);

/* Attn-QAT forward variant of thrift_attn_fwd (Attn-QAT technical summary, "2. Methodik: Attn-QAT",
 * second principle: the forward pass also computes and stores a high-precision output O', used
 * only for the backward pass's scalar term).  Reading: O' is the FP32 O / l of the same
 * mixed-precision computation, written before the FP16 rounding of `out`; out is the FP16 round
 * to nearest even of out_hp element by element.  out_hp: device float [B,Hq,N,d] (required);
 * every other argument as thrift_attn_fwd (mask only; no counts or lists).  Same kernel, one
 * more epilogue store per output row. */
thrift_status thrift_attn_fwd_qat(const void* q, const void* k, const void* v,
                                  const thrift_nvfp4* q4, const thrift_nvfp4* k4,
                                  const thrift_nvfp4* v4, const uint32_t* mask, void* out,
                                  float* out_hp, float* lse, const thrift_cfg* cfg, void* ws,
                                  size_t ws_bytes, void* stream);

/* thrift_attn_fwd with strided FP16 operands and output: q, k, v and out are [B,H,N,d] views
 * with strides qs, ks, vs, os (NULL = dense); the FP16 tiles are fetched through 4-D tensor maps,
 * so the layout costs nothing in the kernel.  q4, k4, v4, mask and lse are dense.  Arguments and
 * errors otherwise as thrift_attn_fwd (mask only). */
thrift_status thrift_attn_fwd_strided(const void* q, const thrift_strides* qs, const void* k,
                                      const thrift_strides* ks, const void* v,
                                      const thrift_strides* vs, const thrift_nvfp4* q4,
                                      const thrift_nvfp4* k4, const thrift_nvfp4* v4,
                                      const uint32_t* mask, void* out, const thrift_strides* os,
                                      float* lse, const thrift_cfg* cfg, void* ws, size_t ws_bytes,
                                      void* stream);

/* thrift_attn_fwd with the other reading of the two-level P requantisation (ThriftAttention
 * "Methodologie", "Online Samenvoeging": the probability blocks get a two-level quantisation
 * adapted from SageAttention3, inside an online softmax).
 * thrift_attn_fwd takes each key block's own row maximum M as the first level: P^ = exp(S - M),
 * so every block's largest probability requantises at the top of the NVFP4 range.  Here the
 * first level is the row's running maximum m over the key blocks visited so far, in the kernel's
 * fixed order -- the NVFP4 blocks in ascending key-block index, then the FP16 blocks ascending:
 * m = max(m, M), P^ = exp(S - m), the E4M3 group scales of 2688 P^ and the E2M1 codes follow,
 * and the denominator adds the unquantised sum of P^.  A block below the running maximum thus
 * requantises with smaller group scales; the output depends on the visiting order and differs
 * from thrift_attn_fwd's by the requantisation error.  Arguments, requirements and errors as
 * thrift_attn_fwd (mask only; no counts or lists). */
thrift_status thrift_attn_fwd_running_max(const void* q, const void* k, const void* v,
                                          const thrift_nvfp4* q4, const thrift_nvfp4* k4,
                                          const thrift_nvfp4* v4, const uint32_t* mask, void* out,
                                          float* lse, const thrift_cfg* cfg, void* ws,
                                          size_t ws_bytes, void* stream);

/* Compute-matched sparse variant of thrift_attn_fwd (ThriftAttention compares against sparse
 * attention at a matched compute budget): only the selected pairs of `mask` run, in FP16 with the
 * FP16 q, k, v; every other pair is dropped as if masked.  A row left with no key gets output 0
 * and lse -inf.  No NVFP4 tensor is read; mask required; counts and lists may be NULL.  The same
 * fused kernel with an entry list of FP16 entries only. */
thrift_status thrift_attn_fwd_sparse(const void* q, const void* k, const void* v, const uint32_t* mask,
                                     const int32_t* counts, const int16_t* lists, void* out, float* lse,
                                     const thrift_cfg* cfg, void* ws, size_t ws_bytes, void* stream);

/* Workspace bytes of thrift_attn_fwd_auto (it also holds the NVFP4 copies and the selection). */
size_t thrift_auto_workspace_bytes(const thrift_cfg* cfg);

/* The whole path in one call: quantise Q, K, V, select, attend. */
thrift_status thrift_attn_fwd_auto(const void* q, const void* k, const void* v, void* out,
                                   float* lse, const thrift_cfg* cfg, void* ws,
                                   size_t ws_bytes, void* stream);

/* thrift_attn_fwd_auto with strided q, k, v and out ([B,H,N,d] views, NULL = dense): the whole
 * path reads the inputs and writes the output in their own layouts; the NVFP4 copies and the
 * selection in the workspace stay dense. */
thrift_status thrift_attn_fwd_auto_strided(const void* q, const thrift_strides* qs, const void* k,
                                           const thrift_strides* ks, const void* v,
                                           const thrift_strides* vs, void* out,
                                           const thrift_strides* os, float* lse,
                                           const thrift_cfg* cfg, void* ws, size_t ws_bytes,
                                           void* stream);

/* ------------------------------------------------------------------ decode
 *
 * Decode form of the same method (ThriftAttention technical summary, "Methodologie" for the
 * computation; "Resultaten" for its decode use against a KV cache held in FP16 and NVFP4).
 * A step has Nq new query rows per query head; they are the newest Nq positions of a cache of
 * Nk keys (the rows of this step already appended), so with causal = 1 key t is visible to
 * query row r (0-based among the Nq) when t <= Nk - Nq + r.  The Nq rows of a head form one
 * query block: selection picks the k key blocks with the largest qbar . kbar_j per (batch,
 * query head), qbar the mean of the Nq rows, k = topk_abs or ceil(topk_bp * nKb / 10000).
 * The query rows are quantised to NVFP4 as one tensor (their own FP32 tensor scale).  Every
 * other step -- NVFP4 scores on the other blocks, two-level re-quantisation of the probability
 * blocks, FP16 on the selected blocks, one softmax -- is the prefill computation.
 *
 * The cache: k, v FP16 [B,Hkv,Nk,d]; k4 = thrift_quantize_nvfp4(k, group_axis 0), v4 =
 * thrift_quantize_nvfp4(v, group_axis 1); kbar = thrift_kv_block_means(k).  All owned by the
 * caller and only read.  q, k, v and the NVFP4 codes, scales and scales_mma buffers must be
 * 16-byte aligned (they are copied with bulk/tensor copies).
 *
 * Errors (every decode entry point): THRIFT_ERR_INVALID_ARG for a null or misaligned pointer or
 * an inconsistent configuration, THRIFT_ERR_UNSUPPORTED outside the implemented sizes,
 * THRIFT_ERR_WORKSPACE for a null, misaligned or too small workspace -- all detected on the host
 * before anything is launched; a device-side wait that runs out is recorded in the workspace
 * status word (thrift_get_device_status). */
typedef struct {
  int32_t B, Hq, Hkv;  /* batch, query heads, key/value heads (Hq % Hkv == 0) */
  int32_t Nq;          /* query rows per head in this step, 1 <= Nq, (Hq/Hkv) * Nq <= 16 */
  int32_t Nk;          /* cache capacity (the layout's key count), a multiple of 128 and of block_k */
  int32_t d;           /* head dim, 64 or 128 */
  int32_t causal;      /* 0 or 1 (bottom-right aligned, see above) */
  int32_t block_k;     /* key block size, 64 or 128 */
  int32_t topk_abs;    /* >= 0: FP16 key blocks per (batch, query head); -1: use topk_bp */
  int32_t topk_bp;     /* budget in basis points of the nKb = Nk/block_k key blocks
                          (0 = every block NVFP4, 10000 = every block FP16) */
  float softmax_scale; /* tau; 0 selects 1/sqrt(d) rounded to FP32 */
  int32_t n_valid;     /* keys held by the cache, Nq <= n_valid <= Nk (any value); 0 means Nk.
                          Query row r is at position n_valid - Nq + r; keys at or past n_valid
                          are masked, key blocks starting at or past it are skipped and left
                          out of the budget (nKb above counts the blocks below n_valid).  The
                          cache beyond n_valid must hold finite values (thrift_kv_append keeps
                          it zero). */
} thrift_decode_cfg;

/* Block means of the cache's keys: kbar [outer, Nk/block_k, d] float64, the exact FP16 sum of
 * each column over the block's tokens divided by block_k (k: device FP16 [outer, Nk, d]).
 * Computed once per cache; thrift_decode_select reads it.  Requires d in {64,128}, block_k in
 * {64,128}, Nk a multiple of block_k. */
thrift_status thrift_kv_block_means(const void* k, int64_t outer, int32_t Nk, int32_t d, int32_t block_k,
                                    double* kbar, void* stream);

/* FP32 tensor scale of an FP16 array: tensor_scale (device float[1]) = amax|x| / 2688 (1 for an
 * all-zero array), the scale thrift_quantize_nvfp4 would use.  x: device FP16, n elements (n a
 * multiple of 8, 16-byte aligned).  ws: workspace of at least 256 bytes (its header's scratch
 * word is used).  Sets a double-cached KV cache's fixed scales from its first tokens (the
 * capacity buffers hold zeros past them, which leaves the amax unchanged). */
thrift_status thrift_nvfp4_tensor_scale(const void* x, int64_t n, float* tensor_scale, void* ws,
                                        size_t ws_bytes, void* stream);

/* Appending to the double-cached KV cache (ThriftAttention technical summary, "Betekenis en
 * Beweringen": the cache held in FP16 and NVFP4; reading R-append for the update rule).
 * The cache of `outer` = B*Hkv (batch, KV head) pairs has capacity Ncap keys and holds `len`:
 *   k, v          device FP16 [outer, Ncap, d], zero past the keys held (the caller zero-fills
 *                 them once; the library writes only positions below len + T);
 *   k4 / v4       their NVFP4 copies (group_axis 0 / 1, capacity layouts) whose tensor_scale
 *                 holds the cache's fixed scale;
 *   kbar          device float64 [outer, Ncap/block_k, d] key block means.
 * T new keys per pair: k_new, v_new device FP16 [outer, T, d] are copied to positions
 * [len, len + T) (either may be NULL when the caller already wrote them there).  Then: the new K
 * rows are encoded with k4's fixed tensor scale (groups along d); every 16-token V group that the
 * new keys touch is re-encoded from the FP16 cache with v4's fixed scale (groups along tokens;
 * the group's positions past len + T read zero); the means of the touched key blocks are
 * recomputed over the keys each holds (exact FP16 sums in float64 divided by the count).  The
 * result is bit for bit the NVFP4 quantisation, with the fixed scales, of the zero-padded cache
 * of len + T keys, whatever the sequence of appends.  Values above the build-time amax saturate
 * (E4M3 448, E2M1 6).  Requirements: d in {64,128}; block_k in {64,128}; Ncap a multiple of 128
 * and of block_k; 0 <= len, 1 <= T, len + T <= Ncap; 16-byte aligned buffers.  Five launches on
 * `stream`; decode the grown cache with thrift_decode_cfg.n_valid = len + T. */
thrift_status thrift_kv_append(const void* k_new, const void* v_new, int64_t outer, int32_t Ncap, int32_t d,
                               int32_t block_k, int32_t len, int32_t T, void* k, void* v,
                               const thrift_nvfp4* k4, const thrift_nvfp4* v4, double* kbar,
                               void* stream);

/* Workspace bytes of thrift_decode_select, thrift_decode_attn and thrift_decode_fwd (the
 * query rows' NVFP4 copy, the selection of thrift_decode_fwd and the splits' partial sums).
 * 0 for an unsupported configuration. */
size_t thrift_decode_workspace_bytes(const thrift_decode_cfg* cfg);

/* Decode selection.  q: device FP16 [B,Hq,Nq,d]; kbar: device [B,Hkv,nKb,d] float64.
 * Outputs (device): mask [B,Hq,ceil(nKb/32)] u32 (bit j%32 of word j/32: key block j in FP16),
 * counts [B,Hq] i32, lists [B,Hq,nKb] i16 (ascending, -1 past counts), scores [B,Hq,nKb]
 * float64 S^_j (may be NULL).  Ties in S^ go to the smaller j. */
thrift_status thrift_decode_select(const void* q, const double* kbar, const thrift_decode_cfg* cfg,
                                   uint32_t* mask, int32_t* counts, int16_t* lists, double* scores,
                                   void* ws, size_t ws_bytes, void* stream);

/* Decode attention.  q: device FP16 [B,Hq,Nq,d]; k, v: the FP16 cache (may be NULL when the
 * budget is 0); k4, v4: its NVFP4 copies (may be NULL when the budget is 10000); mask: the
 * selection of thrift_decode_select (may be NULL for budgets 0 and 10000).
 * out: device FP16 [B,Hq,Nq,d]; lse: device float [B,Hq,Nq] (may be NULL).
 * Launches: the query rows' NVFP4 quantisation, a split-over-key-blocks kernel (m16n8k16
 * tensor-core tiles, bulk/tensor copies into shared memory, bounded waits) and a kernel that
 * combines the splits. */
thrift_status thrift_decode_attn(const void* q, const void* k, const void* v, const thrift_nvfp4* k4,
                                 const thrift_nvfp4* v4, const uint32_t* mask, void* out, float* lse,
                                 const thrift_decode_cfg* cfg, void* ws, size_t ws_bytes, void* stream);

/* Compute-matched sparse variant of thrift_decode_attn (the baseline the pages compare against:
 * only the selected key blocks, in FP16, every other block dropped; a row left with no key gets
 * output 0 and lse -inf).  Same arguments without the NVFP4 cache; mask required. */
thrift_status thrift_decode_attn_sparse(const void* q, const void* k, const void* v, const uint32_t* mask,
                                        void* out, float* lse, const thrift_decode_cfg* cfg, void* ws,
                                        size_t ws_bytes, void* stream);

/* One decode step: thrift_decode_select (selection kept in the workspace), then
 * thrift_decode_attn. */
thrift_status thrift_decode_fwd(const void* q, const void* k, const void* v, const thrift_nvfp4* k4,
                                const thrift_nvfp4* v4, const double* kbar, void* out, float* lse,
                                const thrift_decode_cfg* cfg, void* ws, size_t ws_bytes, void* stream);

/* Zero the device status word at the start of the workspace (enqueued on stream). */
thrift_status thrift_reset_device_status(void* ws, void* stream);

/* Copy the device status word to *status_out (0 = no device-side error, otherwise a
 * thrift_status).  Synchronises `stream`. */
thrift_status thrift_get_device_status(const void* ws, void* stream, int32_t* status_out);

/* Launch a kernel whose mbarrier wait can never complete; its bounded wait gives up after
 * about `limit_cycles` SM clock cycles and records THRIFT_ERR_TIMEOUT in the status word.
 * Exists so that tests can check the timeout path without hanging a GPU. */
thrift_status thrift_debug_wait_timeout(void* ws, int64_t limit_cycles, void* stream);

/* Static string for a status code. */
const char* thrift_status_str(thrift_status s);

#ifdef __cplusplus
}
#endif

#endif /* THRIFT_H */
