/*
 * tq.h -- C ABI of libtq: TurboQuant-style KV-cache compression and decode attention over
 * the compressed cache, for one NVIDIA B200 (sm_100a).
 *
 * The method (web pages on TurboQuant):
 *   "Closing - The Three-Step Summary", Step 1 Rotate: a Walsh-Hadamard transform with
 *     random signs is applied to each K/V vector; it preserves inner products.
 *   Step 2 Quantize: each rotated coordinate gets a Lloyd-Max scalar code for the Gaussian,
 *     centroids scaled by 1/sqrt(d).
 *   Step 3 Correct: below 3 bits, (b-1)-bit codes plus a 1-bit QJL sketch of the residual
 *     (TurboQuant_prod); at 3+ bits, codes only (TurboQuant_mse).
 *   "What the Paper Doesn't Tell You", Finding 1: keys and values take separate bit-widths.
 *   "Where This Fits in the Inference Stack", TensorRT-LLM section: dequantisation happens
 *     inside the attention kernel, in registers, while K/V tiles stream from HBM.
 *   "Why the KV Cache Exists", What's in the KV Cache: per layer and KV head, K and V are
 *     [T x d] matrices; a decode query attends to all T cached tokens.
 *
 * Conventions shared by every entry point
 *   - Return: int status, TQ_OK (0) on success. On failure nothing is launched and
 *     tq_last_error() returns a message (thread-local; valid until the next failing call on
 *     the same thread). Size queries return 0 on invalid arguments.
 *   - Memory: every pointer is caller-owned. The library never allocates, frees or
 *     synchronises; device work is enqueued on the given stream (a cudaStream_t passed as
 *     void*, NULL = legacy default stream) and is asynchronous. Device pointers must be
 *     16-byte aligned. Host pointers have no alignment rule.
 *   - Shapes: d (head_dim) is a power of two in 16..256. Bit-widths are 1..4.
 *     qjl_m (QJL sketch length) is 0 (meaning d) or a multiple of 8 in 8..256.
 *   - Arrays are row-major and C-contiguous. The cache is token-major per (batch, KV head):
 *     element (b, h, t) of a cache array lives at index (b*Hkv + h)*T_cap + t.
 *   - GQA: query head hq reads KV head hq / (Hq/Hkv) (consecutive query heads share a KV
 *     head); Hq must be a multiple of Hkv.
 *   - Rotation: R x = H D x / sqrt(d), H the natural-order (Sylvester) Hadamard matrix,
 *     D = diag(+-1) with D_ii = -1 iff bit i of the SplitMix64(seed) stream is set (bit i%64
 *     of output i/64). One sign vector per cache, shared by K, V and the query.
 *   - Codes: code i of a record occupies bits [i*w, i*w+w) of a little-endian bit stream
 *     (stream bit k = bit k%8 of byte k/8); codes index the Lloyd-Max levels in ascending
 *     order; a coordinate exactly on a boundary takes the lower level. QJL bit j = 1 iff
 *     (S r)_j < 0.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TQ_OK 0
#define TQ_ERR_INVALID_ARG 1 /* null pointer, bad size or shape, misaligned pointer      */
#define TQ_ERR_UNSUPPORTED 2 /* d, bits, mode or qjl_m outside the supported set          */
#define TQ_ERR_WORKSPACE 3   /* workspace missing or smaller than the size query says      */
#define TQ_ERR_CUDA 4        /* a CUDA runtime call or kernel launch failed                */

#define TQ_MSE 0  /* TurboQuant_mse: b-bit Lloyd-Max codes                                  */
#define TQ_PROD 1 /* TurboQuant_prod: (b-1)-bit codes + 1-bit QJL residual sketch + ||r||   */
/* TurboQuant_mse records whose 4-bit codes live on Blackwell's FP4 (E2M1) grid instead of the
 * Lloyd-Max levels ("Where This Fits in the Inference Stack", Blackwell FP4: whether the
 * centroids map onto E2M1 is an open question there). Levels, ascending: s * (-6, -4, -3, -2,
 * -1.5, -1, -0.5, -0, +0, 0.5, 1, 1.5, 2, 3, 4, 6) on the N(0,1) scale of the rotated
 * coordinates (divided by sqrt(d) for a unit vector), s = 0.48708 the Gaussian-MSE-optimal
 * stretch; boundaries at the midpoints, 0 between the two zeros (a coordinate takes the zero
 * of its own sign). Code i is the level's index, as for TQ_MSE; its E2M1 bit pattern is
 * i - 8 for i >= 8 and 15 - i for i < 8. Gaussian MSE 0.01268, 1.335x the 4-bit Lloyd-Max
 * codebook's. bits must be 4; records are laid out as 4-bit TQ_MSE records. */
#define TQ_E2M1 2

#define TQ_F32 0
#define TQ_BF16 1
#define TQ_F16 2

/* Quantiser of one tensor (keys or values). */
typedef struct {
  int bits;  /* total bits per coordinate, 1..4                                          */
  int mode;  /* TQ_MSE, TQ_PROD ("Closing", Step 3: PROD is meant for bits <= 2) or TQ_E2M1 */
  int qjl_m; /* PROD only: QJL rows m (0 = d); ignored for TQ_MSE                          */
} tq_qcfg;

/* One layer's compressed KV cache. All pointers are device pointers owned by the caller.
 * Per (b, h, t) record, for each of K and V:
 *   codes  [B][Hkv][T_cap][tq_code_bytes]  uint8   Lloyd-Max codes (absent when 0 bits)
 *   norm   [B][Hkv][T_cap]                 uint16  IEEE fp16 bits of ||x||
 *   signs  [B][Hkv][T_cap][tq_sign_bytes]  uint8   PROD only: QJL sign bits, else NULL
 *   rnorm  [B][Hkv][T_cap]                 uint16  PROD only: fp16 ||r||, else NULL
 *   qjl    [m][d]                          float   PROD only: the projection S (fill it
 *                                                  with tq_make_qjl_matrix), else NULL  */
typedef struct {
  int B, Hkv, T_cap, d;
  uint64_t seed; /* rotation seed: fixed per model load, so records are reproducible    */
  tq_qcfg kc, vc;
  uint8_t *k_codes, *v_codes;
  uint16_t *k_norm, *v_norm;
  uint8_t *k_signs, *v_signs;
  uint16_t *k_rnorm, *v_rnorm;
  const float *k_qjl, *v_qjl;
} tq_cache;

/* A paged compressed KV cache (one layer): records live in pages of page_size positions
 * (a power of two, >= 16) drawn from a pool the caller manages; row b of the block table
 * maps sequence b's logical page j (positions [j page_size, (j+1) page_size)) to a physical
 * page. All pointers are device pointers owned by the caller. Per tensor:
 *   codes  [num_pages][Hkv][page_size][tq_code_bytes]  uint8   Lloyd-Max codes
 *   norm   [num_pages][Hkv][page_size]                 uint16  fp16 bits of ||x||
 *   signs  [num_pages][Hkv][page_size][tq_sign_bytes]  uint8   PROD only: QJL sign bits, else NULL
 *   rnorm  [num_pages][Hkv][page_size]                 uint16  PROD only: fp16 ||r||, else NULL
 *   qjl    [m][d]                                      float   PROD only: the projection S, else NULL
 *   block_table [B][max_pages]                         int32   physical page of each logical
 *                                                              page (entries in 0..num_pages-1)
 * Supported: head_dim 128 TurboQuant_mse keys and values (3/4-bit keys, 2..4-bit values for
 * decode), or head_dim 64 TurboQuant_prod keys and values with m = 64 (2-bit for decode);
 * writes take 16-bit input. A sequence may hold at most max_pages * page_size positions. */
typedef struct {
  int B, Hkv, d, page_size, num_pages, max_pages;
  uint64_t seed;
  tq_qcfg kc, vc;
  uint8_t *k_codes, *v_codes;
  uint16_t *k_norm, *v_norm;
  const int32_t *block_table;
  uint8_t *k_signs, *v_signs;
  uint16_t *k_rnorm, *v_rnorm;
  const float *k_qjl, *v_qjl;
} tq_paged_cache;

/* Message for the last failure on the calling thread ("" if none). */
const char *tq_last_error(void);

/* ---------------------------------------------------------------- host-side helpers */

/* Gaussian Lloyd-Max codebook for `bits` (1..4) at head dimension d ("Closing", Step 2):
 * writes 2^bits centroids (ascending) and 2^bits - 1 decision boundaries, both already
 * scaled by 1/sqrt(d) (the unit-norm vector's scale), into caller host arrays. Computed in
 * double by alternating the midpoint and conditional-mean conditions to a 1e-13 fixed
 * point. Errors: TQ_ERR_UNSUPPORTED, TQ_ERR_INVALID_ARG (null outputs). */
int tq_make_codebook(int bits, int d, float *centroids, float *bounds);

/* The rotation's sign vector as d bits (d/8 bytes, host): bit i set means D_ii = -1.
 * 16 bytes at d = 128 ("What the Paper Doesn't Tell You", Finding 4). */
int tq_make_signs(uint64_t seed, int d, uint8_t *signs);

/* QJL projection S [m][d] (host, row-major float32), i.i.d. N(0,1): entries 2k, 2k+1 are
 * the Box-Muller pair of the SplitMix64(seed) uniforms u = (word >> 11) * 2^-53 numbered
 * 2k, 2k+1 (rho = sqrt(-2 ln(1-u_2k)), theta = 2 pi u_2k+1), computed in double and rounded
 * to float32. m*d must be even; m, d in the supported ranges ("Closing", Step 3). */
int tq_make_qjl_matrix(uint64_t seed, int m, int d, float *S);

/* Bytes per vector: packed codes (d * Lloyd-Max bits / 8), QJL sign bytes (m/8 in PROD,
 * else 0), and the whole stored record (codes + signs + 2-byte norm [+ 2-byte rnorm]).
 * At d = 128 a 3-bit MSE record is 50 bytes ("Finding 3": 5.12x vs fp16). 0 if invalid. */
size_t tq_code_bytes(int d, tq_qcfg c);
size_t tq_sign_bytes(int d, tq_qcfg c);
size_t tq_record_bytes(int d, tq_qcfg c);

/* ---------------------------------------------------------------- device entry points */

/* Quantise-on-write ("Closing", Steps 1-3). K and V are device arrays [B][Hkv][T][d] of
 * `dtype` (TQ_F32 / TQ_BF16 / TQ_F16); either may be NULL to write only the other. Token t
 * is stored at cache position t_offset + t (0 <= t_offset, t_offset + T <= T_cap). T = 0
 * is a no-op. Per vector: n = ||x|| (fp32, stored fp16, rounded to nearest: a norm of 65520
 * or more is stored as +inf, and attention over such a record is not finite); z = H D x / n;
 * codes by the boundary count (fp32 decisions); PROD: r = (z - c[code]) / sqrt(d),
 * rnorm = ||r||, QJL bits of S r. A zero vector stores norm 0 (its reconstruction is 0). */
int tq_quantize_kv(const void *K, const void *V, int dtype, int T, int t_offset,
                   const tq_cache *cache, void *stream);

/* Workspace bytes tq_decode_attention needs for this shape (split-K partials: running
 * max, running sum and the rotated-domain accumulator per split and query head). The pages
 * place the attention over the compressed cache in the decode step ("Where This Fits in the
 * Inference Stack", TensorRT-LLM section: flash-decoding splits the context); the partial
 * records of those splits live in this caller-owned workspace, since the library never
 * allocates. B is the batch, Hq the query heads, T_len the attended positions. 0 if
 * invalid. Depends on the current device's SM count. The plain sizes come first and the
 * cache last (rather than the cache before T_len): B must equal cache->B, and the call reads
 * only the cache's shape and bit widths. */
size_t tq_decode_workspace_bytes(int B, int Hq, int T_len, const tq_cache *cache);

/* Decode attention over cache positions [0, T_len) of every (b, KV head) ("Where This
 * Fits", TensorRT-LLM section: dequantise in registers inside the attention kernel).
 * q [B][Hq][d] of `dtype`; out [B][Hq][d] float32; scale is the softmax scale (e.g.
 * 1/sqrt(d)). The query is rotated once (q~ = scale H D q / d), so that
 * scale q.k_hat = ||k|| sum_i q~_i c[code_i] (+ the QJL term); split-K online softmax;
 * values accumulate in the rotated domain; one inverse rotation per output. Arithmetic of
 * the d = 128 MSE configurations: scores on int8 tensor cores from 16-bit fixed-point
 * centroids and 24-bit fixed-point queries (int32 sums, exact up to the centroids' 16-bit
 * rounding), softmax in fp32, P.V with fp16 weights (times ||v||) and fp32 accumulation; the
 * output stays within 2e-3 relative L2 of exact attention over the dequantised cache, keys
 * at 50x the values' norm included. Needs T_len >= 1 and ws_bytes >=
 * tq_decode_workspace_bytes(...). Errors as above plus TQ_ERR_WORKSPACE. */
int tq_decode_attention(const void *q, int dtype, int Hq, int T_len, float scale,
                        const tq_cache *cache, float *out, void *ws, size_t ws_bytes,
                        void *stream);

/* Decode attention without a workspace and without any allocation. The pages have no
 * counterpart to this call; it exists for callers that cannot allocate device memory at this
 * point: runtimes that hand out all device memory from their own pool and forbid a library
 * to call cudaMalloc, decode loops that cannot afford cudaMalloc/cudaFree (they can stall
 * the whole device), and plugin interfaces that pass a kernel only its inputs and outputs.
 * Arguments, results and errors are those of tq_decode_attention; q, out and the cache stay
 * caller-owned. The split-K partials live in one fixed 8 MiB device array inside libtq
 * (present on every GPU that loads the library, until the process exits); a shape whose
 * tq_decode_workspace_bytes exceeds 8 MiB is rejected with TQ_ERR_WORKSPACE and nothing is
 * launched. The first call on a device looks up the array's device address (a host-side
 * symbol lookup) with that device current. Every call on a device shares the
 * same array and leaves its partials behind; a call writes every element it later reads, so
 * nothing needs clearing, but calls that overlap on the GPU (other streams, other host
 * threads) race on the array and must be serialised by the caller. The looked-up address is
 * kept for the life of the process: after a reset of the device (cudaDeviceReset, or another
 * library destroying the primary context) the array may move, and this call must not be used
 * on that device again. */
int tq_decode_attention_noalloc(const void *q, int dtype, int Hq, int T_len, float scale,
                                const tq_cache *cache, float *out, void *stream);

/* Ragged decode (the sequences of one batch have different context lengths): like
 * tq_decode_attention, but sequence b attends to its first T_lens[b] cached
 * positions. T_lens is a HOST array of B = cache->B ints, each in 1..T_cap; it is read during
 * the call only (the lengths travel to the kernels as launch parameters, so a captured graph
 * keeps the values of the capture). The work is split evenly over the ragged (sequence, KV
 * head, 16-token tile) space. Supported for the tensor-core configurations: d = 128 with MSE
 * keys of 3/4 bits, MSE values of 2..4 bits and at most 8 query heads per KV head, and d = 64
 * with 2-bit TurboQuant_prod keys and values of 64 sketch rows and 1 or 2 query heads per KV
 * head; B <= 512; other configurations return TQ_ERR_UNSUPPORTED. Workspace size from
 * tq_decode_varlen_workspace_bytes (0 on invalid arguments). Errors as tq_decode_attention.
 * This extends the pages' decode ("Where This Fits in the Inference Stack": real serving
 * batches sequences of different lengths). */
size_t tq_decode_varlen_workspace_bytes(int Hq, const tq_cache *cache, const int *T_lens);
int tq_decode_attention_varlen(const void *q, int dtype, int Hq, const int *T_lens, float scale,
                               const tq_cache *cache, float *out, void *ws, size_t ws_bytes,
                               void *stream);

/* How many kernels tq_quantize_kv (K and V both given, `dtype` input, T new positions) and
 * tq_decode_attention (Hq query heads over T_len positions) launch for this cache on the
 * current device. The pages have no counterpart to this call; benchmarks use it to count the
 * library's launches. Writes *quantize_launches and *decode_launches (either may be NULL);
 * returns TQ_OK, or the error the two calls would return for these arguments. */
int tq_launch_counts(const tq_cache *cache, int dtype, int T, int Hq, int T_len,
                     int *quantize_launches, int *decode_launches);

/* Dequantise cache positions [0, T_len) of K (which = 0) or V (which = 1) into out
 * [B][Hkv][T_len][d] of `dtype` (TQ_F32 / TQ_BF16 / TQ_F16, device, caller-owned) in the
 * original domain: x_hat = n D H c / d (MSE), plus the QJL residual estimate
 * sqrt(d) gamma sqrt(pi/2)/m S^T s inside the bracket (PROD). This is the reconstruction
 * the pages describe ("Closing - The Three-Step Summary", Steps 1-3: look up the centroids,
 * undo the rotation, scale by the stored norm; Step 3 adds the QJL correction). Errors:
 * TQ_ERR_INVALID_ARG (which not 0/1, dtype unknown, T_len outside 0..T_cap, null or
 * misaligned out), TQ_ERR_CUDA. T_len = 0 is a no-op. */
int tq_dequantize(const tq_cache *cache, int which, int T_len, void *out, int dtype,
                  void *stream);

/* Same split-K design over an unquantised bf16 cache: K, V [B][Hkv][T_cap][d] bf16
 * (positions [0, T_len) are read), q [B][Hq][d] bf16, out [B][Hq][d] float32. The
 * comparator for the compressed kernel and the path for layers kept at full precision
 * ("What the Paper Doesn't Tell You", Finding 1: boundary layers). */
size_t tq_decode_bf16_workspace_bytes(int B, int Hq, int Hkv, int T_len, int d);
int tq_decode_attention_bf16(const void *q, int Hq, const void *K, const void *V, int B,
                             int Hkv, int T_cap, int T_len, int d, float scale, float *out,
                             void *ws, size_t ws_bytes, void *stream);

/* Paged counterparts of tq_quantize_kv and tq_decode_attention_varlen: the same
 * computation, with record (b, h, t) at page block_table[b][t / page_size], head h, slot
 * t % page_size. tq_quantize_kv_paged takes 16-bit K, V [B][Hkv][T][d] and writes positions
 * t_offset .. t_offset + T - 1 of every sequence (their pages must be mapped). The decode takes
 * per-sequence lengths (host array, 1..max_pages * page_size). Errors: TQ_ERR_INVALID_ARG
 * (shapes, pointers, page size, lengths), TQ_ERR_UNSUPPORTED (other d, modes or dtypes),
 * TQ_ERR_WORKSPACE, TQ_ERR_CUDA; nothing is launched on error. The block-table entries are
 * read by the kernels and must be valid page indices. These extend the pages' decode
 * ("Where This Fits in the Inference Stack": PagedAttention allocates the cache this way). */
int tq_quantize_kv_paged(const void *K, const void *V, int dtype, int T, int t_offset,
                         const tq_paged_cache *cache, void *stream);
size_t tq_decode_paged_workspace_bytes(int Hq, const tq_paged_cache *cache, const int *T_lens);
int tq_decode_attention_paged(const void *q, int dtype, int Hq, const int *T_lens, float scale,
                              const tq_paged_cache *cache, float *out, void *ws, size_t ws_bytes,
                              void *stream);

/* Prefill (chunked) attention over the compressed cache ("Where This Fits in the Inference
 * Stack", Decode Throughput vs. Time to First Token: at long contexts the attention of prefill
 * reads the compressed cache as well; TensorRT-LLM section: chunked attention). A chunk of Lq
 * queries q [B][Lq][Hq][d] of `dtype` at positions t0 .. t0 + Lq - 1 (their own keys and values
 * already written to the cache, e.g. by tq_quantize_kv with t_offset = t0) attends causally:
 * query i of sequence b and query head hq reads cache positions 0 .. t0 + i of KV head
 * hq / (Hq / Hkv). out [B][Lq][Hq][d] float32 (device, caller-owned). The arithmetic is that
 * of the decode call (scores from 16-bit fixed-point centroids and 24-bit fixed-point queries
 * on int8 tensor cores, softmax in fp32, P.V with fp16 weights times ||v|| and fp32
 * accumulation). Keys on the E2M1 grid (TQ_E2M1) enter the score MMAs as E2M1 operands
 * (tcgen05 kind::f8f6f4) against the query as the sum of four E4M3 parts ("Where This Fits in
 * the Inference Stack", Blackwell FP4), within the same 2e-3 bar. No workspace. Supported:
 * d = 128, TurboQuant_mse keys of 3 or 4 bits or TQ_E2M1 keys, values of 2..4 bits, Hq / Hkv
 * dividing 128; other configurations return TQ_ERR_UNSUPPORTED.
 * Errors: TQ_ERR_INVALID_ARG (pointers, shapes, t0 + Lq > T_cap), TQ_ERR_CUDA. */
int tq_prefill_attention(const void *q, int dtype, int Hq, int Lq, int t0, float scale,
                         const tq_cache *cache, float *out, void *stream);

/* Device-side faults recorded since the last call, as bits: bit 0 = a tensor-core kernel
 * (tcgen05 write path of TurboQuant_prod records) gave up waiting for its MMAs after about a
 * second, recorded a fault, freed its tensor memory and returned without writing the rest of
 * its records; bit 1 = the prefill kernel gave up waiting on one of its pipeline stages the
 * same way and ran to its end without further waits (its outputs undefined). Reading
 * synchronises the device and clears the bits. Writes *flags; returns
 * TQ_OK or TQ_ERR_CUDA. A set bit means a tensor-core
 * operation may still have been in flight when its tensor memory was released: the
 * library's device state (and the outputs of that call) are then undefined, and the caller
 * should treat the CUDA context as lost and tear it down. The pages have no counterpart to
 * this call. */
int tq_device_faults(unsigned *flags);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
