// Private interface between the C-ABI host layer (host.cpp) and the CUDA launchers.
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace tq {

constexpr int kMaxM = 256;       // longest QJL sketch supported
constexpr int kMaxSplits = 1024; // split-K upper bound per (b, q-head)

// Lloyd-Max codebook on the N(0,1) scale (the kernels work on z = H D x / ||x||).
struct Codebook {
  float c[16];    // centroids, ascending (levels entries used)
  float beta[15]; // decision boundaries, ascending (levels - 1 used)
  int levels;     // 2^wbits; 1 when a PROD record carries no Lloyd-Max codes
  float fix_scale; // 16-bit fixed-point scale of the centroids (|rint(c * fix_scale)| <= 32639)
};

// One tensor (K or V) of a cache, resolved from tq_cache + tq_qcfg.
struct TensorArgs {
  int bits, mode;  // as given
  int wbits;       // Lloyd-Max bits per coordinate (bits, or bits - 1 in PROD)
  int m;           // QJL rows (PROD), else 0
  int code_bytes;  // d * wbits / 8
  int sign_bytes;  // m / 8 (PROD), else 0
  uint8_t *codes;
  uint16_t *norm;
  uint8_t *signs;
  uint16_t *rnorm;
  const float *S;  // [m][d] (PROD)
  Codebook cb;
};

// Paging of a cache (pshift < 0: the dense [B][Hkv][T_cap] layout): record (b, h, t) sits at
// page bt[b * maxp + (t >> pshift)], head h, slot t & (2^pshift - 1).
struct Paging {
  const int *bt;
  int pshift, maxp;
};

struct QuantArgs {
  const void *x;
  int dtype;
  int B, Hkv, T, T_cap, t_offset, d;
  uint64_t seed;
  uint64_t sign_words[4]; // SplitMix64 outputs 0..3 of `seed`: bit i set <=> D_ii = -1
  TensorArgs t;
  Paging pg; // pshift = -1 unless writing a paged cache
};

struct DequantArgs {
  void *out;
  int dtype;
  int B, Hkv, T_len, T_cap, d;
  uint64_t seed;
  TensorArgs t;
};

struct DecodePlan {
  int path;      // 0: generic split-K kernel; 1: tensor-core MSE kernel (decode_mma.cu);
                 // 2: tensor-core PROD kernel (decode_prod.cu); 3: tensor-core bf16 kernel
                 // (decode_bf16.cu)
  int tile;      // tokens per pipeline tile
  int splits;    // context splits per (b, KV head) (path 0)
  int chunk;     // tokens per split (a multiple of tile) (path 0)
  int gc;        // query heads handled by one CTA (path 0: power of two; path 1: G)
  int ws_stride; // floats per partial record
  // path 1: the (b, KV head, 16-token tile) space is cut into equal per-warp ranges
  int tiles_per_bh, tiles_per_cta, tiles_per_warp, ctas, slots;
  size_t part_bytes; // bytes of partial records (the query-prep area follows)
  size_t ws_bytes;
};

// Per-sequence context lengths of a ragged decode call, passed by value to the kernels: the
// flattened (b, KV head, 16-token tile) space gives sequence b ceil(len[b] / 16) tiles per KV
// head, starting at tile boff[b].
constexpr int kMaxVarlenB = 512;
struct VarLen {
  int on; // 0: every sequence has the call's T_len
  int boff[kMaxVarlenB + 1];
  int blen[kMaxVarlenB];
};

struct DecodeArgs {
  const int *T_lens; // host array of B per-sequence lengths, or NULL (uniform T_len)
  Paging pg;         // pshift = -1 unless reading a paged cache (then T_lens is set)
  const void *q;
  int q_dtype;
  int B, Hq, Hkv, d, T_len, T_cap;
  float scale;
  uint64_t seed;
  TensorArgs k, v;
  float *out;
  float *ws;
  DecodePlan plan;
};

struct DecodeBf16Args {
  const void *q, *K, *V;
  int B, Hq, Hkv, d, T_len, T_cap;
  float scale;
  float *out;
  float *ws;
  DecodePlan plan;
};

// Launchers (quantize.cu, decode.cu). Return the launch status.
cudaError_t launch_quantize(const QuantArgs &a, cudaStream_t s);

// Streaming quantiser (quantize_fast.cu): MSE records of bf16/f16 input, head_dim 64 or 128.
// K and V (either may be NULL, both must be supported and share dtype, d and seed) are
// written by one launch.
bool quantize_fast_supported(const QuantArgs &a);
cudaError_t launch_quantize_fast(const QuantArgs *k, const QuantArgs *v, int sm_count,
                                 cudaStream_t s);

// TurboQuant_prod quantiser with the QJL sketch on the tensor cores (quantize_prod.cu):
// head_dim 64, 64 sketch rows, 1- or 2-bit records, bf16/f16 input; K and V in one launch.
bool quantize_prod_supported(const QuantArgs &a);
cudaError_t read_and_clear_prod_faults(unsigned *flags);
cudaError_t launch_quantize_prod(const QuantArgs *k, const QuantArgs *v, int sm_count,
                                 cudaStream_t s);
cudaError_t launch_dequantize(const DequantArgs &a, cudaStream_t s);
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s);
cudaError_t launch_decode_bf16(const DecodeBf16Args &a, cudaStream_t s);

// Device address and size (bytes) of the fixed scratch array behind
// tq_decode_attention_noalloc (decode.cu). The first call on a device looks the address up
// with that device current; later calls return the cached address.
cudaError_t fixed_scratch(float **ptr, size_t *bytes);

// Split-K plan for the compressed and bf16 decode kernels (decode.cu). `fast` selects a
// tensor-core kernel: 0 (none), (key bits << 4) | value bits (MSE, see
// fast_decode_supported) or kProdFast (see prod_decode_supported).
DecodePlan plan_decode(int B, int Hq, int Hkv, int d, int T_len, int v_m, int sm_count,
                       bool bf16, int fast = 0);

// Tensor-core decode (decode_mma.cu): head_dim 128, MSE keys of 3 or 4 bits, MSE values of
// 2, 3 or 4 bits, 1..8 query heads per KV head.
bool fast_decode_supported(int d, int k_mode, int k_wbits, int v_mode, int v_wbits, int G);
// T_lens: NULL (every sequence T_len long) or B per-sequence lengths (ragged call).
void plan_fast(int B, int Hq, int Hkv, int T_len, int sm_count, int kb, int vb, DecodePlan *p,
               const int *T_lens = nullptr);
cudaError_t launch_fast_decode(const DecodeArgs &a, cudaStream_t s);

// Prefill (chunked) attention over the compressed cache on tcgen05 tensor cores (prefill.cu):
// head_dim 128, MSE keys of 3 or 4 bits, MSE values of 2..4 bits, G dividing 128. The Lq
// queries q[B][Lq][Hq][128] at positions t0 .. t0 + Lq - 1 attend causally to the cache.
struct PrefillLaunch {
  const void *q;
  int q_dtype;
  int B, Hq, Hkv, Lq, t0, T_cap;
  float scale;
  uint64_t seed;
  TensorArgs k, v;
  float *out;
  bool k_e2m1; // keys on the E2M1 grid (TQ_E2M1): the kernel feeds them to E2M1 tensor-core MMAs
};
bool prefill_supported(int d, int k_mode, int k_wbits, int v_mode, int v_wbits, int G);
cudaError_t launch_prefill(const PrefillLaunch &l, cudaStream_t s);
cudaError_t read_and_clear_prefill_faults(unsigned *flags);

// Tensor-core decode of TurboQuant_prod records (decode_prod.cu): head_dim 64, 2-bit keys and
// values with 64 QJL rows each, 1..2 query heads per KV head. Plan code kProdFast.
constexpr int kProdFast = 0x200;
bool prod_decode_supported(int d, int k_mode, int k_bits, int k_m, int v_mode, int v_bits, int v_m,
                           int G);
// T_lens: NULL (every sequence T_len long) or B per-sequence lengths (ragged call; T_len is then
// the longest).
void plan_prod(int B, int Hq, int Hkv, int T_len, int sm_count, DecodePlan *p, const int *T_lens = nullptr);
cudaError_t launch_prod_decode(const DecodeArgs &a, cudaStream_t s);

// Tensor-core bf16 decode (decode_bf16.cu): head_dim 128, 1..8 query heads per KV head.
bool bf16_decode_supported(int d, int G);
void plan_bf16_mma(int B, int Hq, int Hkv, int T_len, int sm_count, DecodePlan *p);
cudaError_t launch_bf16_mma(const DecodeBf16Args &a, cudaStream_t s);

} // namespace tq
