// Quantise-on-write and dequantise kernels ("Closing - The Three-Step Summary", Steps 1-3).
//
// One thread owns one head_dim vector (two threads when d = 256): it loads the vector with
// 16-byte loads, applies the seeded signs, runs the Walsh-Hadamard butterflies in
// registers, divides by the norm, counts boundaries for each coordinate, bit-packs the
// codes and stores them with the widest stores the record alignment allows. TurboQuant_prod
// additionally forms the unit-domain residual, its norm and the QJL sign bits of S r.
#include "tq_device.cuh"

namespace tq {
namespace {

constexpr int kThreads = 128;

// Cross-thread butterfly for the last Walsh-Hadamard stage when two threads share a vector:
// the lower half keeps a + b, the upper half a - b.
template <int EPT, int TPV>
__device__ __forceinline__ void fwht_pair(float (&x)[EPT], int part) {
  if constexpr (TPV == 2) {
#pragma unroll
    for (int i = 0; i < EPT; ++i) {
      float o = __shfl_xor_sync(0xffffffffu, x[i], 1);
      x[i] = part == 0 ? x[i] + o : o - x[i];
    }
  }
}

template <int TPV>
__device__ __forceinline__ float pair_sum(float v) {
  if constexpr (TPV == 2) v += __shfl_xor_sync(0xffffffffu, v, 1);
  return v;
}

template <int EPT>
__device__ __forceinline__ void apply_signs(float (&x)[EPT], uint64_t seed, int first) {
  constexpr int NW = (EPT + 63) / 64;
  uint64_t sw[NW];
#pragma unroll
  for (int k = 0; k < NW; ++k) sw[k] = dev_splitmix64(seed, static_cast<uint64_t>(first / 64 + k));
#pragma unroll
  for (int i = 0; i < EPT; ++i)
    if ((sw[i / 64] >> (i % 64)) & 1ull) x[i] = -x[i];
}

template <int EPT, int TPV, int WBITS, bool PROD>
__global__ void __launch_bounds__(kThreads) quantize_kernel(const QuantArgs a) {
  constexpr int D = EPT * TPV;
  constexpr int NB = EPT * WBITS / 8; // code bytes written by this thread
  constexpr int NWORDS = NB > 0 ? (NB + 3) / 4 : 1;
  const long long nvec = static_cast<long long>(a.B) * a.Hkv * a.T;
  const long long gt = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long v = gt / TPV;
  const int part = TPV == 1 ? 0 : static_cast<int>(gt % TPV);
  const bool active = v < nvec;
  const long long vc = active ? v : nvec - 1;
  const long long bh = vc / a.T;
  const int t = static_cast<int>(vc - bh * a.T);
  const size_t rec = static_cast<size_t>(bh) * a.T_cap + a.t_offset + t;

  float x[EPT];
  load_vec<EPT>(a.x, a.dtype, static_cast<size_t>(vc) * D + part * EPT, x);
  apply_signs<EPT>(x, a.seed, part * EPT);
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < EPT; ++i) ss = fmaf(x[i], x[i], ss);
  ss = pair_sum<TPV>(ss);
  fwht_reg<EPT>(x);
  fwht_pair<EPT, TPV>(x, part);
  const float n = sqrtf(ss);
  const float inv = n > 0.f ? 1.0f / n : 0.0f;

  uint32_t words[NWORDS];
#pragma unroll
  for (int k = 0; k < NWORDS; ++k) words[k] = 0;
  const float inv_sqrt_d = rsqrtf(static_cast<float>(D));
  float rr = 0.f;
#pragma unroll
  for (int i = 0; i < EPT; ++i) {
    const float z = x[i] * inv;
    uint32_t code = 0;
    float cv = WBITS > 0 ? a.t.cb.c[0] : 0.f;
#pragma unroll
    for (int j = 0; j + 1 < (1 << WBITS); ++j) {
      const bool above = z > a.t.cb.beta[j];
      code += above ? 1u : 0u;
      if (PROD) cv = above ? a.t.cb.c[j + 1] : cv;
    }
    if constexpr (WBITS > 0) {
      const int bit = i * WBITS;
      words[bit >> 5] |= code << (bit & 31);
      if ((bit & 31) + WBITS > 32) words[(bit >> 5) + 1] |= code >> (32 - (bit & 31));
    }
    if (PROD) {
      x[i] = (z - cv) * inv_sqrt_d; // residual r in the unit-norm rotated domain
      rr = fmaf(x[i], x[i], rr);
    }
  }
  if constexpr (WBITS > 0) {
    if (active)
      store_bytes<NB>(a.t.codes + rec * a.t.code_bytes + part * NB, words);
  }
  if (active && part == 0) a.t.norm[rec] = f32_to_f16_bits(n);

  if constexpr (PROD) {
    rr = pair_sum<TPV>(rr);
    if (active && part == 0) a.t.rnorm[rec] = f32_to_f16_bits(sqrtf(rr));
    uint8_t *sdst = a.t.signs + rec * a.t.sign_bytes;
    uint32_t byte = 0;
    for (int j = 0; j < a.t.m; ++j) {
      const float4 *row = reinterpret_cast<const float4 *>(a.t.S + static_cast<size_t>(j) * D +
                                                           part * EPT);
      float acc = 0.f;
#pragma unroll
      for (int k = 0; k < EPT / 4; ++k) {
        const float4 s4 = __ldg(row + k);
        acc = fmaf(s4.x, x[4 * k], acc);
        acc = fmaf(s4.y, x[4 * k + 1], acc);
        acc = fmaf(s4.z, x[4 * k + 2], acc);
        acc = fmaf(s4.w, x[4 * k + 3], acc);
      }
      acc = pair_sum<TPV>(acc);
      byte |= (acc < 0.f ? 1u : 0u) << (j & 7);
      if ((j & 7) == 7) {
        if (active && part == 0) sdst[j >> 3] = static_cast<uint8_t>(byte);
        byte = 0;
      }
    }
  }
}

template <int EPT, int TPV, int WBITS, bool PROD>
__global__ void __launch_bounds__(kThreads) dequantize_kernel(const DequantArgs a) {
  constexpr int D = EPT * TPV;
  constexpr int NB = EPT * WBITS / 8;
  constexpr int NWORDS = NB > 0 ? (NB + 3) / 4 + 1 : 1;
  __shared__ float lut[16];
  if (threadIdx.x < 16) lut[threadIdx.x] = threadIdx.x < a.t.cb.levels ? a.t.cb.c[threadIdx.x] : 0.f;
  __syncthreads();
  const long long nvec = static_cast<long long>(a.B) * a.Hkv * a.T_len;
  const long long gt = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long v = gt / TPV;
  const int part = TPV == 1 ? 0 : static_cast<int>(gt % TPV);
  const bool active = v < nvec;
  const long long vc = active ? v : nvec - 1;
  const long long bh = vc / a.T_len;
  const int t = static_cast<int>(vc - bh * a.T_len);
  const size_t rec = static_cast<size_t>(bh) * a.T_cap + t;

  float y[EPT];
  if constexpr (WBITS > 0) {
    uint32_t words[NWORDS];
    words[NWORDS - 1] = 0;
    load_bytes<NB>(a.t.codes + rec * a.t.code_bytes + part * NB, words);
#pragma unroll
    for (int i = 0; i < EPT; ++i) {
      const int bit = i * WBITS;
      uint32_t c = words[bit >> 5] >> (bit & 31);
      if ((bit & 31) + WBITS > 32) c |= words[(bit >> 5) + 1] << (32 - (bit & 31));
      y[i] = lut[c & ((1u << WBITS) - 1u)];
    }
  } else {
#pragma unroll
    for (int i = 0; i < EPT; ++i) y[i] = 0.f;
  }
  if constexpr (PROD) {
    const float gamma = f16_bits_to_f32(a.t.rnorm[rec]);
    const float kappa = sqrtf(static_cast<float>(D)) * gamma * 1.2533141373155003f /
                        static_cast<float>(a.t.m); // sqrt(pi/2)
    const uint8_t *sb = a.t.signs + rec * a.t.sign_bytes;
    for (int j = 0; j < a.t.m; ++j) {
      const bool neg = (__ldg(sb + (j >> 3)) >> (j & 7)) & 1;
      const float coef = neg ? -kappa : kappa;
      const float4 *row = reinterpret_cast<const float4 *>(a.t.S + static_cast<size_t>(j) * D +
                                                           part * EPT);
#pragma unroll
      for (int k = 0; k < EPT / 4; ++k) {
        const float4 s4 = __ldg(row + k);
        y[4 * k] = fmaf(coef, s4.x, y[4 * k]);
        y[4 * k + 1] = fmaf(coef, s4.y, y[4 * k + 1]);
        y[4 * k + 2] = fmaf(coef, s4.z, y[4 * k + 2]);
        y[4 * k + 3] = fmaf(coef, s4.w, y[4 * k + 3]);
      }
    }
  }
  fwht_reg<EPT>(y);
  fwht_pair<EPT, TPV>(y, part);
  const float scale = f16_bits_to_f32(a.t.norm[rec]) / static_cast<float>(D);
#pragma unroll
  for (int i = 0; i < EPT; ++i) y[i] *= scale;
  apply_signs<EPT>(y, a.seed, part * EPT);
  if (active) store_vec<EPT>(a.out, a.dtype, static_cast<size_t>(vc) * D + part * EPT, y);
}

template <int EPT, int TPV, int WBITS, bool PROD>
cudaError_t run_quantize(const QuantArgs &a, cudaStream_t s) {
  const long long threads = static_cast<long long>(a.B) * a.Hkv * a.T * TPV;
  const long long blocks = (threads + kThreads - 1) / kThreads;
  if (blocks > 0x7fffffffll) return cudaErrorInvalidValue;
  quantize_kernel<EPT, TPV, WBITS, PROD><<<static_cast<unsigned>(blocks), kThreads, 0, s>>>(a);
  return cudaGetLastError();
}

template <int EPT, int TPV, int WBITS, bool PROD>
cudaError_t run_dequantize(const DequantArgs &a, cudaStream_t s) {
  const long long threads = static_cast<long long>(a.B) * a.Hkv * a.T_len * TPV;
  const long long blocks = (threads + kThreads - 1) / kThreads;
  if (blocks > 0x7fffffffll) return cudaErrorInvalidValue;
  dequantize_kernel<EPT, TPV, WBITS, PROD><<<static_cast<unsigned>(blocks), kThreads, 0, s>>>(a);
  return cudaGetLastError();
}

// (wbits, prod, d) -> template dispatch.
#define TQ_DISPATCH_BITS(RUN, EPT, TPV)                                        \
  do {                                                                         \
    if (!prod) {                                                               \
      switch (wbits) {                                                         \
      case 1: return RUN<EPT, TPV, 1, false>(a, s);                            \
      case 2: return RUN<EPT, TPV, 2, false>(a, s);                            \
      case 3: return RUN<EPT, TPV, 3, false>(a, s);                            \
      case 4: return RUN<EPT, TPV, 4, false>(a, s);                            \
      }                                                                        \
    } else {                                                                   \
      switch (wbits) {                                                         \
      case 0: return RUN<EPT, TPV, 0, true>(a, s);                             \
      case 1: return RUN<EPT, TPV, 1, true>(a, s);                             \
      case 2: return RUN<EPT, TPV, 2, true>(a, s);                             \
      case 3: return RUN<EPT, TPV, 3, true>(a, s);                             \
      }                                                                        \
    }                                                                          \
    return cudaErrorInvalidValue;                                              \
  } while (0)

#define TQ_DISPATCH_D(RUN)                                                     \
  do {                                                                         \
    const int wbits = a.t.wbits;                                               \
    const bool prod = a.t.mode == TQ_PROD;                                     \
    switch (a.d) {                                                             \
    case 16: TQ_DISPATCH_BITS(RUN, 16, 1);                                     \
    case 32: TQ_DISPATCH_BITS(RUN, 32, 1);                                     \
    case 64: TQ_DISPATCH_BITS(RUN, 64, 1);                                     \
    case 128: TQ_DISPATCH_BITS(RUN, 128, 1);                                   \
    case 256: TQ_DISPATCH_BITS(RUN, 128, 2);                                   \
    }                                                                          \
    return cudaErrorInvalidValue;                                              \
  } while (0)

} // namespace

cudaError_t launch_quantize(const QuantArgs &a, cudaStream_t s) { TQ_DISPATCH_D(run_quantize); }

cudaError_t launch_dequantize(const DequantArgs &a, cudaStream_t s) {
  TQ_DISPATCH_D(run_dequantize);
}

} // namespace tq
