// Device helpers shared by the libtq kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "../../include/tq.h"
#include "tq_internal.h"

namespace tq {

// SplitMix64 output k from seed (Steele, Lea & Flood, OOPSLA 2014). Counter-based, so any
// thread can draw any word of the rotation's sign stream.
__device__ __forceinline__ uint64_t dev_splitmix64(uint64_t seed, uint64_t k) {
  uint64_t z = seed + (k + 1) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// D_ii = -1 iff bit i of the sign stream is set.
__device__ __forceinline__ bool sign_is_neg(uint64_t seed, int i) {
  return (dev_splitmix64(seed, static_cast<uint64_t>(i >> 6)) >> (i & 63)) & 1ull;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float load_scalar(const void *p, int dtype, size_t i) {
  if (dtype == TQ_F32) return static_cast<const float *>(p)[i];
  if (dtype == TQ_BF16) return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]);
  return __half2float(static_cast<const __half *>(p)[i]);
}

// N consecutive elements starting at element i (i a multiple of 8, base 16-byte aligned).
template <int N>
__device__ __forceinline__ void load_vec(const void *p, int dtype, size_t i, float (&x)[N]) {
  static_assert(N % 8 == 0, "vector loads move 8 elements at a time");
  if (dtype == TQ_F32) {
    const float4 *s = reinterpret_cast<const float4 *>(static_cast<const float *>(p) + i);
#pragma unroll
    for (int k = 0; k < N / 4; ++k) {
      float4 v = __ldg(s + k);
      x[4 * k] = v.x;
      x[4 * k + 1] = v.y;
      x[4 * k + 2] = v.z;
      x[4 * k + 3] = v.w;
    }
  } else if (dtype == TQ_BF16) {
    const uint4 *s = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(p) + i);
#pragma unroll
    for (int k = 0; k < N / 8; ++k) {
      uint4 v = __ldg(s + k);
      uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        x[8 * k + 2 * e] = bf16_lo(w[e]);
        x[8 * k + 2 * e + 1] = bf16_hi(w[e]);
      }
    }
  } else {
    const uint4 *s = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(p) + i);
#pragma unroll
    for (int k = 0; k < N / 8; ++k) {
      uint4 v = __ldg(s + k);
      uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        __half2 h = *reinterpret_cast<__half2 *>(&w[e]);
        float2 f = __half22float2(h);
        x[8 * k + 2 * e] = f.x;
        x[8 * k + 2 * e + 1] = f.y;
      }
    }
  }
}

// Store N elements (N a multiple of 8, 16-byte aligned destination) as `dtype`.
template <int N>
__device__ __forceinline__ void store_vec(void *p, int dtype, size_t i, const float (&x)[N]) {
  if (dtype == TQ_F32) {
    float4 *d = reinterpret_cast<float4 *>(static_cast<float *>(p) + i);
#pragma unroll
    for (int k = 0; k < N / 4; ++k)
      d[k] = make_float4(x[4 * k], x[4 * k + 1], x[4 * k + 2], x[4 * k + 3]);
  } else {
    uint4 *d = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p) + i);
#pragma unroll
    for (int k = 0; k < N / 8; ++k) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float a = x[8 * k + 2 * e], b = x[8 * k + 2 * e + 1];
        if (dtype == TQ_BF16) {
          __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
          w[e] = *reinterpret_cast<uint32_t *>(&h);
        } else {
          __half2 h = __floats2half2_rn(a, b);
          w[e] = *reinterpret_cast<uint32_t *>(&h);
        }
      }
      d[k] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

// Unnormalised in-register fast Walsh-Hadamard transform (natural order).
template <int N>
__device__ __forceinline__ void fwht_reg(float (&x)[N]) {
#pragma unroll
  for (int h = 1; h < N; h <<= 1) {
#pragma unroll
    for (int i = 0; i < N; ++i) {
      if ((i & h) == 0) {
        float a = x[i], b = x[i + h];
        x[i] = a + b;
        x[i + h] = a - b;
      }
    }
  }
}

// Store NB bytes held little-endian in w[] to dst, using the widest stores its alignment
// allows.
template <int NB>
__device__ __forceinline__ void store_bytes(uint8_t *dst, const uint32_t *w) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(dst);
  if constexpr (NB % 16 == 0) {
    if ((a & 15) == 0) {
#pragma unroll
      for (int k = 0; k < NB / 16; ++k)
        reinterpret_cast<uint4 *>(dst)[k] =
            make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
      return;
    }
  }
  if constexpr (NB % 8 == 0) {
    if ((a & 7) == 0) {
#pragma unroll
      for (int k = 0; k < NB / 8; ++k)
        reinterpret_cast<uint2 *>(dst)[k] = make_uint2(w[2 * k], w[2 * k + 1]);
      return;
    }
  }
  if constexpr (NB % 4 == 0) {
    if ((a & 3) == 0) {
#pragma unroll
      for (int k = 0; k < NB / 4; ++k) reinterpret_cast<uint32_t *>(dst)[k] = w[k];
      return;
    }
  }
  if constexpr (NB % 2 == 0) {
    if ((a & 1) == 0) {
#pragma unroll
      for (int k = 0; k < NB / 2; ++k)
        reinterpret_cast<uint16_t *>(dst)[k] = static_cast<uint16_t>(w[k / 2] >> (16 * (k & 1)));
      return;
    }
  }
#pragma unroll
  for (int k = 0; k < NB; ++k) dst[k] = static_cast<uint8_t>(w[k / 4] >> (8 * (k & 3)));
}

// Load NB bytes from src into w[] (little-endian words), widest loads first.
template <int NB>
__device__ __forceinline__ void load_bytes(const uint8_t *src, uint32_t *w) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(src);
  if constexpr (NB % 16 == 0) {
    if ((a & 15) == 0) {
#pragma unroll
      for (int k = 0; k < NB / 16; ++k) {
        uint4 v = __ldg(reinterpret_cast<const uint4 *>(src) + k);
        w[4 * k] = v.x;
        w[4 * k + 1] = v.y;
        w[4 * k + 2] = v.z;
        w[4 * k + 3] = v.w;
      }
      return;
    }
  }
  if constexpr (NB % 4 == 0) {
    if ((a & 3) == 0) {
#pragma unroll
      for (int k = 0; k < NB / 4; ++k) w[k] = __ldg(reinterpret_cast<const uint32_t *>(src) + k);
      return;
    }
  }
#pragma unroll
  for (int k = 0; k < (NB + 3) / 4; ++k) w[k] = 0;
#pragma unroll
  for (int k = 0; k < NB; ++k) w[k / 4] |= static_cast<uint32_t>(__ldg(src + k)) << (8 * (k & 3));
}

__device__ __forceinline__ uint16_t f32_to_f16_bits(float v) {
  return __half_as_ushort(__float2half_rn(v));
}
__device__ __forceinline__ float f16_bits_to_f32(uint16_t b) {
  return __half2float(__ushort_as_half(b));
}

// 2^x for online-softmax weights and rescale factors (x <= 0 or -inf): the hardware
// approximation (MUFU.EX2, relative error ~2^-22) with results below 2^-126 flushed to zero,
// which a softmax weight can afford; NaN stays NaN.
__device__ __forceinline__ float softmax_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Programmatic dependent launch. A kernel launched with launch_pdl may start while the
// kernel before it in the stream is still running; it must call pdl_wait() before it reads
// anything an earlier kernel wrote (or writes anything an earlier kernel reads), and may call
// pdl_trigger() to let the next such kernel start early.
// Blackwell packed fp32 pairs: one instruction operates on both lanes of a 64-bit register pair.
typedef unsigned long long f2_t; // two fp32 lanes in one 64-bit register pair

__device__ __forceinline__ f2_t f2(float a, float b) {
  f2_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_split(f2_t v, float &a, float &b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ f2_t add2(f2_t a, f2_t b) {
  f2_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f2_t sub2(f2_t a, f2_t b) {
  f2_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f2_t mul2(f2_t a, f2_t b) {
  f2_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f2_t fma2(f2_t a, f2_t b, f2_t c) {
  f2_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

} // namespace tq
