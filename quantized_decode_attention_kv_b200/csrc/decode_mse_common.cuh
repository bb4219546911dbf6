// Pieces of the tensor-core attention kernels over TurboQuant_mse records at head_dim 128: the
// fixed-point query preparation, the score accumulators' float read-back constants,
// shared-memory table loads with immediate offsets and bit-field helpers.
#pragma once

#include "mma_ops.cuh"

namespace tq {
namespace mse {
using namespace mma_ops;

constexpr int kD = 128;
// Magnitude of the largest 24-bit fixed-point query coordinate: below 127 * 65536 + 127 * 256
// + 127 = 8355711 with a margin for the float rounding of max|q~| * (8355000 / max|q~|), so the
// int8 parts stay in [-127, 127] (hi) and [-128, 127] (mid, lo).
constexpr float kQFixMax = 8355000.0f;
// Score accumulators start at the bits of 1.5 * 2^23: an int32 sum s with |s| < 2^22 (each
// column sums 128 products of two int8 parts, one of them <= 127 in magnitude, or two such
// sums) reads back as the float 1.5 * 2^23 + s exactly. kMagicAdj = 1.5 * 2^23 *
// (1 + 2^-8 + 2^-16) removes the three offsets of col0 + col1 / 2^8 + col2 / 2^16.
constexpr int kMagic = 0x4B400000;
constexpr float kMagicAdj = 12632256.0f;
constexpr float kLog2e = 1.4426950408889634f;
// The first dynamic shared address of a kernel without static shared memory on sm_100 (the
// 1 KB below it is reserved by the hardware); the kernel checks it before relying on it.
constexpr uint32_t kFixedBase = 1024;

template <uint32_t OFF>
__device__ __forceinline__ uint32_t lds32_off(uint32_t smem_addr) {
  uint32_t v;
  asm("ld.shared.u32 %0, [%1+%2];" : "=r"(v) : "r"(smem_addr), "n"(OFF));
  return v;
}

template <uint32_t OFF>
__device__ __forceinline__ uint2 lds64_off(uint32_t smem_addr) {
  uint2 v;
  // not volatile: the tables are read-only after the fill barrier, and leaving the loads free
  // lets the compiler hoist them ahead of the MMAs that consume them
  asm("ld.shared.v2.u32 {%0, %1}, [%2+%3];" : "=r"(v.x), "=r"(v.y) : "r"(smem_addr), "n"(OFF));
  return v;
}
// A prepared query: rotated once (q'' = H D q), scaled (q~ = scale q'' / d), as a 24-bit
// fixed-point vector q_int = rint(q~ * 8355839 / max|q~|) split into int8 parts
// q_int = 65536 hi + 256 mid + lo. The decode kernel builds one per query head of a segment in
// shared memory.
struct QPrep {
  int8_t hi[kD];
  int8_t mid[kD];
  int8_t lo[kD];
  float inv; // score = ||k|| * inv * (col0 + col1 / 2^8 + col2 / 2^16), see the score MMA
  float pad[3];
};


// Rotation and scaling of one query by one warp: q~ = scale (H D q) / d. Lane l holds
// coordinates 4 l .. 4 l + 3; the butterflies of span 1, 2 run in the lane, those of span
// 4 .. 64 across lanes (the lane with the span bit set keeps partner - own).
__device__ __forceinline__ void rotate_query(const void *q, int dtype, size_t bq, float scale,
                                             uint64_t seed, int lane, float (&x)[4]) {
  const uint64_t sw = dev_splitmix64(seed, static_cast<uint64_t>(lane >> 4)); // coordinates 64 k ..
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int i = 4 * lane + e;
    x[e] = load_scalar(q, dtype, bq * kD + i);
    if ((sw >> (i & 63)) & 1ull) x[e] = -x[e];
  }
  {
    const float a0 = x[0] + x[1], a1 = x[0] - x[1], a2 = x[2] + x[3], a3 = x[2] - x[3];
    x[0] = a0 + a2;
    x[2] = a0 - a2;
    x[1] = a1 + a3;
    x[3] = a1 - a3;
  }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float o = __shfl_xor_sync(0xffffffffu, x[e], m);
      x[e] = upper ? o - x[e] : x[e] + o;
    }
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) x[e] *= scale / static_cast<float>(kD);
}

// Query prep of one query by one warp: rotate and scale (rotate_query), round to 24-bit fixed
// point at the full range and split into int8 hi, mid and lo; csc is the centroids'
// fixed-point scale.
__device__ __forceinline__ void prep_query(const void *q, int dtype, size_t bq, float scale,
                                           uint64_t seed, float csc, QPrep *out, int lane) {
  float x[4];
  rotate_query(q, dtype, bq, scale, seed, lane, x);
  float mx = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) mx = fmaxf(mx, fabsf(x[e]));
  mx = warp_max(mx);
  // fmaxf ignores NaN, so a NaN anywhere in the query (the rotation spreads it to every
  // coordinate) is detected separately
  const bool has_nan = __any_sync(0xffffffffu, isnan(x[0]) || isnan(x[1]) || isnan(x[2]) || isnan(x[3]));
  // A query whose largest coordinate is below 1e-30 (zero included) gets zero scores (its
  // exact scores are below 1e-30 times the key norms). A query holding a NaN or an infinity
  // gets the score factor NaN: its scores, softmax weights and output are NaN, as exact
  // attention would give.
  const bool ok = !has_nan && mx > 1e-30f && isfinite(mx);
  const float qsc = ok ? kQFixMax / mx : 0.f;
  uint32_t hw = 0, mw = 0, lw = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int qi = __float2int_rn(x[e] * qsc);
    const int lo = ((qi + 128) & 255) - 128;
    const int q1 = (qi - lo) >> 8;
    const int mid = ((q1 + 128) & 255) - 128;
    const int hi = (q1 - mid) >> 8;
    hw |= static_cast<uint32_t>(hi & 255) << (8 * e);
    mw |= static_cast<uint32_t>(mid & 255) << (8 * e);
    lw |= static_cast<uint32_t>(lo & 255) << (8 * e);
  }
  reinterpret_cast<uint32_t *>(out->hi)[lane] = hw;
  reinterpret_cast<uint32_t *>(out->mid)[lane] = mw;
  reinterpret_cast<uint32_t *>(out->lo)[lane] = lw;
  if (lane == 0) out->inv = ok ? 16777216.0f / (qsc * csc) : (!has_nan && isfinite(mx) ? 0.f : __int_as_float(0x7fc00000));
}

// Bits [o, o + n) of the little-endian bit string w[0..NWD) moved to bit DST (other bits
// of the result are unspecified above DST + n and zero below DST when o >= DST).
template <int NWD>
__device__ __forceinline__ uint32_t bits_at(const uint32_t (&w)[NWD], int o, int dst) {
  const int sh = o - dst;
  if (sh < 0) return w[0] << (-sh);
  const int wi = sh >> 5, bi = sh & 31;
  if (bi == 0) return w[wi];
  const uint32_t hi = wi + 1 < NWD ? w[wi + 1] : 0u;
  return __funnelshift_r(w[wi], hi, bi);
}

__device__ __forceinline__ uint32_t lop_and_or(uint32_t a, uint32_t mask, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(c)); // (a & mask) | c
  return d;
}

} // namespace mse
} // namespace tq
