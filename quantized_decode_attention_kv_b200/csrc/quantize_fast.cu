// Streaming quantise-on-write for MSE records of 16-bit K/V ("Closing - The Three-Step
// Summary", Steps 1-3; the spec write path: norm, seeded-sign Walsh-Hadamard rotation,
// Lloyd-Max codes, LSB-first packing).
//
// Design (B200):
//  * Persistent CTAs of 128 threads walk 128-vector batches of K and then V in one launch.
//    Each batch (128 x d 16-bit elements, contiguous in memory) is copied into shared memory
//    with coalesced 16-byte cp.async copies, double-buffered so the next batch is in flight
//    while this one is computed. Rows are padded by 16 bytes so that the 16-byte row reads of
//    one thread per vector never share a bank.
//  * One thread owns one vector: the whole transform stays in registers. Coordinates are
//    held as packed fp32 pairs (x_j, x_{j+d/2}); the sum of squares and all but one of the
//    log2(d) butterfly stages run as Blackwell f32x2 instructions (two lanes of work per
//    instruction). Signs are applied while widening the 16-bit inputs (an add of 2^31 to the
//    fp32 bit pattern flips its sign).
//  * Code search: z is mapped to one of 256 cells of width 1/4 on the N(0,1) scale with one
//    fused multiply-add (the cell index lands in the low mantissa bits of a float offset by
//    1.5 * 2^23); a shared-memory table gives, per cell, the number of decision boundaries
//    below it and the single boundary inside it (Lloyd-Max boundaries of <= 4 bits are more
//    than 1/4 apart), so every code costs one table read and one compare. A zero vector maps
//    to z = 0, whose cell holds the boundary 0, and gets the lower code as a tie should.
#include "tq_device.cuh"

namespace tq {
namespace {

constexpr int kQThreads = 128; // vectors per batch, one per thread
constexpr int kCells = 256;
constexpr float kCellScale = 32.0f;                 // 8 / cell width
constexpr float kCellMagic = 12582912.0f + 1024.0f; // 1.5 * 2^23 + 8 * 128

struct FastTensor {
  const uint8_t *x; // [nvec][d] 16-bit elements
  uint8_t *codes;
  uint16_t *norm;
  long long nbatch;
  unsigned nvec;
  int T, T_cap, t_offset, wbits, code_bytes, nbeta;
  float beta[15];
};

struct FastQuantArgs {
  FastTensor t[2];
  long long nbatch_total;
  // bit 31 set where D flips coordinate 2p (lo) / 2p + 1 (hi) of 16-bit pair p
  uint32_t sgn_lo[64], sgn_hi[64];
};

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

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

__device__ __forceinline__ uint4 lds128(const uint8_t *p) {
  return *reinterpret_cast<const uint4 *>(p);
}

// Add `code` (WB bits) into the record at coordinate i (the record starts zeroed and codes
// occupy disjoint bits, so the add is an OR that can fold into one shift-add).
template <int WB>
__device__ __forceinline__ void put_code(uint32_t *words, int i, uint32_t code) {
  const int bit = i * WB, wi = bit >> 5, sh = bit & 31;
  words[wi] += code << sh;
  if (sh + WB > 32) words[wi + 1] += code >> (32 - sh);
}

// Cell-table entry {boundary bits, base code} for the cell index held in the low mantissa
// bits of u: (u & 0x7F8) | table is one LOP3 because the table is 2048-byte aligned.
__device__ __forceinline__ uint2 cell_entry(float u, uint32_t table) {
  uint32_t addr;
  asm("lop3.b32 %0, %1, 0x7F8, %2, 0xEA;" : "=r"(addr) : "r"(__float_as_uint(u)), "r"(table));
  uint2 e;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(e.x), "=r"(e.y) : "r"(addr));
  return e;
}

template <int D, int WB, bool BF16>
__device__ __forceinline__ void quantize_row(const uint8_t *row, uint32_t cells,
                                             const FastQuantArgs &a, const FastTensor &t,
                                             unsigned v) {
  constexpr int H = D / 2; // pair stride: P[j] = (x_j, x_{j+H})
  constexpr int NW = D * WB / 32;
  float x[D];
#pragma unroll
  for (int k = 0; k < D / 8; ++k) {
    const uint4 q = lds128(row + 16 * k);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int p = 4 * k + e;
      if (BF16) {
        x[2 * p] = __uint_as_float(w[e] * 65536u + a.sgn_lo[p]);
        x[2 * p + 1] = __uint_as_float((w[e] & 0xFFFF0000u) ^ a.sgn_hi[p]);
      } else {
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[e]));
        x[2 * p] = __uint_as_float(__float_as_uint(f.x) ^ a.sgn_lo[p]);
        x[2 * p + 1] = __uint_as_float(__float_as_uint(f.y) ^ a.sgn_hi[p]);
      }
    }
  }
  // butterfly stage of span H (within a pair), then the sum of squares on the pairs
  f2_t P[H];
  f2_t ss2 = 0ull;
#pragma unroll
  for (int j = 0; j < H; ++j) {
    P[j] = f2(x[j] + x[j + H], x[j] - x[j + H]);
    ss2 = fma2(P[j], P[j], ss2);
  }
  // the remaining stages, spans 1 .. H/2, between pairs
#pragma unroll
  for (int h = 1; h < H; h <<= 1) {
#pragma unroll
    for (int j = 0; j < H; ++j) {
      if ((j & h) == 0) {
        const f2_t u = P[j], w = P[j + h];
        P[j] = add2(u, w);
        P[j + h] = sub2(u, w);
      }
    }
  }
  float s0, s1;
  f2_split(ss2, s0, s1);
  const float n = sqrtf(0.5f * (s0 + s1)); // the first stage doubled the squared norm
  const float inv = n > 0.f ? 1.0f / n : 0.0f;
  const f2_t inv2 = f2(inv, inv);
  const f2_t cs2 = f2(kCellScale, kCellScale), cm2 = f2(kCellMagic, kCellMagic);

  uint32_t words[NW];
#pragma unroll
  for (int k = 0; k < NW; ++k) words[k] = 0u;
#pragma unroll
  for (int j = 0; j < H; ++j) {
    const f2_t z2 = mul2(P[j], inv2);
    const f2_t u2 = fma2(z2, cs2, cm2);
    float z0, z1, u0, u1;
    f2_split(z2, z0, z1);
    f2_split(u2, u0, u1);
    const uint2 e0 = cell_entry(u0, cells);
    const uint2 e1 = cell_entry(u1, cells);
    put_code<WB>(words, j, e0.y + (z0 > __uint_as_float(e0.x) ? 1u : 0u));
    put_code<WB>(words, j + H, e1.y + (z1 > __uint_as_float(e1.x) ? 1u : 0u));
  }

  const unsigned bh = v / static_cast<unsigned>(t.T);
  const unsigned tt = v - bh * static_cast<unsigned>(t.T);
  const size_t rec = static_cast<size_t>(bh) * t.T_cap + t.t_offset + tt;
  uint8_t *dst = t.codes + rec * (NW * 4);
  if constexpr (NW % 4 == 0) {
#pragma unroll
    for (int k = 0; k < NW / 4; ++k)
      reinterpret_cast<uint4 *>(dst)[k] =
          make_uint4(words[4 * k], words[4 * k + 1], words[4 * k + 2], words[4 * k + 3]);
  } else {
#pragma unroll
    for (int k = 0; k < NW / 2; ++k)
      reinterpret_cast<uint2 *>(dst)[k] = make_uint2(words[2 * k], words[2 * k + 1]);
  }
  t.norm[rec] = f32_to_f16_bits(n);
}

template <int D, bool BF16>
__global__ void __launch_bounds__(kQThreads, 3) quantize_fast_kernel(const FastQuantArgs a) {
  constexpr int ROW = 2 * D + 16;        // padded row bytes
  constexpr int BUF = kQThreads * ROW;   // one staging buffer
  constexpr int CPR = 2 * D / 16;        // 16-byte chunks per row
  extern __shared__ __align__(16) uint8_t smem[];
  // [2 tensors][256 cells] {boundary bits, base code} at the first 2048-byte aligned shared
  // address, then the two staging buffers
  const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  const uint32_t pad = ((sbase + 2047u) & ~2047u) - sbase;
  uint8_t *cells = smem + pad;
  const uint32_t cells_s = sbase + pad;
  uint8_t *stage = cells + 2 * kCells * 8;
  const int tid = threadIdx.x;

  // Cell k covers z in [(8k - 1024.5) / 32, (8k - 1016.5) / 32): the FMA z * 32 + 1.5 * 2^23
  // + 1024 rounds to an integer j and the bits (j & 0x7F8) select k.
  for (int idx = tid; idx < 2 * kCells; idx += kQThreads) {
    const FastTensor &t = a.t[idx / kCells];
    const int k = idx % kCells;
    const float lo = (8.0f * k - 1024.5f) / 32.0f, hi = lo + 0.25f;
    uint32_t base = 0;
    float inner = INFINITY;
    for (int j = 0; j < t.nbeta; ++j) {
      const float b = t.beta[j];
      if (b <= lo) ++base;
      else if (b < hi) inner = b;
    }
    reinterpret_cast<uint2 *>(cells)[idx] = make_uint2(__float_as_uint(inner), base);
  }

  auto issue = [&](long long g, int buf) {
    const int ti = g < a.t[0].nbatch ? 0 : 1;
    const FastTensor &t = a.t[ti];
    const long long lb = g - (ti ? a.t[0].nbatch : 0);
    const unsigned v0 = static_cast<unsigned>(lb * kQThreads);
    const int nv = static_cast<int>(min(static_cast<unsigned>(kQThreads), t.nvec - v0));
    const uint8_t *src = t.x + static_cast<size_t>(v0) * (2 * D);
    const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(stage + buf * BUF));
    if (nv == kQThreads) {
      // chunk j = tid + 128 k: row tid / CPR + k * 128 / CPR, column tid % CPR
      const uint32_t d0 = dst + (tid / CPR) * ROW + (tid % CPR) * 16;
      const uint8_t *s0 = src + tid * 16;
#pragma unroll
      for (int k = 0; k < CPR; ++k)
        cp_async16(d0 + k * (kQThreads / CPR) * ROW, s0 + k * kQThreads * 16);
    } else {
      for (int j = tid; j < nv * CPR; j += kQThreads)
        cp_async16(dst + (j / CPR) * ROW + (j % CPR) * 16, src + static_cast<size_t>(j) * 16);
    }
  };

  pdl_wait(); // K/V may come from the kernel before; the cache may still be read by it
  pdl_trigger();
  long long g = blockIdx.x;
  int buf = 0;
  if (g < a.nbatch_total) issue(g, 0);
  cp_async_commit();
  for (; g < a.nbatch_total; g += gridDim.x, buf ^= 1) {
    const long long gn = g + gridDim.x;
    if (gn < a.nbatch_total) issue(gn, buf ^ 1);
    cp_async_commit();
    cp_async_wait1();
    __syncthreads();
    const int ti = g < a.t[0].nbatch ? 0 : 1;
    const FastTensor &t = a.t[ti];
    const long long lb = g - (ti ? a.t[0].nbatch : 0);
    const unsigned v = static_cast<unsigned>(lb * kQThreads) + tid;
    if (v < t.nvec) {
      const uint8_t *row = stage + buf * BUF + tid * ROW;
      const uint32_t cl = cells_s + ti * kCells * 8;
      switch (t.wbits) {
      case 1: quantize_row<D, 1, BF16>(row, cl, a, t, v); break;
      case 2: quantize_row<D, 2, BF16>(row, cl, a, t, v); break;
      case 3: quantize_row<D, 3, BF16>(row, cl, a, t, v); break;
      default: quantize_row<D, 4, BF16>(row, cl, a, t, v); break;
      }
    }
    __syncthreads();
  }
}

// Few vectors (a decode step's new token): one warp per vector with compact, looped code, so
// that a launch that finds its instructions evicted from L2 by the decode stream still starts
// fast. Lane l holds coordinates [E l, E l + E); the butterflies of span >= E run across
// lanes with shuffles; codes count the boundaries below z; the packed record is assembled in
// shared memory and written by the first lanes.
template <int D, bool BF16>
__global__ void __launch_bounds__(kQThreads) quantize_small_kernel(const FastQuantArgs a) {
  constexpr int E = D / 32;        // coordinates per lane
  constexpr int WPB = kQThreads / 32;
  __shared__ uint32_t rec_words[WPB][D * 4 / 32];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const unsigned gv = blockIdx.x * WPB + wib;
  const unsigned nv0 = a.t[0].nvec;
  const int ti = gv < nv0 ? 0 : 1;
  const FastTensor &t = a.t[ti];
  const unsigned v = gv - (ti ? nv0 : 0u);
  pdl_wait(); // K/V may come from the kernel before; the cache may still be read by it
  pdl_trigger();
  if (ti == 1 && (a.nbatch_total == a.t[0].nbatch || v >= t.nvec)) return;

  float x[E];
  const uint8_t *src = t.x + (static_cast<size_t>(v) * D + E * lane) * 2;
  uint32_t w[E / 2];
  if constexpr (E == 4) {
    const uint2 q = *reinterpret_cast<const uint2 *>(src);
    w[0] = q.x;
    w[1] = q.y;
  } else {
    w[0] = *reinterpret_cast<const uint32_t *>(src);
  }
  float ss = 0.f;
#pragma unroll
  for (int p = 0; p < E / 2; ++p) {
    const int pp = (E * lane) / 2 + p; // 16-bit pair index within the vector
    float lo, hi;
    if (BF16) {
      lo = __uint_as_float(w[p] << 16);
      hi = __uint_as_float(w[p] & 0xFFFF0000u);
    } else {
      const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[p]));
      lo = f.x;
      hi = f.y;
    }
    x[2 * p] = __uint_as_float(__float_as_uint(lo) ^ a.sgn_lo[pp]);
    x[2 * p + 1] = __uint_as_float(__float_as_uint(hi) ^ a.sgn_hi[pp]);
  }
#pragma unroll
  for (int e = 0; e < E; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  // butterflies within the lane
#pragma unroll
  for (int h = 1; h < E; h <<= 1)
#pragma unroll
    for (int e = 0; e < E; ++e)
      if ((e & h) == 0) {
        const float u = x[e], y = x[e + h];
        x[e] = u + y;
        x[e + h] = u - y;
      }
  // butterflies across lanes: the lane with the span bit set keeps partner - own
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float o = __shfl_xor_sync(0xffffffffu, x[e], m);
      x[e] = upper ? o - x[e] : x[e] + o;
    }
  }
  const float n = sqrtf(ss);
  const float inv = n > 0.f ? 1.0f / n : 0.0f;
  const int WB = t.wbits;
  uint32_t bits = 0; // this lane's E codes, E * WB bits
  for (int e = 0; e < E; ++e) {
    const float z = x[e] * inv;
    uint32_t code = 0;
    for (int j = 0; j < t.nbeta; ++j) code += z > t.beta[j] ? 1u : 0u;
    bits |= code << (e * WB);
  }
  const int nw = D * WB / 32;
  uint32_t *rw = rec_words[wib];
  if (lane < nw) rw[lane] = 0u;
  __syncwarp();
  const int bit = lane * E * WB, wi = bit >> 5, sh = bit & 31;
  atomicOr(&rw[wi], bits << sh);
  if (sh + E * WB > 32) atomicOr(&rw[wi + 1], bits >> (32 - sh));
  __syncwarp();
  const unsigned bh = v / static_cast<unsigned>(t.T);
  const unsigned tt = v - bh * static_cast<unsigned>(t.T);
  const size_t rec = static_cast<size_t>(bh) * t.T_cap + t.t_offset + tt;
  if (lane < nw) reinterpret_cast<uint32_t *>(t.codes + rec * (nw * 4))[lane] = rw[lane];
  if (lane == 0) t.norm[rec] = f32_to_f16_bits(n);
}

template <int D, bool BF16>
cudaError_t run_fast(const FastQuantArgs &f, int sms, cudaStream_t s) {
  const unsigned nvec = f.t[0].nvec + (f.nbatch_total > f.t[0].nbatch ? f.t[1].nvec : 0u);
  if (f.nbatch_total < sms) { // fewer than one 128-vector batch per SM
    const unsigned blocks = (nvec + kQThreads / 32 - 1) / (kQThreads / 32);
    return launch_pdl(quantize_small_kernel<D, BF16>, dim3(blocks), dim3(kQThreads), 0, s, f);
  }
  const int smem = 2048 + 2 * kCells * 8 + 2 * kQThreads * (2 * D + 16); // 2048: alignment slack
  cudaError_t e = cudaFuncSetAttribute(quantize_fast_kernel<D, BF16>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const long long grid = std::min<long long>(f.nbatch_total, 3ll * sms);
  return launch_pdl(quantize_fast_kernel<D, BF16>, dim3(static_cast<unsigned>(grid)), dim3(kQThreads),
                    smem, s, f);
}

} // namespace

bool quantize_fast_supported(const QuantArgs &a) {
  if (a.t.mode != TQ_MSE || a.t.wbits < 1 || a.t.wbits > 4) return false;
  if (a.dtype != TQ_BF16 && a.dtype != TQ_F16) return false;
  if (a.d != 64 && a.d != 128) return false;
  if (static_cast<long long>(a.B) * a.Hkv * a.T >= (1ll << 32) - kQThreads) return false;
  // every cell of width 1/4 must hold at most one boundary, and all boundaries must lie
  // well inside the cell range [-32, 32)
  for (int j = 0; j + 1 < a.t.cb.levels; ++j) {
    if (std::fabs(a.t.cb.beta[j]) > 16.0f) return false;
    if (j > 0 && a.t.cb.beta[j] - a.t.cb.beta[j - 1] <= 0.25f) return false;
  }
  return true;
}

cudaError_t launch_quantize_fast(const QuantArgs *k, const QuantArgs *v, int sms, cudaStream_t s) {
  const QuantArgs *in[2] = {k, v};
  FastQuantArgs f{};
  const QuantArgs *first = k ? k : v;
  int nt = 0;
  for (int i = 0; i < 2; ++i) {
    if (!in[i]) continue;
    const QuantArgs &q = *in[i];
    FastTensor &t = f.t[nt++];
    t.x = static_cast<const uint8_t *>(q.x);
    t.codes = q.t.codes;
    t.norm = q.t.norm;
    t.nvec = static_cast<unsigned>(static_cast<long long>(q.B) * q.Hkv * q.T);
    t.nbatch = (t.nvec + kQThreads - 1) / kQThreads;
    t.T = q.T;
    t.T_cap = q.T_cap;
    t.t_offset = q.t_offset;
    t.wbits = q.t.wbits;
    t.code_bytes = q.t.code_bytes;
    t.nbeta = q.t.cb.levels - 1;
    for (int j = 0; j < t.nbeta; ++j) t.beta[j] = q.t.cb.beta[j];
  }
  if (nt == 0) return cudaSuccess;
  f.nbatch_total = f.t[0].nbatch + (nt == 2 ? f.t[1].nbatch : 0);
  const int d = first->d;
  for (int p = 0; p < d / 2; ++p) {
    f.sgn_lo[p] = ((first->sign_words[(2 * p) / 64] >> ((2 * p) % 64)) & 1ull) ? 0x80000000u : 0u;
    f.sgn_hi[p] = ((first->sign_words[(2 * p + 1) / 64] >> ((2 * p + 1) % 64)) & 1ull) ? 0x80000000u : 0u;
  }
  const bool bf16 = first->dtype == TQ_BF16;
  if (d == 128) return bf16 ? run_fast<128, true>(f, sms, s) : run_fast<128, false>(f, sms, s);
  return bf16 ? run_fast<64, true>(f, sms, s) : run_fast<64, false>(f, sms, s);
}

} // namespace tq
