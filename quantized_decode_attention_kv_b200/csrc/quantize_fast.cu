// Quantise-on-write for MSE records of 16-bit K/V ("Closing - The Three-Step Summary",
// Steps 1-3: norm, seeded-sign Walsh-Hadamard rotation, Lloyd-Max codes, LSB-first packing).
//
// Design (B200):
//  * head_dim 128 (quantize_mma_kernel): one warp quantises 16 vectors; the 16-point factor
//    of the Hadamard transform runs on the tensor cores, the 8-point factor in registers
//    (the kernel's own comment block below gives the index mapping).
//  * head_dim 64 (quantize_fast_kernel): persistent CTAs of 128 threads walk 128-vector
//    batches of K and then V in one launch. Each batch (128 x d 16-bit elements, contiguous
//    in memory) is copied into shared memory with coalesced 16-byte cp.async copies,
//    double-buffered so the next batch is in flight while this one is computed. Rows are
//    padded by 16 bytes so that the 16-byte row reads of one thread per vector never share a
//    bank. One thread owns one vector: the whole transform stays in registers. Coordinates are
//    held as packed fp32 pairs (x_j, x_{j+d/2}); the sum of squares and all but one of the
//    log2(d) butterfly stages run as Blackwell f32x2 instructions (two lanes of work per
//    instruction). Signs are applied while widening the 16-bit inputs (an add of 2^31 to the
//    fp32 bit pattern flips its sign).
//  * A few vectors (a decode step's new token): quantize_small_kernel, one warp per vector.
//  * Code search (all three): z is mapped to one of 256 cells of width 1/4 on the N(0,1)
//    scale with one fused multiply-add (the cell index lands in the low mantissa bits of a
//    float offset by 1.5 * 2^23); a shared-memory table gives, per cell, the number of
//    decision boundaries below it and the single boundary inside it (Lloyd-Max boundaries of
//    <= 4 bits are more than 1/4 apart), so every code costs one table read and one compare.
//    A zero vector maps to z = 0, whose cell holds the boundary 0, and gets the lower code as
//    a tie should.
#include "tq_device.cuh"

#include <type_traits>

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
  const int *bt; // paged cache: block table [B][maxp] (nullptr: dense [B][Hkv][T_cap] layout)
  int pshift, maxp, Hkv;
};

// Record index of new position tt of (b, KV head) bh: dense, or through the block table.
__device__ __forceinline__ size_t rec_index(const FastTensor &t, unsigned bh, unsigned tt) {
  const unsigned pos = static_cast<unsigned>(t.t_offset) + tt;
  if (!t.bt) return static_cast<size_t>(bh) * t.T_cap + pos;
  const unsigned b = bh / static_cast<unsigned>(t.Hkv), h = bh - b * static_cast<unsigned>(t.Hkv);
  const unsigned page = static_cast<unsigned>(__ldg(t.bt + static_cast<size_t>(b) * t.maxp + (pos >> t.pshift)));
  return ((static_cast<size_t>(page) * t.Hkv + h) << t.pshift) + (pos & ((1u << t.pshift) - 1u));
}

struct FastQuantArgs {
  FastTensor t[2];
  long long nbatch_total;
  // bit 31 set where D flips coordinate 2p (lo) / 2p + 1 (hi) of 16-bit pair p
  uint32_t sgn_lo[64], sgn_hi[64];
  uint32_t sbits[4]; // D's sign bits of coordinates 0..127 (bit j % 32 of word j / 32)
};

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
  const size_t rec = rec_index(t, bh, tt);
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
  const size_t rec = rec_index(t, bh, tt);
  if (lane < nw) reinterpret_cast<uint32_t *>(t.codes + rec * (nw * 4))[lane] = rw[lane];
  if (lane == 0) t.norm[rec] = f32_to_f16_bits(n);
}

// ---------------------------------------------------------------------------------------------
// Tensor-core variant for d = 128: one warp quantises 16 vectors at a time.
//
// The unnormalised Sylvester Hadamard matrix factors over the bits of the coordinate index,
// H_128 = H_S (x) H_T with S = bits 3..6 and T = bits 0..2. For each value j_T of the low bits
// (a "block" of 16 input coordinates 8 m + j_T, m = 0..15) one m16n8k16 MMA pair applies H_S:
// A = 16 vectors x the block's 16 coordinates (the 16-bit inputs with D's signs flipped),
// B = the 16 x 16 matrix of +-1. The 8-point transform over T then runs in registers.
// Lane (r, c) loads 16-byte chunks c, c+4, c+8, c+12 of vectors r and r+8 (k index
// k = 2c' + e + 8t' holds chunk c' + 4e + 8t'), and the output column n of its accumulators
// is mapped to coordinate bits so that after the 8-point stage the lane holds output
// coordinates [32c, 32c+32) of both vectors: packing and the record store stay lane-local.
template <bool BF16>
__device__ __forceinline__ void mma_pm1(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  if constexpr (BF16)
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, "
                 "{%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
                 : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
  else
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, "
                 "{%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
                 : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

__device__ __forceinline__ uint32_t prmt_b32(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Codes of one vector's 32 coordinates held by this lane (local index o = o_T + 8 e + 16 t),
// packed LSB-first into WB words, then stored at the lane's place in the record.
template <int WB>
__device__ __forceinline__ void mma_codes_store(const float (&acc)[8][2][4], int rho, float inv,
                                                uint32_t cells, uint8_t *dst) {
  uint32_t words[WB];
#pragma unroll
  for (int k = 0; k < WB; ++k) words[k] = 0u;
  const f2_t inv2 = f2(inv, inv);
  const f2_t cs2 = f2(kCellScale, kCellScale), cm2 = f2(kCellMagic, kCellMagic);
#pragma unroll
  for (int ot = 0; ot < 8; ++ot) {
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const f2_t z2 = mul2(f2(acc[ot][t][2 * rho], acc[ot][t][2 * rho + 1]), inv2);
      const f2_t u2 = fma2(z2, cs2, cm2);
      float z0, z1, u0, u1;
      f2_split(z2, z0, z1);
      f2_split(u2, u0, u1);
      const uint2 e0 = cell_entry(u0, cells);
      const uint2 e1 = cell_entry(u1, cells);
      put_code<WB>(words, ot + 16 * t, e0.y + (z0 > __uint_as_float(e0.x) ? 1u : 0u));
      put_code<WB>(words, ot + 8 + 16 * t, e1.y + (z1 > __uint_as_float(e1.x) ? 1u : 0u));
    }
  }
  if constexpr (WB == 4) {
    *reinterpret_cast<uint4 *>(dst) = make_uint4(words[0], words[1], words[2], words[3]);
  } else if constexpr (WB == 2) {
    *reinterpret_cast<uint2 *>(dst) = make_uint2(words[0], words[1]);
  } else {
#pragma unroll
    for (int k = 0; k < WB; ++k) reinterpret_cast<uint32_t *>(dst)[k] = words[k];
  }
}

constexpr int kMmaWarps = 4;

template <bool BF16>
__global__ void __launch_bounds__(kMmaWarps * 32, 3) quantize_mma_kernel(const FastQuantArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  const uint32_t pad = ((sbase + 2047u) & ~2047u) - sbase;
  uint8_t *cells = smem + pad;
  const uint32_t cells_s = sbase + pad;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = lane >> 2, c = lane & 3;

  // cell tables, as in the streaming kernel
  for (int idx = tid; idx < 2 * kCells; idx += kMmaWarps * 32) {
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

  // B fragments of H_S: element (k, n) = (-1)^popc(kappa(k) & sigma(n)), kappa(k) = the chunk
  // held at k, sigma(n) = output coordinate bits 3..6 of column n (bit 3 = n0, bit 4 = n3,
  // bit 5 = n1, bit 6 = n2)
  const uint32_t one = BF16 ? 0x3F80u : 0x3C00u;
  uint32_t hb[2][2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int n = 8 * t + r;
    const int sigma = (n & 1) | (((n >> 3) & 1) << 1) | (((n >> 1) & 1) << 2) | (((n >> 2) & 1) << 3);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t w = 0;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int k = 8 * h + 2 * c + e;
        const int kappa = ((k >> 1) & 3) | ((k & 1) << 2) | ((k >> 3) << 3);
        const uint32_t v = one | ((__popc(kappa & sigma) & 1) ? 0x8000u : 0u);
        w |= v << (16 * e);
      }
      hb[t][h] = w;
    }
  }
  // D's sign flips for the 16-bit pairs p of chunks c + 4 i (bit 15 / 31 of the XOR mask)
  uint32_t sg[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = c + 4 * i; // chunk: coordinates 8 m .. 8 m + 7
    const uint32_t byte = (a.sbits[m >> 2] >> (8 * (m & 3))) & 0xFFu;
#pragma unroll
    for (int p = 0; p < 4; ++p)
      sg[i][p] = (((byte >> (2 * p)) & 1u) << 15) | (((byte >> (2 * p + 1)) & 1u) << 31);
  }
  __syncthreads();
  pdl_wait(); // K/V may come from the kernel before; the cache may still be read by it
  pdl_trigger();

  const long long ng0 = (a.t[0].nvec + 15) / 16;
  const bool two = a.nbatch_total > a.t[0].nbatch;
  const long long ngt = ng0 + (two ? (a.t[1].nvec + 15) / 16 : 0);
  const long long stride = static_cast<long long>(gridDim.x) * kMmaWarps;
  long long g = static_cast<long long>(blockIdx.x) * kMmaWarps + warp;

  uint4 R[2][4]; // [row r / r+8][chunk c + 4 i]
  auto load = [&](long long gg) {
    const int ti = gg < ng0 ? 0 : 1;
    const FastTensor &t = a.t[ti];
    const unsigned v0 = static_cast<unsigned>((gg - (ti ? ng0 : 0)) * 16);
#pragma unroll
    for (int rho = 0; rho < 2; ++rho) {
      const unsigned v = min(v0 + r + 8 * rho, t.nvec - 1);
      const uint4 *src = reinterpret_cast<const uint4 *>(t.x + static_cast<size_t>(v) * 256) + c;
#pragma unroll
      for (int i = 0; i < 4; ++i) R[rho][i] = __ldcs(src + 4 * i);
    }
  };

  // One phase per tensor (K, then V) with its bit width fixed at compile time; the next
  // group's loads are issued after this group's MMAs (they may belong to the next phase).
  auto phase = [&](auto ti_tag, auto wb_tag, long long gend) {
    constexpr int TI = decltype(ti_tag)::value, WB = decltype(wb_tag)::value;
    const FastTensor &t = a.t[TI];
    const uint32_t cl = cells_s + TI * kCells * 8;
    const unsigned T = static_cast<unsigned>(t.T);
    for (; g < gend; g += stride) {
      const unsigned v0 = static_cast<unsigned>((g - (TI ? ng0 : 0)) * 16);

      // ---- H_S on the tensor cores, one block j_T per MMA pair
      uint32_t X[2][4][4];
#pragma unroll
      for (int rho = 0; rho < 2; ++rho)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          X[rho][i][0] = R[rho][i].x ^ sg[i][0];
          X[rho][i][1] = R[rho][i].y ^ sg[i][1];
          X[rho][i][2] = R[rho][i].z ^ sg[i][2];
          X[rho][i][3] = R[rho][i].w ^ sg[i][3];
        }
      float acc[8][2][4];
#pragma unroll
      for (int jt = 0; jt < 8; ++jt) {
        const int p = jt >> 1;
        const uint32_t sel = (jt & 1) ? 0x7632u : 0x5410u;
        const uint32_t a0 = prmt_b32(X[0][0][p], X[0][1][p], sel);
        const uint32_t a1 = prmt_b32(X[1][0][p], X[1][1][p], sel);
        const uint32_t a2 = prmt_b32(X[0][2][p], X[0][3][p], sel);
        const uint32_t a3 = prmt_b32(X[1][2][p], X[1][3][p], sel);
        mma_pm1<BF16>(acc[jt][0], a0, a1, a2, a3, hb[0][0], hb[0][1]);
        mma_pm1<BF16>(acc[jt][1], a0, a1, a2, a3, hb[1][0], hb[1][1]);
      }
      if (g + stride < ngt) load(g + stride);

      // ---- H_T: 8-point butterflies over the blocks, per (n-tile, accumulator pair)
#pragma unroll
      for (int t2 = 0; t2 < 2; ++t2)
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          f2_t y[8];
#pragma unroll
          for (int jt = 0; jt < 8; ++jt) y[jt] = f2(acc[jt][t2][2 * q], acc[jt][t2][2 * q + 1]);
#pragma unroll
          for (int h = 1; h < 8; h <<= 1)
#pragma unroll
            for (int jt = 0; jt < 8; ++jt)
              if ((jt & h) == 0) {
                const f2_t u = y[jt], w = y[jt + h];
                y[jt] = add2(u, w);
                y[jt + h] = sub2(u, w);
              }
#pragma unroll
          for (int jt = 0; jt < 8; ++jt) f2_split(y[jt], acc[jt][t2][2 * q], acc[jt][t2][2 * q + 1]);
        }

      // ---- norms: ||H D x||^2 = 128 ||x||^2, summed over the 4 lanes of each vector
      f2_t s2a = 0ull, s2b = 0ull;
#pragma unroll
      for (int jt = 0; jt < 8; ++jt)
#pragma unroll
        for (int t2 = 0; t2 < 2; ++t2) {
          const f2_t ya = f2(acc[jt][t2][0], acc[jt][t2][1]);
          const f2_t yb = f2(acc[jt][t2][2], acc[jt][t2][3]);
          s2a = fma2(ya, ya, s2a);
          s2b = fma2(yb, yb, s2b);
        }
      float sa0, sa1, sb0, sb1;
      f2_split(s2a, sa0, sa1);
      f2_split(s2b, sb0, sb1);
      float sa = sa0 + sa1, sb = sb0 + sb1;
      sa += __shfl_xor_sync(0xffffffffu, sa, 1);
      sb += __shfl_xor_sync(0xffffffffu, sb, 1);
      sa += __shfl_xor_sync(0xffffffffu, sa, 2);
      sb += __shfl_xor_sync(0xffffffffu, sb, 2);

      // record of vector v0 (the group's first), then of this lane's rows
      const unsigned bh0 = v0 / T, tt0 = v0 - bh0 * T;
#pragma unroll
      for (int rho = 0; rho < 2; ++rho) {
        const unsigned v = v0 + r + 8 * rho;
        unsigned bh = bh0, tt = tt0 + r + 8 * rho;
        while (tt >= T) { // T < 16 wraps more than once
          tt -= T;
          ++bh;
        }
        const float n = sqrtf((rho ? sb : sa) * (1.0f / 128.0f));
        const float inv = n > 0.f ? __frcp_rn(n) : 0.0f;
        if (v < t.nvec) {
          const size_t rec = rec_index(t, bh, tt);
          mma_codes_store<WB>(acc, rho, inv, cl, t.codes + rec * (16 * WB) + c * (4 * WB));
          if (c == 0) t.norm[rec] = f32_to_f16_bits(n);
        }
      }
    }
  };
  using I0 = std::integral_constant<int, 0>;
  using I1 = std::integral_constant<int, 1>;
  if (g < ngt) load(g);
  switch (a.t[0].wbits) {
  case 1: phase(I0{}, std::integral_constant<int, 1>{}, ng0); break;
  case 2: phase(I0{}, std::integral_constant<int, 2>{}, ng0); break;
  case 3: phase(I0{}, std::integral_constant<int, 3>{}, ng0); break;
  default: phase(I0{}, std::integral_constant<int, 4>{}, ng0); break;
  }
  if (two) {
    switch (a.t[1].wbits) {
    case 1: phase(I1{}, std::integral_constant<int, 1>{}, ngt); break;
    case 2: phase(I1{}, std::integral_constant<int, 2>{}, ngt); break;
    case 3: phase(I1{}, std::integral_constant<int, 3>{}, ngt); break;
    default: phase(I1{}, std::integral_constant<int, 4>{}, ngt); break;
    }
  }
}

template <int D, bool BF16>
cudaError_t run_fast(const FastQuantArgs &f, int sms, cudaStream_t s) {
  const unsigned nvec = f.t[0].nvec + (f.nbatch_total > f.t[0].nbatch ? f.t[1].nvec : 0u);
  if (f.nbatch_total < sms) { // fewer than one 128-vector batch per SM
    const unsigned blocks = (nvec + kQThreads / 32 - 1) / (kQThreads / 32);
    return launch_pdl(quantize_small_kernel<D, BF16>, dim3(blocks), dim3(kQThreads), 0, s, f);
  }
  if constexpr (D == 128) {
    const unsigned ngt = (f.t[0].nvec + 15) / 16 +
                         (f.nbatch_total > f.t[0].nbatch ? (f.t[1].nvec + 15) / 16 : 0u);
    const int msmem = 2048 + 2 * kCells * 8;
    const long long grid = std::min<long long>((ngt + kMmaWarps - 1) / kMmaWarps, 3ll * sms);
    return launch_pdl(quantize_mma_kernel<BF16>, dim3(static_cast<unsigned>(grid)),
                      dim3(kMmaWarps * 32), msmem, s, f);
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
  // the cell-table code search needs adjacent boundaries more than one cell (1/4) apart: true
  // of every Lloyd-Max codebook of <= 4 bits, not of the E2M1 grid near zero
  for (int j = 0; j + 2 < a.t.cb.levels; ++j)
    if (a.t.cb.beta[j + 1] - a.t.cb.beta[j] <= 0.25f) return false;
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
    t.bt = q.pg.bt;
    t.pshift = q.pg.pshift;
    t.maxp = q.pg.maxp;
    t.Hkv = q.Hkv;
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
  for (int k = 0; k < 4; ++k)
    f.sbits[k] = static_cast<uint32_t>(first->sign_words[k / 2] >> (32 * (k & 1)));
  const bool bf16 = first->dtype == TQ_BF16;
  if (d == 128) return bf16 ? run_fast<128, true>(f, sms, s) : run_fast<128, false>(f, sms, s);
  return bf16 ? run_fast<64, true>(f, sms, s) : run_fast<64, false>(f, sms, s);
}

} // namespace tq
