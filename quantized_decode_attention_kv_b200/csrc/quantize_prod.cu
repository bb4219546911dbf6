// Quantise-on-write for TurboQuant_prod records of head_dim 64 with a 64-row QJL sketch and
// 1- or 2-bit records ("Closing - The Three-Step Summary", Steps 1-3: rotate, 1-bit Lloyd-Max
// code, then the sign sketch of the residual; "What the Paper Doesn't Tell You", Finding 2).
//
// The sketch s = sign(S r) is a 64 x 64 matrix-vector product per vector, i.e. a GEMM over a
// batch of vectors, so it runs on the tensor cores (mma.sync m16n8k16, fp16 x fp16 -> fp32):
// a warp takes 16 vectors at a time; the residuals form the A operand and S^T the B operand,
// both split into an fp16 part and a 2^12-scaled fp16 residual, and the three significant
// products (hi hi, lo hi, hi lo) give the projections to ~2^-21 relative, well inside the
// 1e-5 ||r|| band where a sign may legitimately differ from a float64 evaluation.
//
// Lane (r, c) of a warp owns coordinates [16 c, 16 c + 16) of vectors r and r + 8 of the
// group: the Walsh-Hadamard butterflies of spans 1..8 run in registers, spans 16 and 32 across
// the four lanes of a row with shuffles; norms and residual norms are reduced the same way.
// The lane's residual slice is already the A-operand layout once the contraction index is
// permuted (k-step s takes coordinates 16 c + 4 s .. + 3); the B fragments of S for that
// permutation are built once per CTA in shared memory.
#include "mma_ops.cuh"
#include "tc_ops.cuh"

#include <type_traits>

namespace tq {
namespace {
using namespace mma_ops;

constexpr int kRD = 64, kRM = 64;
constexpr int kRWarps = 4;
constexpr float kRLo = 4096.0f, kRLoInv = 1.0f / 4096.0f;

struct ProdQuantTensor {
  const uint8_t *x; // [nvec][64] 16-bit elements
  uint8_t *codes, *signs;
  uint16_t *norm, *rnorm;
  const float *S; // [64][64]
  unsigned nvec;
  int T, T_cap, t_offset, wbits;
  float c1;      // the positive 1-bit centroid (wbits = 1)
  const int *bt; // paged cache: block table [B][maxp] (nullptr: dense [B][Hkv][T_cap] layout)
  int pshift, maxp, Hkv;
};

// Record index of new position tt of (b, KV head) bh: dense, or through the block table.
__device__ __forceinline__ size_t prod_rec(const ProdQuantTensor &t, unsigned bh, unsigned tt) {
  const unsigned pos = static_cast<unsigned>(t.t_offset) + tt;
  if (!t.bt) return static_cast<size_t>(bh) * t.T_cap + pos;
  const unsigned b = bh / static_cast<unsigned>(t.Hkv), h = bh - b * static_cast<unsigned>(t.Hkv);
  const unsigned page = static_cast<unsigned>(__ldg(t.bt + static_cast<size_t>(b) * t.maxp + (pos >> t.pshift)));
  return ((static_cast<size_t>(page) * t.Hkv + h) << t.pshift) + (pos & ((1u << t.pshift) - 1u));
}

struct ProdQuantArgs {
  ProdQuantTensor t[2];
  int ntensors;
  long long groups[2]; // 16-vector groups per tensor
  uint64_t sign_word;  // SplitMix64 output 0 of the seed: bit i set <=> D_ii = -1
};

__device__ __forceinline__ uint32_t h2bits(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }

// fp16 hi pair and 2^12-scaled fp16 residual pair of (a, b)
__device__ __forceinline__ void split2(float a, float b, uint32_t &hi, uint32_t &lo) {
  const __half2 h = __floats2half2_rn(a, b);
  const float2 f = __half22float2(h);
  hi = h2bits(h);
  lo = h2bits(__floats2half2_rn((a - f.x) * kRLo, (b - f.y) * kRLo));
}

template <bool BF16>
__device__ __forceinline__ void mma_x(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                      uint32_t b0, uint32_t b1) {
  if constexpr (BF16)
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, "
                 "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  else
    mma16816(d, a0, a1, a2, a3, b0, b1);
}

// The lane (r, c) loads 16-byte chunks c and c + 4 (coordinates 8 m .. 8 m + 7) of vectors r
// and r + 8; register q of chunk h is the A-operand register of k-step 2 h + (q >> 1) (a0 for
// even q, a2 for odd q). Input coordinate held at k-step s, k index k (0..15):
__host__ __device__ constexpr int prod_in_coord(int s, int k) {
  return 32 * (s >> 1) + 8 * ((k & 7) >> 1) + 4 * (s & 1) + 2 * (k >> 3) + (k & 1);
}

template <bool BF16>
__global__ void __launch_bounds__(kRWarps * 32, 3) quantize_prod_kernel(const ProdQuantArgs a) {
  // B fragments: hfrag[k-step 4][n-tile 8][lane] {b0, b1} of (H D)^T, i.e. element (k, n) =
  // H[n][j] D[j] with j the input coordinate at (s, k) (exact +-1 in the input's 16-bit type);
  // sfrag[tensor][n-tile 8][k-step 4][lane] {b0 hi, b1 hi, b0 lo, b1 lo} of S^T, element
  // (k, j) = S[j][16 s + k] (the z accumulators of n-tiles 2 s and 2 s + 1 are k-step s's A).
  __shared__ uint2 hfrag[4][8][32];
  __shared__ uint4 sfrag[2][8][4][32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = lane >> 2, c = lane & 3;
  const uint32_t one = BF16 ? 0x3F80u : 0x3C00u;
  for (int idx = tid; idx < 4 * 8 * 32; idx += kRWarps * 32) {
    const int s = idx / 256, nt = (idx / 32) % 8, l = idx % 32;
    const int n = 8 * nt + (l >> 2), lc = l & 3;
    uint32_t w[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t v = 0;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int j = prod_in_coord(s, 8 * h + 2 * lc + e);
        const bool neg = ((__popc(n & j) & 1) != 0) != (((a.sign_word >> j) & 1ull) != 0);
        v |= (one | (neg ? 0x8000u : 0u)) << (16 * e);
      }
      w[h] = v;
    }
    hfrag[s][nt][l] = make_uint2(w[0], w[1]);
  }
  for (int idx = tid; idx < a.ntensors * 8 * 4 * 32; idx += kRWarps * 32) {
    const int ti = idx / 1024, rest = idx % 1024;
    const int nt = rest / 128, s = (rest / 32) % 4, l = rest % 32;
    const float *row = a.t[ti].S + static_cast<size_t>(8 * nt + (l >> 2)) * kRD + 16 * s + 2 * (l & 3);
    uint4 f;
    split2(row[0], row[1], f.x, f.z);
    split2(row[8], row[9], f.y, f.w);
    sfrag[ti][nt][s][l] = f;
  }
  __syncthreads();
  pdl_wait(); // K/V may come from the kernel before; the cache may still be read by it
  pdl_trigger();

  const long long g0 = a.groups[0];
  const long long total = g0 + (a.ntensors > 1 ? a.groups[1] : 0);
  const long long stride = static_cast<long long>(gridDim.x) * kRWarps;
  long long gi = static_cast<long long>(blockIdx.x) * kRWarps + warp;

  uint4 R[2][2]; // [vector r / r + 8][chunk c / c + 4]
  auto load = [&](long long g) {
    const int ti = g < g0 ? 0 : 1;
    const ProdQuantTensor &t = a.t[ti];
    const unsigned v0 = static_cast<unsigned>((g - (ti ? g0 : 0)) * 16);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const unsigned v = min(v0 + r + 8 * u, t.nvec - 1);
      const uint4 *src = reinterpret_cast<const uint4 *>(t.x + static_cast<size_t>(v) * (2 * kRD)) + c;
      R[u][0] = __ldcs(src);
      R[u][1] = __ldcs(src + 4);
    }
  };

  // One phase per tensor with its record bit width fixed at compile time.
  auto phase = [&](auto ti_tag, auto wb_tag, long long gend) {
    constexpr int TI = decltype(ti_tag)::value, WB = decltype(wb_tag)::value;
    const ProdQuantTensor &t = a.t[TI];
    const unsigned T = static_cast<unsigned>(t.T);
    const float c1 = t.c1;
    for (; gi < gend; gi += stride) {
      const unsigned v0 = static_cast<unsigned>((gi - (TI ? g0 : 0)) * 16);
      // ---- z = H D x on the tensor cores (exact products, fp32 accumulation)
      float z[8][4];
      {
        uint32_t A[2][8];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          A[u][0] = R[u][0].x; A[u][1] = R[u][0].y; A[u][2] = R[u][0].z; A[u][3] = R[u][0].w;
          A[u][4] = R[u][1].x; A[u][5] = R[u][1].y; A[u][6] = R[u][1].z; A[u][7] = R[u][1].w;
        }
        if (gi + stride < total) load(gi + stride);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          z[nt][0] = z[nt][1] = z[nt][2] = z[nt][3] = 0.f;
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            const uint2 b = hfrag[s][nt][lane];
            mma_x<BF16>(z[nt], A[0][2 * s], A[1][2 * s], A[0][2 * s + 1], A[1][2 * s + 1], b.x, b.y);
          }
        }
      }
      // ---- norms (||H D x||^2 = 64 ||x||^2), codes, residuals r = (z - c^) / sqrt(64)
      float ss[2] = {0.f, 0.f};
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          ss[u] = fmaf(z[nt][2 * u], z[nt][2 * u], ss[u]);
          ss[u] = fmaf(z[nt][2 * u + 1], z[nt][2 * u + 1], ss[u]);
        }
      float inv[2], nrm[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], 1);
        ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], 2);
        nrm[u] = sqrtf(ss[u] * (1.0f / 64.0f));
        inv[u] = nrm[u] > 0.f ? __frcp_rn(nrm[u]) : 0.0f;
      }
      uint32_t cw[2][2] = {{0u, 0u}, {0u, 0u}}; // [vector][word] code bits
      float rr[2] = {0.f, 0.f};
      uint32_t ahi[2][8], alo[2][8]; // S r A operands: [vector][2 s + (a0 | a2)]
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          float res[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float zz = z[nt][2 * u + e] * inv[u];
            float chat = 0.f;
            if constexpr (WB == 1) {
              const bool up = zz > 0.f;
              cw[u][nt >> 2] |= (up ? 1u : 0u) << (8 * (nt & 3) + 2 * c + e);
              chat = up ? c1 : -c1;
            }
            res[e] = (zz - chat) * 0.125f;
            rr[u] = fmaf(res[e], res[e], rr[u]);
          }
          split2(res[0], res[1], ahi[u][nt], alo[u][nt]);
        }
      float gam[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        rr[u] += __shfl_xor_sync(0xffffffffu, rr[u], 1);
        rr[u] += __shfl_xor_sync(0xffffffffu, rr[u], 2);
        gam[u] = sqrtf(rr[u]);
      }
      // ---- sketch S r: three-term fp16 split; bit j = 1 iff (S r)_j < 0
      uint32_t sg[2][2] = {{0u, 0u}, {0u, 0u}};
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        float m0[4] = {0.f, 0.f, 0.f, 0.f}, m1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint4 f = sfrag[TI][nt][s][lane];
          mma16816(m0, ahi[0][2 * s], ahi[1][2 * s], ahi[0][2 * s + 1], ahi[1][2 * s + 1], f.x, f.y);
          mma16816(m1, alo[0][2 * s], alo[1][2 * s], alo[0][2 * s + 1], alo[1][2 * s + 1], f.x, f.y);
          mma16816(m1, ahi[0][2 * s], ahi[1][2 * s], ahi[0][2 * s + 1], ahi[1][2 * s + 1], f.z, f.w);
        }
        const int sh = 8 * (nt & 3) + 2 * c, wi = nt >> 2;
        const float p00 = fmaf(m1[0], kRLoInv, m0[0]), p01 = fmaf(m1[1], kRLoInv, m0[1]);
        const float p10 = fmaf(m1[2], kRLoInv, m0[2]), p11 = fmaf(m1[3], kRLoInv, m0[3]);
        // sign bit = (p < 0): the accumulators start at +0, so an exact zero is +0 (bit 0)
        sg[0][wi] |= ((__float_as_uint(p00) >> 31) | ((__float_as_uint(p01) >> 31) << 1)) << sh;
        sg[1][wi] |= ((__float_as_uint(p10) >> 31) | ((__float_as_uint(p11) >> 31) << 1)) << sh;
      }
      // OR the four lanes of each vector: sign words, code words
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int wi = 0; wi < 2; ++wi) {
          sg[u][wi] |= __shfl_xor_sync(0xffffffffu, sg[u][wi], 1);
          sg[u][wi] |= __shfl_xor_sync(0xffffffffu, sg[u][wi], 2);
          if constexpr (WB == 1) {
            cw[u][wi] |= __shfl_xor_sync(0xffffffffu, cw[u][wi], 1);
            cw[u][wi] |= __shfl_xor_sync(0xffffffffu, cw[u][wi], 2);
          }
        }
      // ---- stores: lane c = 0 writes vector r, lane c = 1 vector r + 8
      if (c < 2) {
        const int u = c;
        const unsigned v = v0 + r + 8 * u;
        if (v < t.nvec) {
          const unsigned bh0 = v0 / T;
          unsigned bh = bh0, tt = v0 - bh0 * T + r + 8 * u;
          while (tt >= T) { // T < 16 wraps more than once
            tt -= T;
            ++bh;
          }
          const size_t rec = prod_rec(t, bh, tt);
          const uint32_t s0 = u ? sg[1][0] : sg[0][0], s1 = u ? sg[1][1] : sg[0][1];
          reinterpret_cast<uint2 *>(t.signs)[rec] = make_uint2(s0, s1);
          if constexpr (WB == 1)
            reinterpret_cast<uint2 *>(t.codes)[rec] = make_uint2(u ? cw[1][0] : cw[0][0], u ? cw[1][1] : cw[0][1]);
          t.norm[rec] = f32_to_f16_bits(u ? nrm[1] : nrm[0]);
          t.rnorm[rec] = f32_to_f16_bits(u ? gam[1] : gam[0]);
        }
      }
    }
  };
  using I0 = std::integral_constant<int, 0>;
  using I1 = std::integral_constant<int, 1>;
  if (gi < total) load(gi);
  if (a.t[0].wbits == 1) phase(I0{}, I1{}, g0);
  else phase(I0{}, I0{}, g0);
  if (a.ntensors > 1) {
    if (a.t[1].wbits == 1) phase(I1{}, I1{}, total);
    else phase(I1{}, I0{}, total);
  }
}

// ---------------------------------------------------------------------------------------------
// tcgen05 variant for bulk writes: one CTA of 128 threads quantises tiles of 128 vectors, one
// thread per vector (row m of every MMA tile is vector m of the tile).
//
//   z   = X (H D)^T      M = 128 vectors, N = 64, K = 64: the 16-bit inputs against the exact
//                        +-1 matrix H D (same 16-bit type), fp32 accumulator in TMEM
//   S r = r S^T          three-term fp16 split, all into one TMEM accumulator: first
//                        r_lo S_hi^T + r_hi S_lo^T (both lo parts scaled by 2^12), then
//                        r_hi S_hi^T with the accumulator scaled by 2^-12 on the way in
//
// Thread m reads its own TMEM lane (row m) back, so the norm, the 1-bit codes, the residual,
// its norm, the hi/lo split and the packing of codes and sketch signs are all thread-local.
// Operands sit in shared memory in the canonical K-major layout of tc_ops.cuh. Every wait on
// the tensor cores is bounded; on a timeout the CTA records a fault bit, frees its TMEM and
// returns.
constexpr int kTcRows = 128;
constexpr uint32_t kTcCols = 64;                 // TMEM columns: z, then the sketch
constexpr int kTcX = 0, kTcAH = 16384, kTcAL = 32768, kTcHB = 49152, kTcSH = 57344, kTcSL = 65536;
constexpr int kTcBar = 73728;                    // two mbarriers, then the TMEM address slot
constexpr int kTcSmem = kTcBar + 32 + 1024;      // + alignment slack
constexpr long long kTcWaitCycles = 2000000000ll; // about one second

__device__ unsigned int g_prod_tc_fault; // bit 0: a tensor-core wait timed out

template <bool BF16>
__global__ void __launch_bounds__(kTcRows, 3) quantize_prod_tc_kernel(const ProdQuantArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint32_t sraw = tc::smem_addr(smem_raw);
  const uint32_t sbase = (sraw + 1023u) & ~1023u;
  uint8_t *sm = smem_raw + (sbase - sraw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t mbar0 = sbase + kTcBar, mbar1 = sbase + kTcBar + 8, tslot = sbase + kTcBar + 16;

  // (H D)^T as the B operand of z: element (n, k) = H[n][k] D[k], exact +-1
  {
    const uint16_t one = BF16 ? 0x3F80u : 0x3C00u;
    for (int idx = tid; idx < kRD * kRD; idx += kTcRows) {
      const int n = idx >> 6, k = idx & 63;
      const bool neg = ((__popc(n & k) & 1) != 0) != (((a.sign_word >> k) & 1ull) != 0);
      *reinterpret_cast<uint16_t *>(sm + kTcHB + tc::kmajor_offset(n, k, kRD)) =
          static_cast<uint16_t>(one | (neg ? 0x8000u : 0u));
    }
  }
  // S of one tensor as hi / 2^12-scaled lo fp16 B operands: element (j, k) = S[j][k]
  auto build_s = [&](int ti) {
    const float *S = a.t[ti].S;
    for (int idx = tid; idx < kRM * kRD; idx += kTcRows) {
      const int j = idx >> 6, k = idx & 63;
      const float v = S[idx];
      const __half h = __float2half_rn(v);
      const __half l = __float2half_rn((v - __half2float(h)) * kRLo);
      const uint32_t off = tc::kmajor_offset(j, k, kRD);
      *reinterpret_cast<__half *>(sm + kTcSH + off) = h;
      *reinterpret_cast<__half *>(sm + kTcSL + off) = l;
    }
  };
  build_s(0);
  if (warp == 0) tc::tmem_alloc(tslot, kTcCols);
  if (tid == 0) {
    tc::mbar_init(mbar0, 1);
    tc::mbar_init(mbar1, 1);
    tc::mbar_init_fence();
  }
  tc::fence_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + kTcBar + 16);
  const uint32_t tlane = tmem + (static_cast<uint32_t>(32 * warp) << 16); // this warp's lanes
  pdl_wait(); // K/V may come from the kernel before; the cache may still be read by it
  pdl_trigger();

  const long long nt0 = (a.t[0].nvec + kTcRows - 1) / kTcRows;
  const long long ntt = nt0 + (a.ntensors > 1 ? (a.t[1].nvec + kTcRows - 1) / kTcRows : 0);
  // cp.async of a tile: chunk (row, kc) of 16 bytes; per instruction a warp covers 8 rows x
  // 4 chunks (64 contiguous bytes per row, 512 distinct shared bytes)
  auto issue = [&](long long tile) {
    const int ti = tile < nt0 ? 0 : 1;
    const ProdQuantTensor &t = a.t[ti];
    const unsigned v0 = static_cast<unsigned>((tile - (ti ? nt0 : 0)) * kTcRows);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int row = (j >> 1) * 32 + warp * 8 + (lane & 7);
      const int kc = (j & 1) * 4 + (lane >> 3);
      const unsigned v = min(v0 + row, t.nvec - 1);
      const uint8_t *src = t.x + static_cast<size_t>(v) * (2 * kRD) + kc * 16;
      const uint32_t dst = sbase + kTcX + tc::kmajor_offset(row, 8 * kc, kRD);
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  const uint32_t id_z = tc::idesc_f16(kTcRows, kRM, BF16);
  const uint32_t id_s = tc::idesc_f16(kTcRows, kRM, false);
  auto dsc = [&](int off, int s) { return tc::desc_kmajor(sbase + off + 256 * s, 128, 1024); };

  long long tile = blockIdx.x;
  uint32_t ph = 0;
  bool fault = false;
  // One phase per tensor, the record bit width a compile-time constant.
  auto phase = [&](auto ti_tag, auto wb_tag, long long tend) {
    constexpr int TI = decltype(ti_tag)::value, WB = decltype(wb_tag)::value;
    const ProdQuantTensor &t = a.t[TI];
    const unsigned T = static_cast<unsigned>(t.T);
    const uint32_t c18 = __float_as_uint(t.c1 * 0.125f);
    for (; tile < tend; tile += gridDim.x) {
      const unsigned v0 = static_cast<unsigned>((tile - (TI ? nt0 : 0)) * kTcRows);
      asm volatile("cp.async.wait_all;" ::: "memory");
      tc::fence_async_smem();
      tc::fence_before_sync();
      __syncthreads();
      tc::fence_after_sync();
      // ---- z = X (H D)^T
      if (tid == 0) {
#pragma unroll
        for (int s = 0; s < 4; ++s) tc::mma_ss(tmem, dsc(kTcX, s), dsc(kTcHB, s), id_z, s > 0);
        tc::commit(mbar0);
      }
      bool ok = tc::mbar_wait(mbar0, ph, kTcWaitCycles);
      if (__syncthreads_or(!ok)) {
        fault = true;
        return;
      }
      tc::fence_after_sync();
      if (tile + gridDim.x < ntt) issue(tile + gridDim.x); // X is free again
      f2_t z[32];
      {
        float h0[32], h1[32];
        tc::tmem_ld32(tlane, h0);
        tc::tmem_ld32(tlane + 32, h1);
        tc::tmem_wait_ld();
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          z[p] = f2(h0[2 * p], h0[2 * p + 1]);
          z[16 + p] = f2(h1[2 * p], h1[2 * p + 1]);
        }
      }
      // ---- norm, codes (bit k = z_k > 0), residual r = (z - c^) / 8, its norm, hi/lo split
      f2_t ss2 = 0ull;
#pragma unroll
      for (int p = 0; p < 32; ++p) ss2 = fma2(z[p], z[p], ss2);
      float s0, s1;
      f2_split(ss2, s0, s1);
      const float nrm = sqrtf((s0 + s1) * (1.0f / 64.0f)); // ||H D x||^2 = 64 ||x||^2
      const float inv = nrm > 0.f ? __frcp_rn(nrm) : 0.0f;
      const f2_t inv2 = f2(inv, inv), inv82 = f2(inv * 0.125f, inv * 0.125f);
      const f2_t tiny2 = f2(-0x1p-149f, -0x1p-149f);
      uint32_t cw[2] = {0u, 0u}, rh[32], rl[32];
      f2_t rr2 = 0ull;
#pragma unroll
      for (int p = 31; p >= 0; --p) {
        f2_t negc2 = 0ull;
        if constexpr (WB == 1) {
          // the sign of z inv - 2^-149 is clear exactly when z inv > 0 (inv >= 0)
          float za, zb;
          f2_split(fma2(z[p], inv2, tiny2), za, zb);
          cw[p >> 4] = __funnelshift_l(__float_as_uint(zb), cw[p >> 4], 1);
          cw[p >> 4] = __funnelshift_l(__float_as_uint(za), cw[p >> 4], 1);
          negc2 = f2(__uint_as_float(c18 | (~__float_as_uint(za) & 0x80000000u)),
                     __uint_as_float(c18 | (~__float_as_uint(zb) & 0x80000000u)));
        }
        const f2_t r2 = fma2(z[p], inv82, negc2); // unit-domain residual / sqrt(64)
        rr2 = fma2(r2, r2, rr2);
        float ra, rb;
        f2_split(r2, ra, rb);
        split2(ra, rb, rh[p], rl[p]);
      }
#pragma unroll
      for (int kc = 0; kc < 8; ++kc) {
        const uint32_t off = tc::kmajor_offset(tid, 8 * kc, kRD);
        *reinterpret_cast<uint4 *>(sm + kTcAH + off) = make_uint4(rh[4 * kc], rh[4 * kc + 1], rh[4 * kc + 2], rh[4 * kc + 3]);
        *reinterpret_cast<uint4 *>(sm + kTcAL + off) = make_uint4(rl[4 * kc], rl[4 * kc + 1], rl[4 * kc + 2], rl[4 * kc + 3]);
      }
      tc::fence_async_smem();
      tc::fence_before_sync();
      __syncthreads();
      tc::fence_after_sync();
      // ---- S r: lo terms, then hi x hi with the lo terms scaled by 2^-12
      if (tid == 0) {
#pragma unroll
        for (int s = 0; s < 4; ++s) tc::mma_ss(tmem, dsc(kTcAL, s), dsc(kTcSH, s), id_s, s > 0);
#pragma unroll
        for (int s = 0; s < 4; ++s) tc::mma_ss(tmem, dsc(kTcAH, s), dsc(kTcSL, s), id_s, 1);
        tc::mma_ss_scaled<12>(tmem, dsc(kTcAH, 0), dsc(kTcSH, 0), id_s);
#pragma unroll
        for (int s = 1; s < 4; ++s) tc::mma_ss(tmem, dsc(kTcAH, s), dsc(kTcSH, s), id_s, 1);
        tc::commit(mbar1);
      }
      ok = tc::mbar_wait(mbar1, ph, kTcWaitCycles);
      if (__syncthreads_or(!ok)) {
        fault = true;
        return;
      }
      tc::fence_after_sync();
      ph ^= 1u;
      uint32_t sg[2] = {0u, 0u};
      {
        float p0[32], p1[32];
        tc::tmem_ld32(tlane, p0);
        tc::tmem_ld32(tlane + 32, p1);
        tc::tmem_wait_ld();
        // bit j = (S r)_j < 0 (sign bit; an exact zero of a sum of products is +0)
#pragma unroll
        for (int j = 31; j >= 0; --j) {
          sg[0] = __funnelshift_l(__float_as_uint(p0[j]), sg[0], 1);
          sg[1] = __funnelshift_l(__float_as_uint(p1[j]), sg[1], 1);
        }
      }
      float q0, q1;
      f2_split(rr2, q0, q1);
      const unsigned v = v0 + tid;
      if (v < t.nvec) {
        const unsigned bh = v / T, tt = v - bh * T;
        const size_t rec = prod_rec(t, bh, tt);
        reinterpret_cast<uint2 *>(t.signs)[rec] = make_uint2(sg[0], sg[1]);
        if constexpr (WB == 1) reinterpret_cast<uint2 *>(t.codes)[rec] = make_uint2(~cw[0], ~cw[1]);
        t.norm[rec] = f32_to_f16_bits(nrm);
        t.rnorm[rec] = f32_to_f16_bits(sqrtf(q0 + q1));
      }
    }
  };
  using I0 = std::integral_constant<int, 0>;
  using I1 = std::integral_constant<int, 1>;
  if (tile < ntt) issue(tile);
  if (a.t[0].wbits == 1) phase(I0{}, I1{}, nt0);
  else phase(I0{}, I0{}, nt0);
  if (!fault && a.ntensors > 1) {
    build_s(1); // every MMA on the first tensor's sketch has completed
    if (a.t[1].wbits == 1) phase(I1{}, I1{}, ntt);
    else phase(I1{}, I0{}, ntt);
  }
  if (fault && tid == 0) atomicOr(&g_prod_tc_fault, 1u);
  asm volatile("cp.async.wait_all;" ::: "memory"); // own copies in flight
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, kTcCols);
}

} // namespace

cudaError_t read_and_clear_prod_faults(unsigned *flags) {
  unsigned v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_prod_tc_fault, sizeof(v));
  if (e != cudaSuccess) return e;
  const unsigned zero = 0;
  e = cudaMemcpyToSymbol(g_prod_tc_fault, &zero, sizeof(zero));
  if (flags) *flags = v;
  return e;
}

bool quantize_prod_supported(const QuantArgs &q) {
  return q.t.mode == TQ_PROD && (q.t.bits == 1 || q.t.bits == 2) && q.d == kRD && q.t.m == kRM &&
         (q.dtype == TQ_BF16 || q.dtype == TQ_F16) &&
         static_cast<long long>(q.B) * q.Hkv * q.T < (1ll << 31);
}

cudaError_t launch_quantize_prod(const QuantArgs *k, const QuantArgs *v, int sms, cudaStream_t s) {
  ProdQuantArgs f{};
  const QuantArgs *in[2] = {k, v};
  const QuantArgs *first = k ? k : v;
  int nt = 0;
  for (int i = 0; i < 2; ++i) {
    if (!in[i]) continue;
    const QuantArgs &q = *in[i];
    ProdQuantTensor &t = f.t[nt];
    t.x = static_cast<const uint8_t *>(q.x);
    t.codes = q.t.codes;
    t.signs = q.t.signs;
    t.norm = q.t.norm;
    t.rnorm = q.t.rnorm;
    t.S = q.t.S;
    t.nvec = static_cast<unsigned>(static_cast<long long>(q.B) * q.Hkv * q.T);
    t.T = q.T;
    t.T_cap = q.T_cap;
    t.t_offset = q.t_offset;
    t.bt = q.pg.bt;
    t.pshift = q.pg.pshift;
    t.maxp = q.pg.maxp;
    t.Hkv = q.Hkv;
    t.wbits = q.t.wbits;
    t.c1 = q.t.wbits == 1 ? q.t.cb.c[1] : 0.f;
    f.groups[nt] = (t.nvec + 15) / 16;
    ++nt;
  }
  if (nt == 0) return cudaSuccess;
  f.ntensors = nt;
  f.sign_word = first->sign_words[0];
  const long long total = f.groups[0] + (nt > 1 ? f.groups[1] : 0);
  const long long blocks = std::min<long long>((total + kRWarps - 1) / kRWarps, 4ll * sms);
  const long long tiles = (f.t[0].nvec + kTcRows - 1) / kTcRows +
                         (nt > 1 ? (f.t[1].nvec + kTcRows - 1) / kTcRows : 0);
  if (tiles >= sms) { // bulk: tensor-core tiles of 128 vectors
    auto tkern = first->dtype == TQ_BF16 ? quantize_prod_tc_kernel<true> : quantize_prod_tc_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(tkern, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmem);
    if (e != cudaSuccess) return e;
    const long long grid = std::min<long long>(tiles, 3ll * sms);
    return launch_pdl(tkern, dim3(static_cast<unsigned>(grid)), dim3(kTcRows), kTcSmem, s, f);
  }
  auto kern = first->dtype == TQ_BF16 ? quantize_prod_kernel<true> : quantize_prod_kernel<false>;
  return launch_pdl(kern, dim3(static_cast<unsigned>(blocks)), dim3(kRWarps * 32), 0, s, f);
}

} // namespace tq
