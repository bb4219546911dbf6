// Prefill (chunked) attention over the compressed cache on the fifth-generation tensor cores:
// head_dim 128, TurboQuant_mse keys of 3 or 4 bits and values of 2, 3 or 4 bits.
//
// "Where This Fits in the Inference Stack", Decode Throughput vs. Time to First Token: at long
// contexts the attention of prefill reads the cache too; TensorRT-LLM section: chunked
// attention is one of the kernels that needs the in-register dequantisation. A chunk of Lq
// queries at positions t0 .. t0 + Lq - 1 (their own keys and values already in the cache)
// attends causally: query i sees cache positions 0 .. t0 + i.
//
// With many queries per KV head the dequantisation of a key or value tile is shared by all of
// them, so the tiles are dequantised once into shared-memory operands and the contractions are
// ordinary tcgen05 MMAs with wide N:
//   S_type = Q_type . K^T (kind::i8, M = 128 query rows, N = 64 tokens, K = 256): the key
//     operand holds the 16-bit fixed-point centroids as {hi, hi, lo, lo} bytes per coordinate
//     pair and the three query operands the 24-bit fixed-point query parts, exactly the score
//     arithmetic of the decode kernels (c.q = 2^24 S_0 + 2^16 S_1 + 2^8 S_2 up to c_lo q_lo);
//   O += P' . V (kind::f16, M = 128, N = 128 coordinates, K = 64 tokens): P' = p ||v|| in fp16
//     written by the softmax threads into shared memory (the A operand, K-major), V the fp16
//     centroids in shared memory (MN-major: each token's coordinates contiguous).
// A CTA takes 128 query rows (128 / G positions x G query heads) of one (batch, KV head):
//   softmax warps (4): thread = query row = TMEM lane; it prepares its queries (rotation,
//     fixed point), and per KV tile reads its row's scores, keeps the row's running maximum and
//     sum (no cross-thread reduction), rescales its output row in TMEM when the maximum moves,
//     and at the end applies the inverse rotation to its row;
//   producer warps (4): dequantise each 64-token tile of codes into the two operands (two
//     buffers each), with the tile's key and value norms, loading the next tile's codes while
//     expanding the current one;
//   MMA warp (1 thread): S MMAs of tile j, then P.V of tile j - 1, with tcgen05.commit
//     signalling completion.
// Every buffer is released by its last reader: a score stage and the tile's norms by the
// softmax warps once read (so the score MMAs of tile j + 2 overlap the softmax of tile j + 1),
// the key operand with them, the value operand and P' by the completion of P.V. TMEM: two
// score stages of 3 x 64 int32 columns, refilled with the read-back constant by the softmax
// threads, and the 128 fp32 output columns. Every mbarrier wait is bounded.
#include "decode_mse_common.cuh"
#include "tc_ops.cuh"

#include <cuda_fp8.h>

#include <algorithm>

namespace tq {
namespace {
using namespace mma_ops;
using namespace mse;

constexpr int kRows = 128;                   // query rows per CTA (TMEM lanes)
constexpr int kKT = 64;                      // KV tokens per tile
constexpr int kSWp = 8, kPWp = 4;            // softmax warps (two per row: half a tile each), producer warps
constexpr int kWarpMMAp = kSWp + kPWp;       // the MMA warp
constexpr int kThreadsP = (kSWp + kPWp + 1) * 32;
constexpr long long kWaitCyclesP = 1ll << 31; // about a second
// TMEM columns. Int8 scores: two score stages of three int32 columns per token, then the 128
// fp32 output columns (512 in all). E2M1 keys (F4): one fp32 score column per token leaves
// room for the MMAs' A operands: the four E4M3 query parts (32 columns each: 4 bytes of a row
// per column), two score stages, two P' buffers (fp16 pairs: 32 columns per 64 tokens), then
// the output columns.
template <bool F4>
struct PfTmem {
  static constexpr uint32_t Q = 0;                          // F4: query parts
  static constexpr uint32_t S0 = F4 ? 128 : 0;              // first score stage
  static constexpr uint32_t S = F4 ? kKT : 3 * kKT;         // one score stage
  static constexpr uint32_t P = S0 + 2 * S;                 // F4: P' buffers
  static constexpr uint32_t O = F4 ? P + 2 * (kKT / 2) : 2 * S; // first output column
  static constexpr uint32_t alloc = 512;
};
constexpr int kQParts4 = 4; // E4M3 parts of the query (F4): about 16 significant bits

__device__ unsigned g_prefill_fault;

struct PrefillArgs {
  const uint8_t *kc, *vc;
  const uint16_t *kn, *vn;
  const void *q; // [B][Lq][Hq][128] of q_dtype
  int q_dtype;
  float *out;    // [B][Lq][Hq][128] float32
  float scale;
  uint64_t seed;
  int Hq, Hkv, G, Lq, t0, T_cap;
  int P;      // query positions per CTA (128 / G)
  int blocks; // CTAs per (batch, KV head)
  float kcent[16];
  float kcsc;
  float vcent[16];
  float kstretch; // F4: the E2M1 grid's stretch (levels = kstretch * E2M1 values)
};

template <int KB, int VB, bool F4>
struct PfLayout {
  // query operands, K-major: 3 x [128 rows][256 bytes] int8, or (F4) 4 x [128 rows][128] E4M3
  static constexpr int kQBytes = F4 ? kQParts4 * kRows * 128 : 3 * kRows * 256;
  // key operand stages, K-major: [64 tokens][256 bytes] int8, or (F4) [64 tokens][8 groups of
  // 16 E2M1 codes: 8 bytes of packed codes + 8 bytes of padding]
  static constexpr int kKStage = F4 ? kKT * 128 : kKT * 256;
  static constexpr int oQ = 0;
  static constexpr int oK = oQ + kQBytes;
  static constexpr int oV = oK + 2 * kKStage;            // 2 x [128 coords][64 tokens] fp16, MN-major
  static constexpr int oP = oV + 2 * kKT * 256;          // 2 x [128 rows][64 tokens] fp16 P', K-major
  static constexpr int oKN = oP + 2 * kRows * kKT * 2;   // 2 x 64 key norms (float)
  static constexpr int oVN = oKN + 2 * kKT * 4;          // 2 x 64 value norms (float)
  static constexpr int oKT = oVN + 2 * kKT * 4;          // key entries {hi, hi, lo, lo} per code pair
  static constexpr int kKRows = F4 ? 0 : KB == 4 ? 256 : 64;
  static constexpr int oVT = oKT + kKRows * 4;           // value table
  static constexpr int kVRows = VB == 2 ? 256 : 1 << (2 * VB);
  static constexpr int kVEntry = VB == 2 ? 8 : 4;        // 2-bit: 4 fp16 per code byte; else fp16x2 per pair
  static constexpr int oQP = oVT + kVRows * kVEntry;     // per softmax warp: one prepared query
  static constexpr int oInv = oQP + kSWp * static_cast<int>(sizeof(QPrep));
  static constexpr int oXch = oInv + kRows * 4;          // [2 tile parities][2 halves][128 rows] float
  static constexpr int oBar = (oXch + 4 * kRows * 4 + 7) & ~7;
  // K_full[2] V_full[2] V_free[2] S_full[2] S_free[2] P_full[2] PV_done Q_ready fin
  static constexpr int nBar = 15;
  static constexpr int oMisc = oBar + nBar * 8;
  static constexpr int kSmem = oMisc + 16 + 1024;        // + alignment of the base
};

__device__ __forceinline__ bool pf_try(uint32_t mbar, uint32_t parity) {
  uint32_t done;
  asm volatile("{\n\t.reg .pred P;\n\tmbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2, %3;\n\t"
               "selp.u32 %0, 1, 0, P;\n\t}\n"
               : "=r"(done)
               : "r"(mbar), "r"(parity), "r"(500000u)
               : "memory");
  return done != 0;
}

__device__ __noinline__ void pf_wait_slow(uint32_t mbar, uint32_t parity, volatile int *dead) {
  const long long t0 = clock64();
  while (!pf_try(mbar, parity)) {
    if (*dead) return;
    if (clock64() - t0 > kWaitCyclesP) {
      *dead = 1;
      atomicOr(&g_prefill_fault, 1u);
      return;
    }
  }
}

// Bounded wait on an mbarrier phase (about a second; after a timeout, or once another warp of
// the CTA timed out, it returns without waiting and the CTA runs to its end).
__device__ __forceinline__ void pf_wait(uint32_t mbar, uint32_t parity, volatile int *dead) {
  if (!pf_try(mbar, parity)) pf_wait_slow(mbar, parity, dead);
}

// The MMA thread's last wait: for the completion of every MMA it issued (which depends on no
// other warp), whether or not the CTA has given up, so that TMEM is never released under a
// running MMA; bounded all the same.
__device__ __noinline__ void pf_wait_own_mmas(uint32_t mbar) {
  const long long t0 = clock64();
  while (!pf_try(mbar, 0)) {
    if (clock64() - t0 > kWaitCyclesP) {
      atomicOr(&g_prefill_fault, 1u);
      return;
    }
  }
}

template <int KB, int VB, bool F4>
__global__ void __launch_bounds__(kThreadsP, 1) prefill_kernel(const PrefillArgs a) {
  using L = PfLayout<KB, VB, F4>;
  constexpr uint32_t kSCols = PfTmem<F4>::S, kOCol = PfTmem<F4>::O, kTmemColsP = PfTmem<F4>::alloc;
  constexpr uint32_t kS0 = PfTmem<F4>::S0, kPCol = PfTmem<F4>::P, kQCol = PfTmem<F4>::Q;
  constexpr int KR = KB * 16, VR = VB * 16; // record bytes
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint32_t raw = static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw));
  const uint32_t sb = (raw + 1023) & ~1023u;
  uint8_t *const sm = smem_raw + (sb - raw);
  const uint32_t bar0 = sb + L::oBar;
  auto K_full = [&](int x) { return bar0 + 8u * x; };
  auto V_full = [&](int x) { return bar0 + 8u * (2 + x); };
  auto V_free = [&](int x) { return bar0 + 8u * (4 + x); };
  auto S_full = [&](int x) { return bar0 + 8u * (6 + x); };
  auto S_free = [&](int x) { return bar0 + 8u * (8 + x); };
  auto P_full = [&](int x) { return bar0 + 8u * (10 + x); };
  const uint32_t PV_done = bar0 + 8u * 12, Q_ready = bar0 + 8u * 13, fin_bar = bar0 + 8u * 14;
  uint32_t *const misc = reinterpret_cast<uint32_t *>(sm + L::oMisc);
  volatile int *const dead = reinterpret_cast<volatile int *>(misc + 1);
  float *const knb = reinterpret_cast<float *>(sm + L::oKN);
  float *const vnb = reinterpret_cast<float *>(sm + L::oVN);
  float *const rinv = reinterpret_cast<float *>(sm + L::oInv);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int blk = blockIdx.x % a.blocks;
  const long long bh = blockIdx.x / a.blocks;
  const int b = static_cast<int>(bh / a.Hkv), h = static_cast<int>(bh % a.Hkv);
  const int i0 = blk * a.P;
  const int i_last = min(a.Lq, i0 + a.P) - 1;
  const int pos_last = a.t0 + i_last;
  const int ntiles = pos_last / kKT + 1;

  // ---- tables: key entries {hi(c0), hi(c1), lo(c0), lo(c1)} of a code pair (the decode
  //      kernels' 16-bit fixed point); values as fp16 centroids
  {
    uint32_t *kt = reinterpret_cast<uint32_t *>(sm + L::oKT);
    for (int e = tid; e < L::kKRows; e += kThreadsP) { // none for E2M1 keys
      const float c0 = a.kcent[e & (KB == 4 ? 15 : 7)], c1 = a.kcent[KB == 4 ? e >> 4 : e >> 3];
      const int x0 = __float2int_rn(c0 * a.kcsc), x1 = __float2int_rn(c1 * a.kcsc);
      const int l0 = ((x0 + 128) & 255) - 128, l1 = ((x1 + 128) & 255) - 128;
      const int h0 = (x0 - l0) >> 8, h1 = (x1 - l1) >> 8;
      kt[e] = static_cast<uint32_t>(h0 & 255) | (static_cast<uint32_t>(h1 & 255) << 8) |
              (static_cast<uint32_t>(l0 & 255) << 16) | (static_cast<uint32_t>(l1 & 255) << 24);
    }
    uint32_t *vt = reinterpret_cast<uint32_t *>(sm + L::oVT);
    for (int e = tid; e < L::kVRows; e += kThreadsP) {
      if constexpr (VB == 2) {
        vt[2 * e] = pack_h2(a.vcent[e & 3], a.vcent[(e >> 2) & 3]);
        vt[2 * e + 1] = pack_h2(a.vcent[(e >> 4) & 3], a.vcent[(e >> 6) & 3]);
      } else {
        vt[e] = pack_h2(a.vcent[e & ((1 << VB) - 1)], a.vcent[e >> VB]);
      }
    }
  }
  if (tid == 0) {
    for (int x = 0; x < 2; ++x) {
      tc::mbar_init(K_full(x), 32 * kPWp);
      tc::mbar_init(V_full(x), 32 * kPWp);
      tc::mbar_init(V_free(x), 1);
      tc::mbar_init(S_full(x), 1);
      tc::mbar_init(S_free(x), kSWp);
      tc::mbar_init(P_full(x), 32 * kSWp);
    }
    tc::mbar_init(PV_done, 1);
    tc::mbar_init(Q_ready, 32 * kSWp);
    tc::mbar_init(fin_bar, 1);
    *dead = 0;
    tc::mbar_init_fence();
  }
  if (warp == kWarpMMAp) tc::tmem_alloc(sb + L::oMisc, kTmemColsP);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = misc[0];
  pdl_wait(); // the queries and the cache are written by earlier kernels
  pdl_trigger();

  if (warp < kSWp) {
    // =============================== softmax warps: two per query row (= TMEM lane), warp
    //      quarter qw holds lanes 32 qw .. 32 qw + 31 and half hf the tokens 32 hf .. 32 hf + 31
    //      of every tile and output coordinates 64 hf .. 64 hf + 63 at the end
    const int qw = warp & 3, hf = warp >> 2;
    const int row = 32 * qw + lane;
    const int ri = row / a.G, rg = row - ri * a.G; // query position within the block, head
    const bool row_ok = ri < a.P && i0 + ri < a.Lq;
    const int my_pos = a.t0 + i0 + ri;
    const int pos_lo = a.t0 + i0 + (32 * qw) / a.G; // the smallest position among the warp's rows
    const uint32_t lrow = static_cast<uint32_t>(32 * qw) << 16;
    float *const xch = reinterpret_cast<float *>(sm + L::oXch);
    // the two warps of a lane quarter meet at named barrier 1 + qw
    auto pair_sync = [&]() {
      __syncwarp();
      asm volatile("bar.sync %0, 64;" ::"r"(1 + qw) : "memory");
    };
    // ---- queries of the warp's 16 rows: rotation and 24-bit fixed point (one warp per query),
    //      written as the three int8 operands {q_hi, q_hi, 0, 0}, {q_mid, q_mid, q_hi, q_hi},
    //      {q_lo, q_lo, q_mid, q_mid} at the {hi, hi, lo, lo} slots of each coordinate pair
    QPrep *qs = reinterpret_cast<QPrep *>(sm + L::oQP) + warp;
#pragma unroll 1
    for (int k = 0; k < 16; ++k) {
      const int rr = 32 * qw + 16 * hf + k;
      const int qi = rr / a.G, qg = rr - qi * a.G;
      const bool ok = qi < a.P && i0 + qi < a.Lq;
      if constexpr (F4) {
        // E2M1 keys: the query as the sum of four E4M3 parts (each the rounding of what the
        // earlier ones left), scaled so that its largest coordinate is 224; the score MMAs
        // accumulate all four in fp32. Part p of row rr, coordinate i: byte (rr & 7) * 16 +
        // (rr >> 3) * 1024 + (i >> 4) * 128 + (i & 15) of part p's operand.
        float x[4] = {0.f, 0.f, 0.f, 0.f};
        if (ok) {
          const size_t bq = (static_cast<size_t>(b) * a.Lq + i0 + qi) * a.Hq + h * a.G + qg;
          rotate_query(a.q, a.q_dtype, bq, a.scale, a.seed, lane, x);
        }
        float mx = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
        mx = warp_max(mx);
        const bool has_nan = __any_sync(0xffffffffu, isnan(x[0]) || isnan(x[1]) || isnan(x[2]) || isnan(x[3]));
        const bool good = !has_nan && mx > 1e-30f && isfinite(mx);
        const float qsc = good ? 224.0f / mx : 0.f;
        float r[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) r[e] = x[e] * qsc;
        const uint32_t off = (rr & 7) * 16 + (rr >> 3) * 1024 + (lane >> 2) * 128 + 4 * (lane & 3);
#pragma unroll
        for (int part = 0; part < kQParts4; ++part) {
          uint32_t w = 0;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_fp8_storage_t f = __nv_cvt_float_to_fp8(r[e], __NV_SATFINITE, __NV_E4M3);
            w |= static_cast<uint32_t>(f) << (8 * e);
            r[e] -= __half2float(__half(__nv_cvt_fp8_to_halfraw(f, __NV_E4M3)));
          }
          *reinterpret_cast<uint32_t *>(sm + L::oQ + part * (kRows * 128) + off) = w;
        }
        // score = ||k|| * (c . q~) = ||k|| * S * kstretch / qsc, S the MMAs' sum over E2M1
        // values; a query with a NaN or an infinity gets NaN, a (near) zero one zero scores
        if (lane == 0)
          rinv[rr] = (good ? a.kstretch / qsc : (!has_nan && isfinite(mx) ? 0.f : __int_as_float(0x7fc00000))) * kLog2e;
        __syncwarp();
        continue;
      }
      if (ok) {
        const size_t bq = (static_cast<size_t>(b) * a.Lq + i0 + qi) * a.Hq + h * a.G + qg;
        prep_query(a.q, a.q_dtype, bq, a.scale, a.seed, a.kcsc, qs, lane);
      } else {
        reinterpret_cast<uint32_t *>(qs->hi)[lane] = 0u;
        reinterpret_cast<uint32_t *>(qs->mid)[lane] = 0u;
        reinterpret_cast<uint32_t *>(qs->lo)[lane] = 0u;
        if (lane == 0) qs->inv = 0.f;
      }
      __syncwarp();
      // lane l: k bytes 8 l .. 8 l + 7 = code pairs 2 l, 2 l + 1 (coordinates 4 l .. 4 l + 3)
      const uint32_t hi = reinterpret_cast<const uint32_t *>(qs->hi)[lane];
      const uint32_t mid = reinterpret_cast<const uint32_t *>(qs->mid)[lane];
      const uint32_t lo = reinterpret_cast<const uint32_t *>(qs->lo)[lane];
      const uint32_t off = (rr & 7) * 16 + (rr >> 3) * 2048 + (lane >> 1) * 128 + 8 * (lane & 1);
      *reinterpret_cast<uint2 *>(sm + L::oQ + off) = make_uint2(hi & 0xFFFFu, hi >> 16);
      *reinterpret_cast<uint2 *>(sm + L::oQ + kRows * 256 + off) =
          make_uint2((mid & 0xFFFFu) | (hi << 16), (mid >> 16) | (hi & 0xFFFF0000u));
      *reinterpret_cast<uint2 *>(sm + L::oQ + 2 * kRows * 256 + off) =
          make_uint2((lo & 0xFFFFu) | (mid << 16), (lo >> 16) | (mid & 0xFFFF0000u));
      if (lane == 0) rinv[rr] = qs->inv * kLog2e;
      __syncwarp();
    }
    // both score stages start at the magic constant: every score MMA accumulates onto it, so
    // an int32 sum s reads back as the float 1.5 * 2^23 + s (each warp its own tokens' columns)
    if constexpr (!F4) {
#pragma unroll
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int t = 0; t < 3; ++t)
          tc::tmem_fill32x32_x32(tbase + lrow + (kS0 + x * kSCols) + kKT * t + 32 * hf, static_cast<uint32_t>(kMagic));
      tc::tmem_wait_st();
    } else {
      // the query parts move from their shared-memory staging (written above by the warp pair,
      // one warp per row) into tensor memory, each thread its own row: parts 2 hf, 2 hf + 1
      pair_sync();
#pragma unroll
      for (int pp = 0; pp < 2; ++pp) {
        const int part = 2 * hf + pp;
        const uint8_t *src = sm + L::oQ + part * (kRows * 128) + (row & 7) * 16 + (row >> 3) * 1024;
        uint32_t qw32[32];
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const uint4 v = *reinterpret_cast<const uint4 *>(src + g * 128);
          qw32[4 * g] = v.x;
          qw32[4 * g + 1] = v.y;
          qw32[4 * g + 2] = v.z;
          qw32[4 * g + 3] = v.w;
        }
        tc::tmem_st32x32_x32(tbase + lrow + kQCol + 32 * part, qw32);
      }
      tc::tmem_wait_st();
    }
    tc::fence_before_sync();
    tc::fence_async_smem();
    tc::mbar_arrive(Q_ready);
    pair_sync(); // the row's scale factor is written by the other warp of the pair for half its rows
    const float qsc = rinv[row];

    // running maximum in units of ||k|| * (c . q~) (the exponent is qsc times it), shared by the
    // pair; running sums per half
    constexpr int kH = kKT / 2; // tokens per warp and tile
    float m_run = -INFINITY, l_run = 0.f;
#pragma unroll 1
    for (int j = 0; j < ntiles; ++j) {
      const int x = j & 1;
      const int tb = kKT * j + kH * hf; // first token of this warp's half tile
      pf_wait(S_full(x), (j >> 1) & 1, dead);
      tc::fence_after_sync();
      // warp-uniform: some row of the warp sees only part of its half tile (the causal diagonal)
      const bool edge = tb + kH - 1 > pos_lo;
      const uint32_t st = tbase + lrow + (kS0 + x * kSCols) + kH * hf;
      const float4 *kn4 = reinterpret_cast<const float4 *>(knb + x * kKT + kH * hf);
      float s[kH];
      if constexpr (F4) {
        // one fp32 column per token
#pragma unroll
        for (int cch = 0; cch < kH / 16; ++cch) {
          uint32_t r0[16];
          tc::tmem_ld32x32_x16(st + 16 * cch, r0);
          tc::tmem_wait_ld();
#pragma unroll
          for (int t4 = 0; t4 < 4; ++t4) {
            const float4 k4 = kn4[4 * cch + t4];
            s[16 * cch + 4 * t4] = k4.x * __uint_as_float(r0[4 * t4]);
            s[16 * cch + 4 * t4 + 1] = k4.y * __uint_as_float(r0[4 * t4 + 1]);
            s[16 * cch + 4 * t4 + 2] = k4.z * __uint_as_float(r0[4 * t4 + 2]);
            s[16 * cch + 4 * t4 + 3] = k4.w * __uint_as_float(r0[4 * t4 + 3]);
          }
        }
      } else {
#pragma unroll
        for (int cch = 0; cch < kH / 16; ++cch) {
          uint32_t r0[16], r1[16], r2[16];
          tc::tmem_ld32x32_x16(st + 16 * cch, r0);
          tc::tmem_ld32x32_x16(st + kKT + 16 * cch, r1);
          tc::tmem_ld32x32_x16(st + 2 * kKT + 16 * cch, r2);
          tc::tmem_wait_ld();
#pragma unroll
          for (int t4 = 0; t4 < 4; ++t4) {
            const float4 k4 = kn4[4 * cch + t4];
            const float kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int t = 4 * t4 + e;
              const float d = fmaf(__uint_as_float(r2[t]), 1.0f / 65536.0f,
                                   fmaf(__uint_as_float(r1[t]), 1.0f / 256.0f, __uint_as_float(r0[t]) - kMagicAdj));
              s[16 * cch + t] = kk[e] * d;
            }
          }
      }
        // the columns back to the magic constant for tile j + 2 (waited for before release)
#pragma unroll
        for (int t = 0; t < 3; ++t) tc::tmem_fill32x32_x32(st + kKT * t, static_cast<uint32_t>(kMagic));
      }
      if (edge) {
#pragma unroll
        for (int t = 0; t < kH; ++t)
          if (tb + t > my_pos) s[t] = -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int t = 1; t < kH; ++t) mx = fmaxf(mx, s[t]);
      // the row's maximum over the whole tile: the halves' maxima meet in shared memory (one
      // slot per tile parity, so that the next tile's write cannot meet this tile's read)
      float *const xs = xch + (j & 1) * 2 * kRows;
      xs[hf * kRows + row] = mx;
      pair_sync();
      mx = fmaxf(mx, xs[(1 - hf) * kRows + row]);
      const float mn = fmaxf(m_run, mx);
      // a row whose maximum moved scales its sum and its half of the output row accumulated so
      // far (once the previous tile's P.V has landed; before the first P.V the output is
      // undefined and is overwritten)
      const bool moved = mn != m_run;
      const float alpha = (moved && j > 0) ? softmax_exp2(qsc * (m_run - mn)) : 1.f;
      l_run *= alpha;
      m_run = mn;
      const float mq = qsc * mn;
      // weights p ||v|| as fp16 (P', the A operand of P.V)
      const float4 *vn4 = reinterpret_cast<const float4 *>(vnb + x * kKT + kH * hf);
      uint32_t pw[kH / 2];
#pragma unroll
      for (int t4 = 0; t4 < kH / 4; ++t4) {
        const float4 v4 = vn4[t4];
        float p[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) p[e] = softmax_exp2(fmaf(s[4 * t4 + e], qsc, -mq));
        if (edge) {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (tb + 4 * t4 + e > my_pos) p[e] = 0.f;
        }
        l_run += (p[0] + p[1]) + (p[2] + p[3]);
        pw[2 * t4] = pack_h2(p[0] * v4.x, p[1] * v4.y);
        pw[2 * t4 + 1] = pack_h2(p[2] * v4.z, p[3] * v4.w);
      }
      // the score columns and the tile's norms are no longer needed: release them to the next
      // score MMAs and the producers
      tc::tmem_wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(S_free(x));
      // P' buffer x was last read by P.V of tile j - 2, complete once S_full(j) arrived (the MMA
      // thread commits S_full(j) after issuing it); this warp's tokens are k chunks 4 hf .. 4 hf + 3
      if constexpr (F4) {
        // P' into its TMEM buffer (the A operand of P.V): 16 columns of fp16 pairs per half tile
        tc::tmem_st32x32_x16(tbase + lrow + kPCol + x * (kKT / 2) + (kH / 2) * hf, pw);
      } else {
        uint8_t *pdst = sm + L::oP + x * (kRows * kKT * 2) + (row & 7) * 16 + (row >> 3) * 1024 + hf * 512;
#pragma unroll
        for (int c = 0; c < kH / 8; ++c)
          *reinterpret_cast<uint4 *>(pdst + c * 128) = make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
        tc::fence_async_smem();
      }
      // the TMEM loads and stores are warp-collective (.sync.aligned), so the whole warp takes
      // this path when any of its rows needs it, the others with factor 1
      if (j > 0 && __any_sync(0xffffffffu, moved)) {
        // completion j - 1 of PV_done: S_full(j) implies P.V of tile j - 2 had completed, and
        // P.V of tile j waits for this tile's P', so the parity identifies it
        pf_wait(PV_done, (j - 1) & 1, dead);
        tc::fence_after_sync();
#pragma unroll 1
        for (int cch = 0; cch < 2; ++cch) {
          uint32_t ov[32];
          const uint32_t oc = tbase + lrow + kOCol + 64 * hf + 32 * cch;
          tc::tmem_ld32x32_x32u(oc, ov);
          tc::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
          tc::tmem_st32x32_x32(oc, ov);
        }
        tc::tmem_wait_st();
      }
      if constexpr (F4) tc::tmem_wait_st(); // P' has landed in tensor memory
      tc::fence_before_sync();
      tc::mbar_arrive(P_full(x));
    }
    // ---- output row: O / l in the rotated domain, then the inverse rotation D H / d (after the
    //      last P.V: the MMA thread commits every MMA of the CTA to fin_bar). Each warp of the
    //      pair transforms its 64 coordinates over the butterfly spans 1 .. 32, the span-64 stage
    //      pairs coordinate i of one half with i of the other through TMEM.
    // the half's sum goes to the slot of parity ntiles (its last reads, at tile ntiles - 2, were
    // done before the partner passed the last tile's pair_sync)
    xch[(ntiles & 1) * 2 * kRows + hf * kRows + row] = l_run;
    pf_wait(fin_bar, 0, dead);
    tc::fence_after_sync();
    float o[64];
#pragma unroll
    for (int cch = 0; cch < 2; ++cch) {
      uint32_t ov[32];
      tc::tmem_ld32x32_x32u(tbase + lrow + kOCol + 64 * hf + 32 * cch, ov);
      tc::tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) o[32 * cch + e] = __uint_as_float(ov[e]);
    }
#pragma unroll
    for (int span = 1; span < 64; span <<= 1) {
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        if ((i & span) == 0) {
          const float u = o[i], v = o[i + span];
          o[i] = u + v;
          o[i + span] = u - v;
        }
      }
    }
    {
      uint32_t ov[32];
#pragma unroll
      for (int cch = 0; cch < 2; ++cch) {
#pragma unroll
        for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(o[32 * cch + e]);
        tc::tmem_st32x32_x32(tbase + lrow + kOCol + 64 * hf + 32 * cch, ov);
      }
      tc::tmem_wait_st();
    }
    tc::fence_before_sync();
    pair_sync();
    tc::fence_after_sync();
    const float l_tot = l_run + xch[(ntiles & 1) * 2 * kRows + (1 - hf) * kRows + row];
#pragma unroll
    for (int cch = 0; cch < 2; ++cch) {
      uint32_t ov[32];
      tc::tmem_ld32x32_x32u(tbase + lrow + kOCol + 64 * (1 - hf) + 32 * cch, ov);
      tc::tmem_wait_ld();
      // half 0 keeps u + v (coordinates 0 .. 63), half 1 u - v (64 .. 127), u being half 0's value
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float other = __uint_as_float(ov[e]);
        o[32 * cch + e] = hf == 0 ? o[32 * cch + e] + other : other - o[32 * cch + e];
      }
    }
    if (row_ok) {
      const float sc = 1.0f / (128.0f * l_tot);
      const uint64_t w = dev_splitmix64(a.seed, hf); // sign bits of coordinates 64 hf .. 64 hf + 63
      float *dst = a.out + ((static_cast<size_t>(b) * a.Lq + i0 + ri) * a.Hq + h * a.G + rg) * 128 + 64 * hf;
#pragma unroll
      for (int i = 0; i < 64; i += 4) {
        float4 v4;
        float *vp = &v4.x;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int ii = i + e;
          const bool neg = ((w >> ii) & 1ull) != 0;
          vp[e] = neg ? -o[ii] * sc : o[ii] * sc;
        }
        *reinterpret_cast<float4 *>(dst + i) = v4;
      }
    }
  } else if (warp < kWarpMMAp) {
    // =============================== producer warps: 64-token tiles of K and V operands; the
    //      codes of the next tile are loaded while the current one is expanded
    const int pt = tid - 32 * kSWp; // 0..127
    const int n = pt >> 1, half = pt & 1;
    const uint32_t *kt = reinterpret_cast<const uint32_t *>(sm + L::oKT);
    const uint8_t *vt = sm + L::oVT;
    struct Codes {
      uint32_t k[KB * 2], v[VB * 2];
      uint16_t nrm; // key norm (half 0) or value norm (half 1) of token n
    };
    auto load = [&](int j, Codes &c) {
      const int tok = min(kKT * j + n, pos_last);
      const size_t rec = static_cast<size_t>(bh) * a.T_cap + tok;
      const uint32_t *kp = reinterpret_cast<const uint32_t *>(a.kc + rec * KR + KB * 8 * half);
#pragma unroll
      for (int k = 0; k < KB * 2; ++k) c.k[k] = __ldg(kp + k);
      const uint32_t *vp = reinterpret_cast<const uint32_t *>(a.vc + rec * VR + VB * 8 * half);
#pragma unroll
      for (int k = 0; k < VB * 2; ++k) c.v[k] = __ldg(vp + k);
      c.nrm = __ldg((half == 0 ? a.kn : a.vn) + rec);
    };
    auto produce = [&](int j, const Codes &c) {
      const int x = j & 1;
      // keys: code pairs 32 half .. 32 half + 31 -> k bytes 128 half .. 128 half + 127 of row n.
      // Buffer x and the norms of tile j - 2 are free once its softmax released the stage.
      if (j >= 2) pf_wait(S_free(x), ((j >> 1) - 1) & 1, dead);
      if constexpr (F4) {
        // E2M1 keys: the stored codes are indices of the ascending E2M1 levels; index i has
        // the bit pattern i ^ 8 (i >= 8) or i ^ 15 (i < 8): per nibble, XOR with 15 - 7 t, t its
        // top bit. Group g of 16 coordinates: 8 bytes of patterns, then 8 bytes of padding.
        uint8_t *kdst = sm + L::oK + x * L::kKStage + (n & 7) * 16 + (n >> 3) * 1024 + half * 4 * 128;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const uint32_t w0 = c.k[2 * g], w1 = c.k[2 * g + 1];
          const uint32_t e0 = w0 ^ (0xFFFFFFFFu - 7u * ((w0 >> 3) & 0x11111111u));
          const uint32_t e1 = w1 ^ (0xFFFFFFFFu - 7u * ((w1 >> 3) & 0x11111111u));
          *reinterpret_cast<uint4 *>(kdst + g * 128) = make_uint4(e0, e1, 0u, 0u);
        }
      } else {
        uint8_t *kdst = sm + L::oK + x * (kKT * 256) + (n & 7) * 16 + (n >> 3) * 2048 + half * 8 * 128;
#pragma unroll
        for (int c16 = 0; c16 < 8; ++c16) { // 16 k bytes = 4 code pairs
          uint32_t e4[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int pp = 4 * c16 + u; // pair within this half
            uint32_t idx;
            if constexpr (KB == 4) {
              idx = (c.k[pp >> 2] >> (8 * (pp & 3))) & 0xFFu;
            } else {
              idx = bits_at(c.k, 6 * pp, 0) & 0x3Fu;
            }
            e4[u] = kt[idx];
          }
          *reinterpret_cast<uint4 *>(kdst + c16 * 128) = make_uint4(e4[0], e4[1], e4[2], e4[3]);
        }
      }
      if (half == 0) knb[x * kKT + n] = f16_bits_to_f32(c.nrm);
      else vnb[x * kKT + n] = f16_bits_to_f32(c.nrm);
      tc::fence_async_smem();
      tc::mbar_arrive(K_full(x));
      // values: coordinates 64 half .. 64 half + 63 of token n as fp16, MN-major; buffer x is
      // free once P.V of tile j - 2 completed
      if (j >= 2) pf_wait(V_free(x), ((j >> 1) - 1) & 1, dead);
      {
        uint8_t *vdst = sm + L::oV + x * (kKT * 256) + (n >> 3) * 128 + (n & 7) * 16 + half * 8 * 1024;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) { // 8 coordinates
          uint32_t e4[4];
          if constexpr (VB == 2) {
            const uint32_t byte0 = (c.v[c8 >> 1] >> (16 * (c8 & 1))) & 0xFFu;
            const uint32_t byte1 = (c.v[c8 >> 1] >> (16 * (c8 & 1) + 8)) & 0xFFu;
            const uint2 q0 = *reinterpret_cast<const uint2 *>(vt + 8 * byte0);
            const uint2 q1 = *reinterpret_cast<const uint2 *>(vt + 8 * byte1);
            e4[0] = q0.x;
            e4[1] = q0.y;
            e4[2] = q1.x;
            e4[3] = q1.y;
          } else {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int pp = 4 * c8 + u; // coordinate pair within this half
              const uint32_t idx = bits_at(c.v, 2 * VB * pp, 0) & ((1u << (2 * VB)) - 1u);
              e4[u] = reinterpret_cast<const uint32_t *>(vt)[idx];
            }
          }
          *reinterpret_cast<uint4 *>(vdst + c8 * 1024) = make_uint4(e4[0], e4[1], e4[2], e4[3]);
        }
      }
      tc::fence_async_smem();
      tc::mbar_arrive(V_full(x));
    };
    Codes c0, c1;
    load(0, c0);
#pragma unroll 1
    for (int j = 0; j < ntiles; j += 2) {
      if (j + 1 < ntiles) load(j + 1, c1);
      produce(j, c0);
      if (j + 1 >= ntiles) break;
      if (j + 2 < ntiles) load(j + 2, c0);
      produce(j + 1, c1);
    }
  } else {
    // =============================== MMA warp: one thread issues every MMA
    if (lane == 0) {
      const uint32_t id_s = F4 ? tc::idesc_e4m3_e2m1(kRows, kKT) : tc::idesc_i8(kRows, kKT);
      const uint32_t id_o = tc::idesc_f16_bmn(kRows, 128);
      pf_wait(Q_ready, 0, dead);
      // after a timeout (dead) no further MMA is issued
      auto pv = [&](int jj) {
        const int x = jj & 1;
        pf_wait(P_full(x), (jj >> 1) & 1, dead);
        pf_wait(V_full(x), (jj >> 1) & 1, dead);
        if (*dead) return;
        tc::fence_after_sync();
#pragma unroll
        for (int s = 0; s < kKT / 16; ++s) {
          if constexpr (F4)
            tc::mma_ts_f16(tbase + kOCol, tbase + kPCol + x * (kKT / 2) + 8 * s,
                           tc::desc_kmajor(sb + L::oV + x * (kKT * 256) + 256 * s, 128, 1024), id_o,
                           (jj > 0 || s > 0) ? 1u : 0u);
          else
            tc::mma_ss(tbase + kOCol, tc::desc_kmajor(sb + L::oP + x * (kRows * kKT * 2) + 256 * s, 128, 1024),
                       tc::desc_kmajor(sb + L::oV + x * (kKT * 256) + 256 * s, 128, 1024), id_o,
                       (jj > 0 || s > 0) ? 1u : 0u);
        }
        tc::commit(V_free(x));
        tc::commit(PV_done);
      };
#pragma unroll 1
      for (int j = 0; j < ntiles; ++j) {
        const int x = j & 1;
        pf_wait(K_full(x), (j >> 1) & 1, dead);
        if (j >= 2) pf_wait(S_free(x), ((j >> 1) - 1) & 1, dead);
        if (*dead) break;
        tc::fence_after_sync();
        if constexpr (F4) {
          // S = sum over the four E4M3 query parts and 4 k-steps of 32 coordinates: E4M3 x E2M1,
          // fp32 accumulation into one column per token
#pragma unroll
          for (int part = 0; part < kQParts4; ++part)
#pragma unroll
            for (int s = 0; s < 4; ++s)
              tc::mma_ts_f8f6f4(tbase + (kS0 + x * kSCols), tbase + kQCol + 32 * part + 8 * s,
                                tc::desc_kmajor(sb + L::oK + x * L::kKStage + 256 * s, 128, 1024), id_s,
                                (part > 0 || s > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int type = 0; type < 3; ++type)
#pragma unroll
            for (int s = 0; s < 8; ++s)
              tc::mma_ss_i8(tbase + (kS0 + x * kSCols) + kKT * type,
                            tc::desc_kmajor8(sb + L::oQ + type * (kRows * 256) + 256 * s, 128, 2048),
                            tc::desc_kmajor8(sb + L::oK + x * (kKT * 256) + 256 * s, 128, 2048), id_s, 1u);
        }
        tc::commit(S_full(x));
        if (j > 0) pv(j - 1);
      }
      pv(ntiles - 1);
      tc::commit(fin_bar);
      pf_wait_own_mmas(fin_bar);
    }
    __syncwarp();
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == kWarpMMAp) tc::tmem_dealloc(tbase, kTmemColsP);
}

template <int KB, int VB, bool F4 = false>
cudaError_t run_prefill(const PrefillArgs &p, int ctas, cudaStream_t s) {
  constexpr int smem = PfLayout<KB, VB, F4>::kSmem;
  auto kern = prefill_kernel<KB, VB, F4>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(ctas), dim3(kThreadsP), smem, s, p);
}

} // namespace

bool prefill_supported(int d, int k_mode, int k_wbits, int v_mode, int v_wbits, int G) {
  return d == 128 && k_mode == TQ_MSE && (k_wbits == 3 || k_wbits == 4) && v_mode == TQ_MSE && v_wbits >= 2 &&
         v_wbits <= 4 && G >= 1 && G <= kRows && kRows % G == 0;
}

cudaError_t launch_prefill(const PrefillLaunch &l, cudaStream_t s) {
  PrefillArgs p;
  p.kc = l.k.codes;
  p.vc = l.v.codes;
  p.kn = l.k.norm;
  p.vn = l.v.norm;
  p.q = l.q;
  p.q_dtype = l.q_dtype;
  p.out = l.out;
  p.scale = l.scale;
  p.seed = l.seed;
  p.Hq = l.Hq;
  p.Hkv = l.Hkv;
  p.G = l.Hq / l.Hkv;
  p.Lq = l.Lq;
  p.t0 = l.t0;
  p.T_cap = l.T_cap;
  p.P = kRows / p.G;
  p.blocks = (l.Lq + p.P - 1) / p.P;
  for (int j = 0; j < 16; ++j) p.kcent[j] = l.k.cb.c[j];
  p.kcsc = l.k.cb.fix_scale;
  for (int j = 0; j < 16; ++j) p.vcent[j] = l.v.cb.c[j];
  p.kstretch = l.k.cb.c[15] / 6.0f; // the largest E2M1 level is 6 x the stretch
  const int ctas = l.B * l.Hkv * p.blocks;
  const int kb = l.k.wbits, vb = l.v.wbits;
  if (l.k_e2m1)
    return vb == 2 ? run_prefill<4, 2, true>(p, ctas, s) : vb == 3 ? run_prefill<4, 3, true>(p, ctas, s)
                                                                  : run_prefill<4, 4, true>(p, ctas, s);
  if (kb == 4) return vb == 2 ? run_prefill<4, 2>(p, ctas, s) : vb == 3 ? run_prefill<4, 3>(p, ctas, s)
                                                                      : run_prefill<4, 4>(p, ctas, s);
  return vb == 2 ? run_prefill<3, 2>(p, ctas, s) : vb == 3 ? run_prefill<3, 3>(p, ctas, s)
                                                           : run_prefill<3, 4>(p, ctas, s);
}

cudaError_t read_and_clear_prefill_faults(unsigned *flags) {
  unsigned v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_prefill_fault, sizeof v);
  if (e != cudaSuccess) return e;
  *flags = v;
  if (v) {
    const unsigned z = 0;
    e = cudaMemcpyToSymbol(g_prefill_fault, &z, sizeof z);
  }
  return e;
}

} // namespace tq
