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
  float c1; // the positive 1-bit centroid (wbits = 1)
};

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
__device__ __forceinline__ float widen(uint32_t w, int half) {
  if (BF16) return __uint_as_float(half ? (w & 0xFFFF0000u) : (w << 16));
  const __half2 h = *reinterpret_cast<const __half2 *>(&w);
  return half ? __high2float(h) : __low2float(h);
}

template <bool BF16>
__global__ void __launch_bounds__(kRWarps * 32) quantize_prod_kernel(const ProdQuantArgs a) {
  // B fragments of S^T per tensor: [tensor][n-tile 8][k-step 4][lane 32] {b0 hi, b1 hi, b0 lo,
  // b1 lo}; lane (r, c) of n-tile nt, k-step s holds S[8 nt + r][16 c + 4 s + 0..3].
  __shared__ uint4 sfrag[2][8][4][32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = lane >> 2, c = lane & 3;
  for (int idx = tid; idx < a.ntensors * 8 * 4 * 32; idx += kRWarps * 32) {
    const int ti = idx / 1024, rest = idx % 1024;
    const int nt = rest / 128, s = (rest / 32) % 4, l = rest % 32;
    const float *row = a.t[ti].S + static_cast<size_t>(8 * nt + (l >> 2)) * kRD + 16 * (l & 3) + 4 * s;
    uint4 f;
    split2(row[0], row[1], f.x, f.z);
    split2(row[2], row[3], f.y, f.w);
    sfrag[ti][nt][s][l] = f;
  }
  // sign masks of the lane's coordinates 16 c .. 16 c + 15 (bit 31 set where D flips it)
  uint32_t sgn[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) sgn[e] = ((a.sign_word >> (16 * c + e)) & 1ull) ? 0x80000000u : 0u;
  __syncthreads();
  pdl_wait(); // K/V may come from the kernel before; the cache may still be read by it
  pdl_trigger();

  const long long total = a.groups[0] + (a.ntensors > 1 ? a.groups[1] : 0);
  for (long long gi = static_cast<long long>(blockIdx.x) * kRWarps + warp; gi < total;
       gi += static_cast<long long>(gridDim.x) * kRWarps) {
    const int ti = gi < a.groups[0] ? 0 : 1;
    const ProdQuantTensor t = a.t[ti]; // one copy of the tensor's fields per group
    const unsigned v0 = static_cast<unsigned>((gi - (ti ? a.groups[0] : 0)) * 16);
    const unsigned va = v0 + r, vb = v0 + r + 8;
    const unsigned la = min(va, t.nvec - 1), lb = min(vb, t.nvec - 1);

    // ---- load (two 16-byte loads per vector), widen, apply the signs
    float x[2][16];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const uint4 *src = reinterpret_cast<const uint4 *>(t.x + (static_cast<size_t>(u ? lb : la) * kRD + 16 * c) * 2);
      const uint4 q0 = __ldcs(src), q1 = __ldcs(src + 1);
      const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
      for (int e = 0; e < 16; ++e)
        x[u][e] = __uint_as_float(__float_as_uint(widen<BF16>(w[e >> 1], e & 1)) ^ sgn[e]);
    }
    // ---- norms
    float ss[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < 16; ++e) acc = fmaf(x[u][e], x[u][e], acc);
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      ss[u] = acc;
    }
    // ---- Walsh-Hadamard: spans 1..8 in the lane, 16 and 32 across lanes c
#pragma unroll
    for (int u = 0; u < 2; ++u) {
#pragma unroll
      for (int h = 1; h < 16; h <<= 1)
#pragma unroll
        for (int e = 0; e < 16; ++e)
          if ((e & h) == 0) {
            const float p = x[u][e], q = x[u][e + h];
            x[u][e] = p + q;
            x[u][e + h] = p - q;
          }
#pragma unroll
      for (int m = 1; m < 4; m <<= 1) {
        const float sgnm = (c & m) ? -1.0f : 1.0f; // upper lane keeps partner - own
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float o = __shfl_xor_sync(0xffffffffu, x[u][e], m);
          x[u][e] = fmaf(x[u][e], sgnm, o);
        }
      }
    }
    const bool wb1 = t.wbits == 1;
    // ---- z, 1-bit codes, unit-domain residual r = (z - c[code]) / sqrt(d) and its norm
    uint32_t code_bits[2] = {0u, 0u}; // bit e: code of coordinate 16 c + e
    float nrm[2], gam[2];
    uint32_t ahi[2][8], alo[2][8]; // A operand pairs (coordinates 16 c + 2 p, + 1), p = 0..7
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      nrm[u] = sqrtf(ss[u]);
      const float inv = nrm[u] > 0.f ? 1.0f / nrm[u] : 0.0f;
      float rr = 0.f;
      float res[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float z = x[u][e] * inv;
        float chat = 0.f;
        if (wb1) {
          const bool up = z > 0.f;
          code_bits[u] |= (up ? 1u : 0u) << e;
          chat = up ? t.c1 : -t.c1;
        }
        res[e] = (z - chat) * 0.125f; // 1 / sqrt(64)
        rr = fmaf(res[e], res[e], rr);
      }
      rr += __shfl_xor_sync(0xffffffffu, rr, 1);
      rr += __shfl_xor_sync(0xffffffffu, rr, 2);
      gam[u] = sqrtf(rr);
#pragma unroll
      for (int p = 0; p < 8; ++p) split2(res[2 * p], res[2 * p + 1], ahi[u][p], alo[u][p]);
    }

    // ---- sketch S r on the tensor cores; bit j = 1 iff (S r)_j < 0
    uint32_t sg[2][2] = {{0u, 0u}, {0u, 0u}}; // [vector][word]
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      float m0[4] = {0.f, 0.f, 0.f, 0.f}, m1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const uint4 f = sfrag[ti][nt][s][lane];
        mma16816(m0, ahi[0][2 * s], ahi[1][2 * s], ahi[0][2 * s + 1], ahi[1][2 * s + 1], f.x, f.y);
        mma16816(m1, alo[0][2 * s], alo[1][2 * s], alo[0][2 * s + 1], alo[1][2 * s + 1], f.x, f.y);
        mma16816(m1, ahi[0][2 * s], ahi[1][2 * s], ahi[0][2 * s + 1], ahi[1][2 * s + 1], f.z, f.w);
      }
      const int j = 8 * nt + 2 * c, wi = j >> 5, sh = j & 31;
      const float p00 = fmaf(m1[0], kRLoInv, m0[0]), p01 = fmaf(m1[1], kRLoInv, m0[1]);
      const float p10 = fmaf(m1[2], kRLoInv, m0[2]), p11 = fmaf(m1[3], kRLoInv, m0[3]);
      // sign bit = (p < 0): the accumulators start at +0, so an exact zero is +0 (bit 0)
      sg[0][wi] |= ((__float_as_uint(p00) >> 31) | ((__float_as_uint(p01) >> 31) << 1)) << sh;
      sg[1][wi] |= ((__float_as_uint(p10) >> 31) | ((__float_as_uint(p11) >> 31) << 1)) << sh;
    }
    // gather the four lanes of the row: signs, codes
#pragma unroll
    for (int u = 0; u < 2; ++u) {
#pragma unroll
      for (int wi = 0; wi < 2; ++wi) {
        sg[u][wi] |= __shfl_xor_sync(0xffffffffu, sg[u][wi], 1);
        sg[u][wi] |= __shfl_xor_sync(0xffffffffu, sg[u][wi], 2);
      }
      code_bits[u] <<= 16 * (c & 1);
      code_bits[u] |= __shfl_xor_sync(0xffffffffu, code_bits[u], 1);
    }
    // code words: lanes c = 0, 1 hold word 0 (coordinates 0..31), c = 2, 3 word 1
    const uint32_t cw1[2] = {__shfl_xor_sync(0xffffffffu, code_bits[0], 2),
                             __shfl_xor_sync(0xffffffffu, code_bits[1], 2)};

    // ---- stores: lane c = 0 writes vector r, lane c = 1 vector r + 8
    if (c < 2) {
      const int u = c;
      const unsigned v = u ? vb : va;
      if (v < t.nvec) {
        const unsigned bh = v / static_cast<unsigned>(t.T);
        const unsigned tt = v - bh * static_cast<unsigned>(t.T);
        const size_t rec = static_cast<size_t>(bh) * t.T_cap + t.t_offset + tt;
        reinterpret_cast<uint2 *>(t.signs)[rec] = make_uint2(sg[u][0], sg[u][1]);
        if (wb1) reinterpret_cast<uint2 *>(t.codes)[rec] = make_uint2(code_bits[u], cw1[u]);
        t.norm[rec] = f32_to_f16_bits(nrm[u]);
        t.rnorm[rec] = f32_to_f16_bits(gam[u]);
      }
    }
  }
}

} // namespace

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
  auto kern = first->dtype == TQ_BF16 ? quantize_prod_kernel<true> : quantize_prod_kernel<false>;
  return launch_pdl(kern, dim3(static_cast<unsigned>(blocks)), dim3(kRWarps * 32), 0, s, f);
}

} // namespace tq
