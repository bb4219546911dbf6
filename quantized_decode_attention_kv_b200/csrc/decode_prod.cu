// Tensor-core decode attention over TurboQuant_prod records of head_dim 64 with 2-bit keys
// and values (1-bit Lloyd-Max codes + a 64-row QJL sign sketch of the residual + the
// residual norm), one or two query heads per KV head ("Closing - The Three-Step Summary",
// Step 3; "What the Paper Doesn't Tell You", Finding 2: the GPT-2 low-bit path).
//
// Every stored bit of a record is a +-1 factor: the 1-bit code selects -c1 or +c1, the QJL
// bit the sign of one projection. So per token the 128 bits (64 codes, then 64 signs) form
// one +-1 vector, exact in fp16, and both products of decode attention are tensor-core MMAs
// (mma.sync m16n8k16, fp16 x fp16 -> fp32) whose +-1 operand is built from the record bits
// with one shift and one mask per register (an A register pairs bits j and j + 16 of one
// record word, which lands them on the two fp16 sign bits; bit set = -1):
//
//   scores  S[16 tokens x 8] = A[16 x 128] . B[128 x 8]; per head four columns: the
//           code part (-c1 q~) and the sketch part (s^ = scale sqrt(pi/2)/(m sqrt(d)) S H D q),
//           each as an fp16 hi and a 2^12-scaled fp16 residual, in the record-bit order the
//           A registers use. score_t = ||k_t|| (code part + gamma_t * sketch part).
//   values  O^T[128 x heads] += A^T[128 x 16 tokens] . P'[16 tokens x heads], code rows with
//           P' = p ||v||, sketch rows with P' = p ||v|| gamma; the combine forms
//           u' = -c1 u (the codes' centroids), adds sqrt(d) sqrt(pi/2)/m S^T w, applies the
//           inverse rotation D H / d once and divides by the softmax sum.
//
// The work split, online softmax and partial records follow the MSE tensor-core kernel. The
// one-query-head kernel below scores on the CUDA cores instead and feeds the value MMAs the
// masked record bits (0 or an exact fp16 subnormal) with the sum of P' added back at the merge.
#include "mma_ops.cuh"

#include <algorithm>
#include <vector>
#include <type_traits>

namespace tq {
namespace {
using namespace mma_ops;

constexpr int kPW = 4;            // warps per CTA
constexpr int kPThreads = kPW * 32;
constexpr int kPD = 64;           // head_dim
constexpr int kPM = 64;           // QJL rows
constexpr float kPLoScale = 4096.0f;
constexpr float kPLoInv = 1.0f / 4096.0f;
constexpr float kPLog2e = 1.4426950408889634f;
constexpr float kPSqrtHalfPi = 1.2533141373155003f;
#ifndef TQ_PROD_PREFETCH
#define TQ_PROD_PREFETCH 3
#endif
constexpr int kPPrefetch = TQ_PROD_PREFETCH; // L2 prefetch distance in warp steps

// Prepared query of one (b, q-head): the B operand of the score MMA in fragment order.
// Word 16 c + 2 s (+1) holds the values at record bits 32 c + 2 s (+1) and 32 c + 2 s + 16
// (+1) of lane group c, k-step s; bits 0..63 are code bits (value -c1 q~_i), 64..127 sketch
// bits (value s^_j). inv[t] undoes the power-of-two normalisation of part t (codes, sketch).
struct QPrepP {
  uint32_t hi[64];
  uint32_t lo[64];
  float inv[2];
  float pad[2];
  float val[128]; // the per-bit values in record order (code part, then sketch part)
  float sum[2];   // sum of the code-part and of the sketch-part values
  float pad2[2];
};

__global__ void __launch_bounds__(kPD) qprep_prod_kernel(const void *q, int dtype, float scale,
                                                         uint64_t seed, const float *Sk, float c1,
                                                         QPrepP *out) {
  __shared__ float v[kPD];
  __shared__ float val[kPD + kPM];
  __shared__ float red[4];
  const int i = threadIdx.x;
  const size_t bq = blockIdx.x;
  pdl_wait(); // q may come from the kernel before
  pdl_trigger();
  float x = load_scalar(q, dtype, bq * kPD + i);
  if (sign_is_neg(seed, i)) x = -x;
  v[i] = x;
  __syncthreads();
  for (int hs = 1; hs < kPD; hs <<= 1) {
    float a = 0.f, b = 0.f;
    const bool lower = (i & hs) == 0;
    if (lower) {
      a = v[i];
      b = v[i + hs];
    }
    __syncthreads();
    if (lower) {
      v[i] = a + b;
      v[i + hs] = a - b;
    }
    __syncthreads();
  }
  // v = H D q; code part -c1 scale v / d, sketch part scale sqrt(pi/2) / (m sqrt(d)) S v
  const float sk_scale = scale * kPSqrtHalfPi / (static_cast<float>(kPM) * sqrtf(static_cast<float>(kPD)));
  float sacc = 0.f;
  const float *srow = Sk + static_cast<size_t>(i) * kPD;
  for (int k = 0; k < kPD; ++k) sacc = fmaf(__ldg(srow + k), v[k], sacc);
  val[i] = -c1 * v[i] * (scale / static_cast<float>(kPD));
  val[kPD + i] = sk_scale * sacc;
  // power-of-two normalisation per part so that max |value| lands in [1, 2)
  float m0 = warp_max(fabsf(val[i])), m1 = warp_max(fabsf(val[kPD + i]));
  if ((i & 31) == 0) {
    red[i >> 5] = m0;
    red[2 + (i >> 5)] = m1;
  }
  __syncthreads();
  float f[2];
  for (int t = 0; t < 2; ++t) {
    const float mx = fmaxf(red[2 * t], red[2 * t + 1]);
    f[t] = 1.0f;
    if (mx > 0.f && isfinite(mx)) {
      int ex;
      frexpf(mx, &ex);
      f[t] = ldexpf(1.0f, 1 - ex);
    }
  }
  // thread i writes fragment word i: lane group c, k-step s, second half of the pair if odd
  const int c = i >> 4, w = i & 15, s = w >> 1, odd = w & 1;
  const int e0 = 32 * c + 2 * s + odd, e1 = e0 + 16;
  const float y0 = val[e0] * f[e0 >> 6], y1 = val[e1] * f[e1 >> 6];
  const __half h0 = __float2half_rn(y0), h1 = __float2half_rn(y1);
  const __half l0 = __float2half_rn((y0 - __half2float(h0)) * kPLoScale);
  const __half l1 = __float2half_rn((y1 - __half2float(h1)) * kPLoScale);
  out[bq].hi[i] = static_cast<uint32_t>(__half_as_ushort(h0)) | (static_cast<uint32_t>(__half_as_ushort(h1)) << 16);
  out[bq].lo[i] = static_cast<uint32_t>(__half_as_ushort(l0)) | (static_cast<uint32_t>(__half_as_ushort(l1)) << 16);
  if (i == 0) {
    out[bq].inv[0] = 1.0f / f[0];
    out[bq].inv[1] = 1.0f / f[1];
  }
  out[bq].val[i] = val[i];
  out[bq].val[kPD + i] = val[kPD + i];
  float s0 = val[i], s1 = val[kPD + i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s0 += __shfl_xor_sync(0xffffffffu, s0, o);
    s1 += __shfl_xor_sync(0xffffffffu, s1, o);
  }
  __syncthreads(); // every thread has read the normalisation maxima from red
  if ((i & 31) == 0) {
    red[i >> 5] = s0;
    red[2 + (i >> 5)] = s1;
  }
  __syncthreads();
  if (i == 0) {
    out[bq].sum[0] = red[0] + red[1];
    out[bq].sum[1] = red[2] + red[3];
  }
}

struct ProdArgs {
  const uint8_t *kc, *ks, *vc, *vs;       // codes and sign sketches, 8 bytes per record each
  const uint16_t *kn, *kg, *vn, *vg;      // norms and residual norms (fp16 bits)
  const QPrepP *qp;
  float *part; // partial records [cta][slot][G][stride]
  int Hq, Hkv, G, T_len, T_cap;
  int tiles_per_bh, tiles_per_cta, slots, stride;
  long long total_tiles;
  uint32_t one2; // fp16 (1, 1): 0x3C003C00
  int B;
  const int *bt; // paged cache (ragged calls only): block table [B][maxp]; record (b, h, t) at
  int pshift, maxp; // ((bt[b][t >> pshift] * Hkv + h) << pshift) + (t mod page); else nullptr
};

// Record index of token t of (b, KV head) bh in a paged cache.
__device__ __forceinline__ long long prod_page_rec(const ProdArgs &a, long long bh, int t) {
  const long long b = bh / a.Hkv, h = bh - b * a.Hkv;
  const long long page = __ldg(a.bt + b * a.maxp + (t >> a.pshift));
  return ((page * a.Hkv + h) << a.pshift) + (t & ((1 << a.pshift) - 1));
}
struct NoVarLenP {};

// The segment of the flattened (b, KV head, 16-token tile) space that starts at tile `seg`:
// its (b, KV head), first tile, end and context length. A ragged call gives sequence b
// ceil(len[b] / 16) tiles per KV head, starting at tile boff[b] (vb: the sequence of the
// previous segment, advanced in place).
template <bool RAG>
__device__ __forceinline__ void prod_segment(const ProdArgs &a, const std::conditional_t<RAG, VarLen, NoVarLenP> &vl,
                                             long long seg, long long range1, int &vb, long long &bh,
                                             long long &seg_end, int &tile0, int &T_len) {
  if constexpr (RAG) {
    while (vb + 1 < a.B && vl.boff[vb + 1] <= seg) ++vb;
    T_len = vl.blen[vb];
    const int tpb = (T_len + 15) >> 4;
    const long long local = seg - vl.boff[vb];
    const int hh = static_cast<int>(local / tpb);
    tile0 = static_cast<int>(local - static_cast<long long>(hh) * tpb);
    bh = static_cast<long long>(vb) * a.Hkv + hh;
    seg_end = min(range1, vl.boff[vb] + static_cast<long long>(hh + 1) * tpb);
  } else {
    T_len = a.T_len;
    bh = seg / a.tiles_per_bh;
    seg_end = min(range1, (bh + 1) * a.tiles_per_bh);
    tile0 = static_cast<int>(seg - bh * a.tiles_per_bh);
  }
}

// +-1 fp16 pair from bits (j, j + 16) of w moved to the sign bits by a left shift of `sh`
// (sh = 15 - j): bit set = -1. `one2` holds fp16 (1, 1) in a register so that the mask and
// the OR are one LOP3.
__device__ __forceinline__ uint32_t pm1(uint32_t w, int sh, uint32_t one2) {
  uint32_t d;
  asm("lop3.b32 %0, %1, 0x80008000, %2, 0xEA;" : "=r"(d) : "r"(w << sh), "r"(one2));
  return d;
}

struct ProdTile {
  uint32_t kw[2];  // record word c (codes 0-1, signs 2-3) of tokens r, r + 8
  uint32_t vm[4];  // code word r / 4 of tokens 2c, 2c+1, 2c+8, 2c+9
  uint32_t vq[4];  // sign word r / 4 of the same tokens
  uint16_t kn[2], kg[2], vn[2], vg[2]; // norms and residual norms of tokens r, r + 8
};

template <bool RAG>
__global__ void __launch_bounds__(kPThreads, 3) decode_prod_kernel(const ProdArgs a,
                                                                   const std::conditional_t<RAG, VarLen, NoVarLenP> vl) {
  __shared__ float mst[kPW * 8];
  __shared__ float gmx[8];
  __shared__ float lsum[8];
  __shared__ float obuf[2][kPD + kPM];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = lane >> 2, c = lane & 3;
  const int gh = c >> 1, part = c & 1; // head and part of this lane's score columns
  const uint32_t one2 = a.one2;
  pdl_wait(); // the prepared queries and the cache are written by earlier kernels
  pdl_trigger();

  const long long range0 = static_cast<long long>(blockIdx.x) * a.tiles_per_cta;
  const long long range1 = min(a.total_tiles, range0 + a.tiles_per_cta);
  int slot = 0;
  int vb = 0;
  for (long long seg = range0; seg < range1; ++slot) {
    long long bh, seg_end;
    int tile0, T_len;
    prod_segment<RAG>(a, vl, seg, range1, vb, bh, seg_end, tile0, T_len);
    const int ntiles = static_cast<int>(seg_end - seg);
    seg = seg_end;
    const int b = static_cast<int>(bh / a.Hkv), h = static_cast<int>(bh % a.Hkv);

    // B operand of the score MMA: column r = head r / 4, part (r / 2) & 1, hi/lo r & 1; only
    // record words of that part (codes: c < 2, sketch: c >= 2) are non-zero.
    uint32_t qb[16];
    {
      const int g = r >> 2, t = (r >> 1) & 1;
      if (g < a.G && (c >= 2) == (t == 1)) {
        const QPrepP *p = a.qp + static_cast<size_t>(b) * a.Hq + h * a.G + g;
        const uint4 *src = reinterpret_cast<const uint4 *>(((r & 1) ? p->lo : p->hi) + 16 * c);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint4 w = __ldg(src + k);
          qb[4 * k] = w.x;
          qb[4 * k + 1] = w.y;
          qb[4 * k + 2] = w.z;
          qb[4 * k + 3] = w.w;
        }
      } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) qb[k] = 0u;
      }
    }
    const float pinv = gh < a.G ? __ldg(&a.qp[static_cast<size_t>(b) * a.Hq + h * a.G + gh].inv[part]) : 0.f;

    float m_run = -INFINITY, l_run = 0.f;
    float o[8][4];
#pragma unroll
    for (int m = 0; m < 8; ++m) o[m][0] = o[m][1] = o[m][2] = o[m][3] = 0.f;

    const size_t rec0 = static_cast<size_t>(bh) * a.T_cap;
    const bool paged = RAG && a.bt != nullptr; // paged: every tile through the block table
    const int tlast = T_len - 1;
    const uint8_t *kbase = (c < 2 ? a.kc : a.ks) + 4 * (c & 1);
    const int vwo = 4 * (r >> 2);
    const uint32_t selx = static_cast<uint32_t>(r & 3) | (static_cast<uint32_t>(4 + (r & 3)) << 8);
    int jl = warp;
    // L2 prefetch, kPrefetchSteps warp steps ahead: lanes 0-3 the 128-byte lines of a tile's
    // key codes, key signs, value codes and value signs; lanes 4-7 its four norm arrays.
    const int tp0 = (tile0 + warp) * 16 + kPPrefetch * kPW * 16;
    const char *pfp = nullptr;
    int pfstep = 0;
    {
      const int q = lane & 3;
      if (lane < 4) {
        const uint8_t *base = q == 0 ? a.kc : q == 1 ? a.ks : q == 2 ? a.vc : a.vs;
        pfp = reinterpret_cast<const char *>(base + (rec0 + tp0) * 8);
        pfstep = kPW * 16 * 8;
      } else if (lane < 8) {
        const uint16_t *base = q == 0 ? a.kn : q == 1 ? a.kg : q == 2 ? a.vn : a.vg;
        pfp = reinterpret_cast<const char *>(base + rec0 + tp0);
        pfstep = kPW * 16 * 2;
      }
    }
    int tpf = tp0;

    // lane pointers of the next full tile this warp loads (a warp advances 64 tokens)
    const int tw0 = (tile0 + warp) * 16;
    const uint8_t *kp = kbase + (rec0 + tw0 + r) * 8;
    const uint8_t *vcp = a.vc + (rec0 + tw0 + 2 * c) * 8 + vwo;
    const uint8_t *vsp = a.vs + (rec0 + tw0 + 2 * c) * 8 + vwo;
    const uint16_t *np[4] = {a.kn + rec0 + tw0 + r, a.kg + rec0 + tw0 + r, a.vn + rec0 + tw0 + r,
                             a.vg + rec0 + tw0 + r};

    auto load_next = [&](ProdTile &T) {
      if (!paged && lane < 8 && tpf + 16 <= T_len && tpf < (tile0 + ntiles) * 16)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(pfp));
      pfp += pfstep;
      tpf += kPW * 16;
      const int t0 = (tile0 + jl) * 16;
      if (!paged && t0 + 16 <= T_len) {
        T.kw[0] = __ldcs(reinterpret_cast<const uint32_t *>(kp));
        T.kw[1] = __ldcs(reinterpret_cast<const uint32_t *>(kp + 64));
        const int toff[4] = {0, 8, 64, 72};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          T.vm[e] = __ldcs(reinterpret_cast<const uint32_t *>(vcp + toff[e]));
          T.vq[e] = __ldcs(reinterpret_cast<const uint32_t *>(vsp + toff[e]));
        }
        T.kn[0] = __ldcs(np[0]);
        T.kn[1] = __ldcs(np[0] + 8);
        T.kg[0] = __ldcs(np[1]);
        T.kg[1] = __ldcs(np[1] + 8);
        T.vn[0] = __ldcs(np[2]);
        T.vn[1] = __ldcs(np[2] + 8);
        T.vg[0] = __ldcs(np[3]);
        T.vg[1] = __ldcs(np[3] + 8);
      } else {
        // record of token t (within this 16-token tile, so within one page) = base + t
        const long long base = paged ? prod_page_rec(a, bh, t0) - t0 : static_cast<long long>(rec0);
        const int tr = min(t0 + r, tlast), tr8 = min(t0 + r + 8, tlast);
        const int tv = t0 + 2 * c;
        const int tvs[4] = {min(tv, tlast), min(tv + 1, tlast), min(tv + 8, tlast), min(tv + 9, tlast)};
        T.kw[0] = __ldcs(reinterpret_cast<const uint32_t *>(kbase + (base + tr) * 8));
        T.kw[1] = __ldcs(reinterpret_cast<const uint32_t *>(kbase + (base + tr8) * 8));
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          T.vm[e] = __ldcs(reinterpret_cast<const uint32_t *>(a.vc + (base + tvs[e]) * 8 + vwo));
          T.vq[e] = __ldcs(reinterpret_cast<const uint32_t *>(a.vs + (base + tvs[e]) * 8 + vwo));
        }
        T.kn[0] = __ldcs(a.kn + base + tr);
        T.kn[1] = __ldcs(a.kn + base + tr8);
        T.kg[0] = __ldcs(a.kg + base + tr);
        T.kg[1] = __ldcs(a.kg + base + tr8);
        T.vn[0] = __ldcs(a.vn + base + tr);
        T.vn[1] = __ldcs(a.vn + base + tr8);
        T.vg[0] = __ldcs(a.vg + base + tr);
        T.vg[1] = __ldcs(a.vg + base + tr8);
      }
      kp += kPW * 16 * 8;
      vcp += kPW * 16 * 8;
      vsp += kPW * 16 * 8;
#pragma unroll
      for (int e = 0; e < 4; ++e) np[e] += kPW * 16;
      jl += kPW;
    };

    auto compute = [&](const ProdTile &T, int t0) {
      // ---- scores: one MMA per k-step; lane (r, c) gets part c & 1 of head c >> 1 for
      //      tokens r, r + 8 (hi in even columns, residual in odd columns)
      float acc[2][4];
#pragma unroll
      for (int u = 0; u < 2; ++u) acc[u][0] = acc[u][1] = acc[u][2] = acc[u][3] = 0.f;
#pragma unroll
      for (int s = 0; s < 8; ++s)
        mma16816(acc[s & 1], pm1(T.kw[0], 15 - 2 * s, one2), pm1(T.kw[1], 15 - 2 * s, one2),
                 pm1(T.kw[0], 14 - 2 * s, one2), pm1(T.kw[1], 14 - 2 * s, one2), qb[2 * s], qb[2 * s + 1]);
      const float mine0 = fmaf(acc[0][1] + acc[1][1], kPLoInv, acc[0][0] + acc[1][0]) * pinv;
      const float mine1 = fmaf(acc[0][3] + acc[1][3], kPLoInv, acc[0][2] + acc[1][2]) * pinv;
      const float oth0 = __shfl_xor_sync(0xffffffffu, mine0, 1);
      const float oth1 = __shfl_xor_sync(0xffffffffu, mine1, 1);
      const float code0 = part ? oth0 : mine0, sk0 = part ? mine0 : oth0;
      const float code1 = part ? oth1 : mine1, sk1 = part ? mine1 : oth1;
      const float kn0 = f16_bits_to_f32(T.kn[0]), kn1 = f16_bits_to_f32(T.kn[1]);
      const float kg0 = f16_bits_to_f32(T.kg[0]), kg1 = f16_bits_to_f32(T.kg[1]);
      const float vn0 = f16_bits_to_f32(T.vn[0]), vn1 = f16_bits_to_f32(T.vn[1]);
      const float vg0 = f16_bits_to_f32(T.vg[0]), vg1 = f16_bits_to_f32(T.vg[1]);
      const bool ok0 = t0 + r < T_len, ok1 = t0 + r + 8 < T_len;
      const float s0 = ok0 ? kn0 * fmaf(kg0, sk0, code0) * kPLog2e : -INFINITY;
      const float s1 = ok1 ? kn1 * fmaf(kg1, sk1, code1) * kPLog2e : -INFINITY;

      // ---- online softmax (log2 domain) over the lane's head. The reference moves only when a
      //      score of the tile exceeds it: one vote decides, and only then are the maxima
      //      reduced across the row group and the accumulators rescaled.
      if (__any_sync(0xffffffffu, s0 > m_run || s1 > m_run)) {
        float mx = fmaxf(s0, s1);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float mn = fmaxf(m_run, mx);
        const float alpha = softmax_exp2(m_run - mn);
        l_run *= alpha;
        m_run = mn;
        // lane (r, c) accumulates heads 2c, 2c + 1: head 0 lives on lanes c = 0, head 1 on c = 2
        const float al0 = __shfl_sync(0xffffffffu, alpha, lane & ~3);
        const float al1 = __shfl_sync(0xffffffffu, alpha, (lane & ~3) | 2);
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          o[m][0] *= al0;
          o[m][1] *= al1;
          o[m][2] *= al0;
          o[m][3] *= al1;
        }
      }
      const float p0 = softmax_exp2(s0 - m_run), p1 = softmax_exp2(s1 - m_run);
      l_run += p0 + p1;
      const uint32_t pkc = pack_h2(p0 * vn0, p1 * vn1);
      const uint32_t pks = pack_h2(p0 * vn0 * vg0, p1 * vn1 * vg1);

      // ---- P' operands (column r = head r): tokens 2c, 2c+1 (b0) and 2c+8, 2c+9 (b1)
      const int srca = 8 * c + 2 * (r & 1), srcb = srca + 4;
      uint32_t xc0 = __shfl_sync(0xffffffffu, pkc, srca), xc1 = __shfl_sync(0xffffffffu, pkc, srcb);
      uint32_t xs0 = __shfl_sync(0xffffffffu, pks, srca), xs1 = __shfl_sync(0xffffffffu, pks, srcb);
      if (r >= a.G) xc0 = xc1 = xs0 = xs1 = 0u;
      const uint32_t pbc0 = prmt(xc0, xc1, 0x5410u), pbc1 = prmt(xc0, xc1, 0x7632u);
      const uint32_t pbs0 = prmt(xs0, xs1, 0x5410u), pbs1 = prmt(xs0, xs1, 0x7632u);

      // ---- values: byte r & 3 of the lane's record word, first token in byte 0, second in
      //      byte 2, so bit i of the byte pair shifts onto the fp16 sign bits
      const uint32_t xm0 = prmt(T.vm[0], T.vm[1], selx), xm1 = prmt(T.vm[2], T.vm[3], selx);
      const uint32_t xq0 = prmt(T.vq[0], T.vq[1], selx), xq1 = prmt(T.vq[2], T.vq[3], selx);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int sh0 = 15 - 2 * m, sh1 = 14 - 2 * m;
        mma16816(o[m], pm1(xm0, sh0, one2), pm1(xm0, sh1, one2), pm1(xm1, sh0, one2),
                 pm1(xm1, sh1, one2), pbc0, pbc1);
        mma16816(o[4 + m], pm1(xq0, sh0, one2), pm1(xq0, sh1, one2), pm1(xq1, sh0, one2),
                 pm1(xq1, sh1, one2), pbs0, pbs1);
      }
    };

    ProdTile ta, tb;
    int jt = warp;
    if (jl < ntiles) load_next(ta);
    while (jt < ntiles) {
      if (jl < ntiles) load_next(tb);
      compute(ta, (tile0 + jt) * 16);
      jt += kPW;
      if (jt >= ntiles) break;
      if (jl < ntiles) load_next(ta);
      compute(tb, (tile0 + jt) * 16);
      jt += kPW;
    }

    // ---- merge the warps: common max per head, rescale, accumulate in shared memory
    float l = l_run;
    l += __shfl_xor_sync(0xffffffffu, l, 4);
    l += __shfl_xor_sync(0xffffffffu, l, 8);
    l += __shfl_xor_sync(0xffffffffu, l, 16);
    if (r == 0 && part == 0) mst[warp * 8 + gh] = m_run;
    for (int idx = tid; idx < 2 * (kPD + kPM); idx += kPThreads) (&obuf[0][0])[idx] = 0.f;
    if (tid < 8) lsum[tid] = 0.f;
    __syncthreads();
    if (tid < 2) {
      float M = -INFINITY;
      for (int w = 0; w < kPW; ++w) M = fmaxf(M, mst[w * 8 + tid]);
      gmx[tid] = M;
    }
    __syncthreads();
    if (r == 0 && part == 0 && gh < a.G) atomicAdd(&lsum[gh], l * exp2f(m_run - gmx[gh]));
    if (c == 0) {
      const float f0 = exp2f(mst[warp * 8] - gmx[0]);
      const float f1 = a.G > 1 ? exp2f(mst[warp * 8 + 1] - gmx[1]) : 0.f;
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int i0 = (m < 4 ? 0 : kPD) + 8 * r + 2 * (m & 3);
        atomicAdd(&obuf[0][i0], o[m][0] * f0);
        atomicAdd(&obuf[0][i0 + 1], o[m][2] * f0);
        if (a.G > 1) {
          atomicAdd(&obuf[1][i0], o[m][1] * f1);
          atomicAdd(&obuf[1][i0 + 1], o[m][3] * f1);
        }
      }
    }
    __syncthreads();
    float *dst = a.part + (static_cast<size_t>(blockIdx.x) * a.slots + slot) * a.G * a.stride;
    for (int idx = tid; idx < a.G * (kPD + kPM); idx += kPThreads) {
      const int g = idx / (kPD + kPM), i = idx - g * (kPD + kPM);
      dst[static_cast<size_t>(g) * a.stride + 2 + i] = obuf[g][i];
    }
    if (tid < a.G) {
      dst[static_cast<size_t>(tid) * a.stride] = gmx[tid];
      dst[static_cast<size_t>(tid) * a.stride + 1] = lsum[tid];
    }
    __syncthreads();
  }
}

// One query head per KV head (multi-head attention): the score of a token is a dot product of
// one query with 128 +-1 factors, so it is computed on the CUDA cores, one token per lane, from
// per-query tables T_p[byte] = -2 * (sum of the values of the set bits of byte p of a record):
// sum_k v_k (1 - 2 bit_k) = sum_k v_k + sum_p T_p[byte_p], 16 table reads per token instead of
// an MMA whose score columns would be 3/4 empty. The values stay on the tensor cores, with the
// record bits themselves (not +-1 factors) as the A operand, one mask per register (below).
struct LutTile {
  uint2 kc, ks;                // key codes and sketch of token `lane` of the group
  uint16_t kn, kg, vn, vg;     // its norms
  uint32_t vm[2][4], vq[2][4]; // value code / sketch word r/4 of tokens 16 h + {2c, 2c+1, 2c+8, 2c+9}
};

template <bool RAG>
__global__ void __launch_bounds__(kPThreads, 3) decode_prod_lut_kernel(const ProdArgs a,
                                                                       const std::conditional_t<RAG, VarLen, NoVarLenP> vl) {
  __shared__ float tab[16 * 256];
  __shared__ float mst[kPW];
  __shared__ float gmx, lsum;
  __shared__ float obuf[kPD + kPM];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = lane >> 2, c = lane & 3;
  const uint32_t one2 = a.one2;
  pdl_wait(); // the prepared queries and the cache are written by earlier kernels
  pdl_trigger();

  const long long range0 = static_cast<long long>(blockIdx.x) * a.tiles_per_cta;
  const long long range1 = min(a.total_tiles, range0 + a.tiles_per_cta);
  int slot = 0;
  int vb = 0;
  for (long long seg = range0; seg < range1; ++slot) {
    long long bh, seg_end;
    int tile0, T_len;
    prod_segment<RAG>(a, vl, seg, range1, vb, bh, seg_end, tile0, T_len);
    const int ntiles = static_cast<int>(seg_end - seg);
    seg = seg_end;
    const int b = static_cast<int>(bh / a.Hkv), h = static_cast<int>(bh % a.Hkv);

    // ---- the query's tables (one query head: q-head h of sequence b)
    const QPrepP *qp = a.qp + static_cast<size_t>(b) * a.Hq + h;
    __syncthreads(); // the previous segment's readers are done with tab
    for (int e = tid; e < 16 * 256; e += kPThreads) {
      const float *v = qp->val + 8 * (e >> 8);
      const int byte = e & 255;
      float acc = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) acc += ((byte >> k) & 1) ? __ldg(v + k) : 0.f;
      tab[e] = -2.0f * acc;
    }
    const float csum = __ldg(&qp->sum[0]), ssum = __ldg(&qp->sum[1]);
    __syncthreads();

    float m_run = -INFINITY, l_run = 0.f;
    float s_code = 0.f, s_sketch = 0.f; // the lane's running sums of P' (code rows, sketch rows)
    float o[8][4];
#pragma unroll
    for (int m = 0; m < 8; ++m) o[m][0] = o[m][1] = o[m][2] = o[m][3] = 0.f;

    const size_t rec0 = static_cast<size_t>(bh) * a.T_cap;
    const bool paged = RAG && a.bt != nullptr; // paged: every record through the block table
    auto recof = [&](int t) -> long long {
      return paged ? prod_page_rec(a, bh, t) : static_cast<long long>(rec0) + t;
    };
    const int ts = tile0 * 16, te = min((tile0 + ntiles) * 16, T_len); // segment tokens
    const int ngroups = (te - ts + 31) / 32;
    const int vwo = 4 * (r >> 2);
    const uint32_t selx = static_cast<uint32_t>(r & 3) | (static_cast<uint32_t>(4 + (r & 3)) << 8);
    int jl = warp;

    // lane pointers of the next full group this warp loads (a warp advances kPW groups)
    const size_t tw0 = rec0 + ts + 32 * warp;
    const uint2 *kcp = reinterpret_cast<const uint2 *>(a.kc) + tw0 + lane;
    const uint2 *ksp = reinterpret_cast<const uint2 *>(a.ks) + tw0 + lane;
    const uint16_t *np[4] = {a.kn + tw0 + lane, a.kg + tw0 + lane, a.vn + tw0 + lane, a.vg + tw0 + lane};
    const uint8_t *vcp = a.vc + (tw0 + 2 * c) * 8 + vwo;
    const uint8_t *vsp = a.vs + (tw0 + 2 * c) * 8 + vwo;

    auto load_next = [&](LutTile &T) {
      const int t0 = ts + 32 * jl;
      if (!paged && t0 + 32 <= te) {
        T.kc = __ldcs(kcp);
        T.ks = __ldcs(ksp);
        T.kn = __ldcs(np[0]);
        T.kg = __ldcs(np[1]);
        T.vn = __ldcs(np[2]);
        T.vg = __ldcs(np[3]);
        const int toff[4] = {0, 8, 64, 72}; // tokens 2c, 2c+1, 2c+8, 2c+9 (bytes)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            T.vm[hh][e] = __ldcs(reinterpret_cast<const uint32_t *>(vcp + 128 * hh + toff[e]));
            T.vq[hh][e] = __ldcs(reinterpret_cast<const uint32_t *>(vsp + 128 * hh + toff[e]));
          }
      } else {
        const long long tk = recof(min(t0 + lane, te - 1));
        T.kc = __ldcs(reinterpret_cast<const uint2 *>(a.kc) + tk);
        T.ks = __ldcs(reinterpret_cast<const uint2 *>(a.ks) + tk);
        T.kn = __ldcs(a.kn + tk);
        T.kg = __ldcs(a.kg + tk);
        T.vn = __ldcs(a.vn + tk);
        T.vg = __ldcs(a.vg + tk);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int tv = t0 + 16 * hh + 2 * c;
          const int tvs[4] = {min(tv, te - 1), min(tv + 1, te - 1), min(tv + 8, te - 1), min(tv + 9, te - 1)};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const long long tr = recof(tvs[e]);
            T.vm[hh][e] = __ldcs(reinterpret_cast<const uint32_t *>(a.vc + tr * 8 + vwo));
            T.vq[hh][e] = __ldcs(reinterpret_cast<const uint32_t *>(a.vs + tr * 8 + vwo));
          }
        }
      }
      kcp += kPW * 32;
      ksp += kPW * 32;
#pragma unroll
      for (int e = 0; e < 4; ++e) np[e] += kPW * 32;
      vcp += kPW * 32 * 8;
      vsp += kPW * 32 * 8;
      jl += kPW;
    };

    // table offset (bytes) of byte k of a record word, for table block p: ((w >> 8k) & 255) * 4
    auto tab_at = [&](uint32_t w, int k, int p) -> float {
      const uint32_t off = (k == 0 ? (w << 2) : (w >> (8 * k - 2))) & 0x3FCu;
      return *reinterpret_cast<const float *>(reinterpret_cast<const uint8_t *>(tab) + p * 1024 + off);
    };

    auto compute = [&](const LutTile &T, int t0) {
      // ---- scores: one token per lane
      float sc = 0.f, sk = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        sc += tab_at(T.kc.x, k, k) + tab_at(T.kc.y, k, 4 + k);
        sk += tab_at(T.ks.x, k, 8 + k) + tab_at(T.ks.y, k, 12 + k);
      }
      const float kn = f16_bits_to_f32(T.kn), kg = f16_bits_to_f32(T.kg);
      const float s = t0 + lane < te ? kn * (csum + sc + kg * (ssum + sk)) * kPLog2e : -INFINITY;
      // ---- online softmax over the 32 tokens of the group (one head: the reference is
      //      warp-uniform); the group's maximum is reduced only when a vote finds a score above
      //      the reference
      if (__any_sync(0xffffffffu, s > m_run)) {
        float mx = s;
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
        const float mn = fmaxf(m_run, mx);
        const float alpha = softmax_exp2(m_run - mn);
        l_run *= alpha;
        s_code *= alpha;
        s_sketch *= alpha;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          o[m][0] *= alpha;
          o[m][1] *= alpha;
          o[m][2] *= alpha;
          o[m][3] *= alpha;
        }
        m_run = mn;
      }
      const float pr = softmax_exp2(s - m_run);
      l_run += pr;
      const float vn = f16_bits_to_f32(T.vn), vg = f16_bits_to_f32(T.vg);
      const uint32_t pk = pack_h2(pr * vn, pr * vn * vg); // (code rows, sketch rows)

      // ---- values: two 16-token MMA groups; P' column 0 = the head (other columns zero).
      //      The operand is the record bit itself, not a +-1 factor: an A register masks bit p of
      //      both halves of the byte-pair word, which is the fp16 value 2^(p-24) where the bit is
      //      set (an exact subnormal) and 0 where it is clear. The group's two MMAs start from
      //      zero, so M = 2^(p-24) sum_t b_t P'_t is small and exact up to the fp32 sum, and the
      //      accumulator takes -2^(25-p) M = -2 sum_t b_t P'_t; the running sums of P' (code and
      //      sketch rows) supply the sum_t P'_t of sum_t P'_t (1 - 2 b_t) at the merge.
      s_code += __low2float(*reinterpret_cast<const __half2 *>(&pk));
      s_sketch += __high2float(*reinterpret_cast<const __half2 *>(&pk));
      uint32_t pbc[2][2], pbs[2][2], xm[2][2], xq[2][2];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int base = 16 * hh + 2 * c;
        const uint32_t x0 = __shfl_sync(0xffffffffu, pk, base), x1 = __shfl_sync(0xffffffffu, pk, base + 1);
        const uint32_t x8 = __shfl_sync(0xffffffffu, pk, base + 8), x9 = __shfl_sync(0xffffffffu, pk, base + 9);
        pbc[hh][0] = r == 0 ? prmt(x0, x1, 0x5410u) : 0u;
        pbc[hh][1] = r == 0 ? prmt(x8, x9, 0x5410u) : 0u;
        pbs[hh][0] = r == 0 ? prmt(x0, x1, 0x7632u) : 0u;
        pbs[hh][1] = r == 0 ? prmt(x8, x9, 0x7632u) : 0u;
        xm[hh][0] = prmt(T.vm[hh][0], T.vm[hh][1], selx);
        xm[hh][1] = prmt(T.vm[hh][2], T.vm[hh][3], selx);
        xq[hh][0] = prmt(T.vq[hh][0], T.vq[hh][1], selx);
        xq[hh][1] = prmt(T.vq[hh][2], T.vq[hh][3], selx);
      }
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const uint32_t mk0 = 0x10001u << (2 * m), mk1 = 0x10001u << (2 * m + 1);
        float mc[4] = {0.f, 0.f, 0.f, 0.f}, ms[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          mma16816(mc, xm[hh][0] & mk0, xm[hh][0] & mk1, xm[hh][1] & mk0, xm[hh][1] & mk1, pbc[hh][0], pbc[hh][1]);
          mma16816(ms, xq[hh][0] & mk0, xq[hh][0] & mk1, xq[hh][1] & mk0, xq[hh][1] & mk1, pbs[hh][0], pbs[hh][1]);
        }
        // rows r (bit 2m) and r + 8 (bit 2m + 1)
        const float c0 = -static_cast<float>(1 << (25 - 2 * m)), c1 = -static_cast<float>(1 << (24 - 2 * m));
        o[m][0] = fmaf(mc[0], c0, o[m][0]);
        o[m][1] = fmaf(mc[1], c0, o[m][1]);
        o[m][2] = fmaf(mc[2], c1, o[m][2]);
        o[m][3] = fmaf(mc[3], c1, o[m][3]);
        o[4 + m][0] = fmaf(ms[0], c0, o[4 + m][0]);
        o[4 + m][1] = fmaf(ms[1], c0, o[4 + m][1]);
        o[4 + m][2] = fmaf(ms[2], c1, o[4 + m][2]);
        o[4 + m][3] = fmaf(ms[3], c1, o[4 + m][3]);
      }
    };

    LutTile ta, tb;
    int jt = warp;
    if (jl < ngroups) load_next(ta);
    while (jt < ngroups) {
      if (jl < ngroups) load_next(tb);
      compute(ta, ts + 32 * jt);
      jt += kPW;
      if (jt >= ngroups) break;
      if (jl < ngroups) load_next(ta);
      compute(tb, ts + 32 * jt);
      jt += kPW;
    }

    // ---- merge the warps (one head); a row's value is sum_t P'_t (1 - 2 b_t) = (the sum of
    //      P' over the warp's tokens) + the accumulator
    float l = l_run;
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) {
      l += __shfl_xor_sync(0xffffffffu, l, o2);
      s_code += __shfl_xor_sync(0xffffffffu, s_code, o2);
      s_sketch += __shfl_xor_sync(0xffffffffu, s_sketch, o2);
    }
    if (lane == 0) mst[warp] = m_run;
    for (int idx = tid; idx < kPD + kPM; idx += kPThreads) obuf[idx] = 0.f;
    if (tid == 0) lsum = 0.f;
    __syncthreads();
    if (tid == 0) {
      float M = -INFINITY;
      for (int w = 0; w < kPW; ++w) M = fmaxf(M, mst[w]);
      gmx = M;
    }
    __syncthreads();
    const float f = exp2f(m_run - gmx);
    if (lane == 0) atomicAdd(&lsum, l * f);
    if (c == 0) {
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int i0 = (m < 4 ? 0 : kPD) + 8 * r + 2 * (m & 3);
        const float sp = m < 4 ? s_code : s_sketch;
        atomicAdd(&obuf[i0], (sp + o[m][0]) * f);
        atomicAdd(&obuf[i0 + 1], (sp + o[m][2]) * f);
      }
    }
    __syncthreads();
    float *dst = a.part + (static_cast<size_t>(blockIdx.x) * a.slots + slot) * a.stride;
    for (int idx = tid; idx < kPD + kPM; idx += kPThreads) dst[2 + idx] = obuf[idx];
    if (tid == 0) {
      dst[0] = gmx;
      dst[1] = lsum;
    }
  }
}

// Merge the partial records of one (b, q-head); u' = -c1 u, add sqrt(d) sqrt(pi/2)/m S^T w,
// apply the inverse rotation D H / d and divide by the softmax sum. One warp per (b, q-head);
// lane l owns coordinates 2 l, 2 l + 1 and sketch rows 2 l, 2 l + 1.
template <bool RAG>
__global__ void __launch_bounds__(128) combine_prod_kernel(const float *part, int B, int Hkv, int G,
                                                           int tiles_per_bh, int tiles_per_cta,
                                                           int slots, int stride, uint64_t seed,
                                                           const float *Sv, float c1v, float *out,
                                                           const std::conditional_t<RAG, VarLen, NoVarLenP> vl) {
  const int lane = threadIdx.x & 31;
  const int Hq = Hkv * G;
  const int gw = blockIdx.x * 4 + (threadIdx.x >> 5);
  pdl_wait(); // the partials come from the decode kernel
  if (gw >= B * Hq) return;
  const int b = gw / Hq, hq = gw - b * Hq;
  const int h = hq / G, g = hq - h * G;
  const long long bh = static_cast<long long>(b) * Hkv + h;
  // the (b, KV head) of flattened tile f (ragged calls: sequence by binary search)
  auto bh_of = [&](long long f) -> long long {
    if constexpr (!RAG) {
      return f / tiles_per_bh;
    } else {
      int lo = 0, hi = B - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (vl.boff[mid] <= f) lo = mid;
        else hi = mid - 1;
      }
      const int tpb = (vl.blen[lo] + 15) >> 4;
      return static_cast<long long>(lo) * Hkv + (f - vl.boff[lo]) / tpb;
    }
  };
  int tpb = tiles_per_bh;
  long long first = bh * tiles_per_bh;
  if constexpr (RAG) {
    tpb = (vl.blen[b] + 15) >> 4;
    first = vl.boff[b] + static_cast<long long>(h) * tpb;
  }
  const long long last = first + tpb - 1;
  const int cta0 = static_cast<int>(first / tiles_per_cta), cta1 = static_cast<int>(last / tiles_per_cta);
  auto rec = [&](int cta) {
    const long long bh0 = bh_of(static_cast<long long>(cta) * tiles_per_cta);
    return part + ((static_cast<size_t>(cta) * slots + (bh - bh0)) * G + g) * stride;
  };
  float M = -INFINITY;
  for (int c = cta0 + lane; c <= cta1; c += 32) M = fmaxf(M, rec(c)[0]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float L = 0.f, u0 = 0.f, u1 = 0.f, w0 = 0.f, w1 = 0.f;
  for (int c0 = cta0; c0 <= cta1; c0 += 32) {
    const int c = c0 + lane;
    float e = 0.f;
    if (c <= cta1) {
      const float *p = rec(c);
      e = exp2f(p[0] - M);
      L = fmaf(e, p[1], L);
    }
    const int n = min(32, cta1 - c0 + 1);
    for (int k = 0; k < n; ++k) {
      const float ek = __shfl_sync(0xffffffffu, e, k);
      const float *p = rec(c0 + k) + 2;
      const float2 uu = *reinterpret_cast<const float2 *>(p + 2 * lane);
      const float2 ww = *reinterpret_cast<const float2 *>(p + kPD + 2 * lane);
      u0 = fmaf(ek, uu.x, u0);
      u1 = fmaf(ek, uu.y, u1);
      w0 = fmaf(ek, ww.x, w0);
      w1 = fmaf(ek, ww.y, w1);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
  // y = S^T w for this lane's two coordinates
  float y0 = 0.f, y1 = 0.f;
#pragma unroll 8
  for (int j = 0; j < kPM; ++j) {
    const float wj = __shfl_sync(0xffffffffu, (j & 1) ? w1 : w0, j >> 1);
    const float2 sj = __ldg(reinterpret_cast<const float2 *>(Sv + static_cast<size_t>(j) * kPD) + lane);
    y0 = fmaf(sj.x, wj, y0);
    y1 = fmaf(sj.y, wj, y1);
  }
  const float kap = sqrtf(static_cast<float>(kPD)) * kPSqrtHalfPi / static_cast<float>(kPM);
  float x0 = fmaf(kap, y0, -c1v * u0), x1 = fmaf(kap, y1, -c1v * u1);
  // inverse rotation: the span-1 butterfly in the lane, spans 2..32 across lanes
  {
    const float a0 = x0 + x1, a1 = x0 - x1;
    x0 = a0;
    x1 = a1;
  }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
    const float o0 = __shfl_xor_sync(0xffffffffu, x0, m);
    const float o1 = __shfl_xor_sync(0xffffffffu, x1, m);
    x0 = upper ? o0 - x0 : x0 + o0;
    x1 = upper ? o1 - x1 : x1 + o1;
  }
  const float sc = 1.0f / (static_cast<float>(kPD) * L);
  const uint64_t sw = dev_splitmix64(seed, 0);
  float2 res;
  res.x = ((sw >> (2 * lane)) & 1ull) ? -x0 * sc : x0 * sc;
  res.y = ((sw >> (2 * lane + 1)) & 1ull) ? -x1 * sc : x1 * sc;
  reinterpret_cast<float2 *>(out + (static_cast<size_t>(b) * Hq + hq) * kPD)[lane] = res;
}

} // namespace

bool prod_decode_supported(int d, int k_mode, int k_bits, int k_m, int v_mode, int v_bits, int v_m,
                           int G) {
  return d == kPD && k_mode == TQ_PROD && k_bits == 2 && k_m == kPM && v_mode == TQ_PROD &&
         v_bits == 2 && v_m == kPM && G >= 1 && G <= 2;
}

void plan_prod(int B, int Hq, int Hkv, int T_len, int sm_count, DecodePlan *p, const int *T_lens) {
  const int G = Hq / Hkv;
  p->path = 2;
  p->tile = 16;
  p->gc = G;
  p->ws_stride = 2 + kPD + kPM + 2; // 132 floats
  p->tiles_per_bh = (T_len + 15) / 16;
  long long total = static_cast<long long>(B) * Hkv * p->tiles_per_bh;
  if (T_lens) {
    total = 0;
    for (int b = 0; b < B; ++b) total += static_cast<long long>(Hkv) * ((T_lens[b] + 15) / 16);
  }
  long long ctas = static_cast<long long>(sm_count) * 3;
  ctas = std::min<long long>(ctas, (total + 7) / 8); // at least 8 tiles per CTA
  ctas = std::max<long long>(ctas, 1);
  p->tiles_per_cta = static_cast<int>((total + ctas - 1) / ctas);
  p->ctas = static_cast<int>((total + p->tiles_per_cta - 1) / p->tiles_per_cta);
  p->slots = (p->tiles_per_cta + p->tiles_per_bh - 1) / p->tiles_per_bh + 1;
  if (T_lens) { // the most (b, KV head) segments any CTA's range touches
    std::vector<int> nseg(p->ctas, 0);
    long long off = 0;
    for (int b = 0; b < B; ++b) {
      const int tpb = (T_lens[b] + 15) / 16;
      for (int h = 0; h < Hkv; ++h, off += tpb) {
        const int c0 = static_cast<int>(off / p->tiles_per_cta);
        const int c1 = static_cast<int>((off + tpb - 1) / p->tiles_per_cta);
        for (int c = c0; c <= c1; ++c) ++nseg[c];
      }
    }
    p->slots = *std::max_element(nseg.begin(), nseg.end());
  }
  p->splits = 0;
  p->chunk = 0;
  p->part_bytes = static_cast<size_t>(p->ctas) * p->slots * G * p->ws_stride * sizeof(float);
  p->part_bytes = (p->part_bytes + 255) / 256 * 256;
  p->ws_bytes = p->part_bytes + static_cast<size_t>(B) * Hq * sizeof(QPrepP);
}

cudaError_t launch_prod_decode(const DecodeArgs &a, cudaStream_t s) {
  const DecodePlan &p = a.plan;
  QPrepP *qp = reinterpret_cast<QPrepP *>(reinterpret_cast<uint8_t *>(a.ws) + p.part_bytes);
  cudaError_t e = launch_pdl(qprep_prod_kernel, dim3(a.B * a.Hq), dim3(kPD), 0, s, a.q, a.q_dtype,
                             a.scale, a.seed, a.k.S, a.k.cb.c[1], qp);
  if (e != cudaSuccess) return e;
  ProdArgs f;
  f.kc = a.k.codes;
  f.ks = a.k.signs;
  f.vc = a.v.codes;
  f.vs = a.v.signs;
  f.kn = a.k.norm;
  f.kg = a.k.rnorm;
  f.vn = a.v.norm;
  f.vg = a.v.rnorm;
  f.qp = qp;
  f.part = a.ws;
  f.Hq = a.Hq;
  f.Hkv = a.Hkv;
  f.G = a.Hq / a.Hkv;
  f.T_len = a.T_len;
  f.T_cap = a.T_cap;
  f.tiles_per_bh = p.tiles_per_bh;
  f.tiles_per_cta = p.tiles_per_cta;
  f.slots = p.slots;
  f.stride = p.ws_stride;
  f.total_tiles = static_cast<long long>(a.B) * a.Hkv * p.tiles_per_bh;
  f.one2 = 0x3C003C00u;
  f.B = a.B;
  f.bt = a.pg.bt;
  f.pshift = a.pg.pshift;
  f.maxp = a.pg.maxp;
  if (a.T_lens) {
    // ragged batch: the per-sequence lengths and tile offsets travel as launch parameters
    VarLen vl;
    vl.on = 1;
    vl.boff[0] = 0;
    for (int b = 0; b < a.B; ++b) {
      vl.blen[b] = a.T_lens[b];
      vl.boff[b + 1] = vl.boff[b] + a.Hkv * ((a.T_lens[b] + 15) / 16);
    }
    f.total_tiles = vl.boff[a.B];
    e = launch_pdl(f.G == 1 ? decode_prod_lut_kernel<true> : decode_prod_kernel<true>, dim3(p.ctas),
                   dim3(kPThreads), 0, s, f, vl);
    if (e != cudaSuccess) return e;
    return launch_pdl(combine_prod_kernel<true>, dim3((a.B * a.Hq + 3) / 4), dim3(128), 0, s,
                      static_cast<const float *>(a.ws), a.B, a.Hkv, f.G, p.tiles_per_bh, p.tiles_per_cta,
                      p.slots, p.ws_stride, a.seed, a.v.S, a.v.cb.c[1], a.out, vl);
  }
  e = launch_pdl(f.G == 1 ? decode_prod_lut_kernel<false> : decode_prod_kernel<false>, dim3(p.ctas),
                 dim3(kPThreads), 0, s, f, NoVarLenP{});
  if (e != cudaSuccess) return e;
  return launch_pdl(combine_prod_kernel<false>, dim3((a.B * a.Hq + 3) / 4), dim3(128), 0, s,
                    static_cast<const float *>(a.ws), a.B, a.Hkv, f.G, p.tiles_per_bh,
                    p.tiles_per_cta, p.slots, p.ws_stride, a.seed, a.v.S, a.v.cb.c[1], a.out, NoVarLenP{});
}
} // namespace tq
