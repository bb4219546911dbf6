// Split-K decode attention over the compressed cache, its combine step, and the same design
// over an unquantised bf16 cache.
//
// "Where This Fits in the Inference Stack", TensorRT-LLM section: the packed K/V codes are
// read from HBM and dequantised in registers inside the attention kernel (no separate
// dequantise pass). The query is rotated once per CTA, so a key's score is
// ||k|| * sum_i q~_i c[code_i] with q~ = scale * H D q / d; values accumulate in the rotated
// domain (u' = sum_t p_t ||v_t|| c[vcode_t]) and the combine kernel applies the single
// inverse rotation D H / d to the merged accumulator.
//
// Grid of the split kernel: (context splits, KV heads x query-head groups, batch).
// Each CTA streams its token range in tiles of 128 tokens: one thread scores one token for
// all of the CTA's query heads, the tile's max and the online-softmax rescale are shared
// through shared memory, then one thread per coordinate accumulates p * ||v|| * c[vcode].
#include "tq_device.cuh"

#include <algorithm>
#include <cmath>
#include <mutex>

namespace tq {
namespace {

constexpr int kThreads = 128;
constexpr int kTile = 128;
constexpr float kSqrtHalfPi = 1.2533141373155003f; // sqrt(pi/2)

__host__ __device__ inline int round_up(int v, int m) { return (v + m - 1) / m * m; }

// Row stride (bytes) of a staged tile of records: at least one spare byte (a code may be read
// as a 16-bit window) and an odd number of 32-bit words, so one-thread-per-row reads hit
// distinct banks.
__host__ __device__ inline int staged_stride(int bytes) {
  if (bytes == 0) return 0;
  int words = (bytes + 1 + 3) / 4;
  if ((words & 1) == 0) ++words;
  return words * 4;
}

struct SmemLayout {
  int lutk, lutv, qt, qsk, kc, vc, ks, vs, kn, vn, krn, vrn, pw, pg, red, es, total;
};

__host__ __device__ inline SmemLayout make_layout(int d, int gc, const TensorArgs &k,
                                                  const TensorArgs &v) {
  SmemLayout L;
  int o = 0;
  auto take = [&](int bytes) {
    int at = o;
    o = round_up(o + bytes, 16);
    return at;
  };
  L.lutk = take(16 * 4);
  L.lutv = take(16 * 4);
  L.qt = take(gc * d * 4);
  L.qsk = take(gc * k.m * 4);
  L.kc = take(kTile * staged_stride(k.code_bytes));
  L.vc = take(kTile * staged_stride(v.code_bytes));
  L.ks = take(kTile * staged_stride(k.sign_bytes));
  L.vs = take(kTile * staged_stride(v.sign_bytes));
  L.kn = take(kTile * 4);
  L.vn = take(kTile * 4);
  L.krn = take(kTile * 4);
  L.vrn = take(kTile * 4);
  L.pw = take(gc * kTile * 4);
  L.pg = take(gc * kTile * 4);
  L.red = take(gc * 8 * 4);
  L.es = 0;
  L.total = o;
  return L;
}

__device__ __forceinline__ uint32_t get_code(const uint8_t *row, int i, int w) {
  const int bit = i * w;
  const uint32_t v = static_cast<uint32_t>(row[bit >> 3]) |
                     (static_cast<uint32_t>(row[(bit >> 3) + 1]) << 8);
  return (v >> (bit & 7)) & ((1u << w) - 1u);
}

// Copy n rows of `bytes` bytes (contiguous in global memory) into a tile with row stride
// `stride`, using 16- or 4-byte accesses when the record size allows.
__device__ __forceinline__ void stage_rows(uint8_t *dst, int stride, const uint8_t *src, int bytes,
                                           int n) {
  if (bytes == 0) return;
  if ((bytes & 15) == 0) {
    const int per = bytes / 16;
    for (int idx = threadIdx.x; idx < n * per; idx += kThreads) {
      const int r = idx / per, c = idx - r * per;
      const uint4 v = __ldg(reinterpret_cast<const uint4 *>(src + static_cast<size_t>(r) * bytes) + c);
      uint32_t *d = reinterpret_cast<uint32_t *>(dst + r * stride + c * 16);
      d[0] = v.x;
      d[1] = v.y;
      d[2] = v.z;
      d[3] = v.w;
    }
  } else if ((bytes & 3) == 0) {
    const int per = bytes / 4;
    for (int idx = threadIdx.x; idx < n * per; idx += kThreads) {
      const int r = idx / per, c = idx - r * per;
      reinterpret_cast<uint32_t *>(dst + r * stride)[c] =
          __ldg(reinterpret_cast<const uint32_t *>(src + static_cast<size_t>(r) * bytes) + c);
    }
  } else {
    for (int idx = threadIdx.x; idx < n * bytes; idx += kThreads) {
      const int r = idx / bytes, c = idx - r * bytes;
      dst[r * stride + c] = __ldg(src + static_cast<size_t>(r) * bytes + c);
    }
  }
}

template <int D, int GC>
__global__ void __launch_bounds__(kThreads) decode_split_kernel(const DecodeArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const SmemLayout L = make_layout(D, GC, a.k, a.v);
  float *lutk = reinterpret_cast<float *>(smem + L.lutk);
  float *lutv = reinterpret_cast<float *>(smem + L.lutv);
  float *qt = reinterpret_cast<float *>(smem + L.qt);
  float *qsk = reinterpret_cast<float *>(smem + L.qsk);
  uint8_t *kc = smem + L.kc;
  uint8_t *vc = smem + L.vc;
  uint8_t *ks = smem + L.ks;
  uint8_t *vs = smem + L.vs;
  float *kn = reinterpret_cast<float *>(smem + L.kn);
  float *vn = reinterpret_cast<float *>(smem + L.vn);
  float *krn = reinterpret_cast<float *>(smem + L.krn);
  float *vrn = reinterpret_cast<float *>(smem + L.vrn);
  float *pw = reinterpret_cast<float *>(smem + L.pw);
  float *pg = reinterpret_cast<float *>(smem + L.pg);
  float *red = reinterpret_cast<float *>(smem + L.red);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = a.Hq / a.Hkv;
  const int ngrp = (G + GC - 1) / GC;
  const int h = blockIdx.y / ngrp, grp = blockIdx.y - h * ngrp;
  const int g0 = grp * GC;
  const int gcount = min(GC, G - g0);
  const int b = blockIdx.z;
  const int split = blockIdx.x;
  const int t_begin = split * a.plan.chunk;
  const int t_end = min(a.T_len, t_begin + a.plan.chunk);
  const size_t bh = static_cast<size_t>(b) * a.Hkv + h;
  const bool kprod = a.k.mode == TQ_PROD, vprod = a.v.mode == TQ_PROD;
  const int kw = a.k.wbits, vw = a.v.wbits;
  const int mk = a.k.m, mv = a.v.m;
  const int kstr = staged_stride(a.k.code_bytes), vstr = staged_stride(a.v.code_bytes);
  const int ksstr = staged_stride(a.k.sign_bytes), vsstr = staged_stride(a.v.sign_bytes);

  if (tid < 16) {
    lutk[tid] = tid < a.k.cb.levels ? a.k.cb.c[tid] : 0.f;
    lutv[tid] = tid < a.v.cb.levels ? a.v.cb.c[tid] : 0.f;
  }
  // ---- rotate the query once: q'' = H D q (unnormalised), kept in shared memory
  for (int idx = tid; idx < GC * D; idx += kThreads) {
    const int g = idx / D, i = idx - (idx / D) * D;
    float v = 0.f;
    if (g < gcount) {
      const size_t qi = (static_cast<size_t>(b) * a.Hq + h * G + g0 + g) * D + i;
      v = load_scalar(a.q, a.q_dtype, qi);
      if (sign_is_neg(a.seed, i)) v = -v;
    }
    qt[idx] = v;
  }
  __syncthreads();
  for (int hs = 1; hs < D; hs <<= 1) {
    for (int idx = tid; idx < GC * (D / 2); idx += kThreads) {
      const int g = idx / (D / 2), k = idx - g * (D / 2);
      const int i = (k / hs) * 2 * hs + (k % hs);
      float *row = qt + g * D;
      const float x0 = row[i], x1 = row[i + hs];
      row[i] = x0 + x1;
      row[i + hs] = x0 - x1;
    }
    __syncthreads();
  }
  // PROD keys: s^_j = scale sqrt(pi/2) / (m sqrt(d)) * (S q'')_j
  if (kprod) {
    const float kap = a.scale * kSqrtHalfPi / (static_cast<float>(mk) * sqrtf(static_cast<float>(D)));
    for (int idx = tid; idx < GC * mk; idx += kThreads) {
      const int g = idx / mk, j = idx - g * mk;
      const float *srow = a.k.S + static_cast<size_t>(j) * D;
      float acc = 0.f;
      for (int i = 0; i < D; ++i) acc = fmaf(__ldg(srow + i), qt[g * D + i], acc);
      qsk[idx] = kap * acc;
    }
    __syncthreads();
  }
  const float qscale = a.scale / static_cast<float>(D);
  for (int idx = tid; idx < GC * D; idx += kThreads) qt[idx] *= qscale;
  __syncthreads();

  float m_run[GC], l_run[GC], u[2][GC], w[2][GC];
#pragma unroll
  for (int g = 0; g < GC; ++g) {
    m_run[g] = -INFINITY;
    l_run[g] = 0.f;
    u[0][g] = u[1][g] = w[0][g] = w[1][g] = 0.f;
  }

  for (int t0 = t_begin; t0 < t_end; t0 += kTile) {
    const int n = min(kTile, t_end - t0);
    const size_t rec0 = bh * a.T_cap + t0;
    stage_rows(kc, kstr, a.k.codes + rec0 * a.k.code_bytes, a.k.code_bytes, n);
    stage_rows(vc, vstr, a.v.codes + rec0 * a.v.code_bytes, a.v.code_bytes, n);
    if (kprod) stage_rows(ks, ksstr, a.k.signs + rec0 * a.k.sign_bytes, a.k.sign_bytes, n);
    if (vprod) stage_rows(vs, vsstr, a.v.signs + rec0 * a.v.sign_bytes, a.v.sign_bytes, n);
    if (tid < n) {
      kn[tid] = f16_bits_to_f32(a.k.norm[rec0 + tid]);
      vn[tid] = f16_bits_to_f32(a.v.norm[rec0 + tid]);
      krn[tid] = kprod ? f16_bits_to_f32(a.k.rnorm[rec0 + tid]) : 0.f;
      vrn[tid] = vprod ? f16_bits_to_f32(a.v.rnorm[rec0 + tid]) : 0.f;
    }
    __syncthreads();

    // ---- scores: one thread per token, all of this CTA's query heads
    float s[GC];
    if (tid < n) {
      float acc[GC];
#pragma unroll
      for (int g = 0; g < GC; ++g) acc[g] = 0.f;
      if (kw > 0) {
        const uint8_t *row = kc + tid * kstr;
        for (int i = 0; i < D; ++i) {
          const float cv = lutk[get_code(row, i, kw)];
#pragma unroll
          for (int g = 0; g < GC; ++g) acc[g] = fmaf(qt[g * D + i], cv, acc[g]);
        }
      }
      if (kprod) {
        const uint8_t *srow = ks + tid * ksstr;
        float sa[GC];
#pragma unroll
        for (int g = 0; g < GC; ++g) sa[g] = 0.f;
        for (int j = 0; j < mk; ++j) {
          const bool neg = (srow[j >> 3] >> (j & 7)) & 1;
#pragma unroll
          for (int g = 0; g < GC; ++g) sa[g] += neg ? -qsk[g * mk + j] : qsk[g * mk + j];
        }
#pragma unroll
        for (int g = 0; g < GC; ++g) acc[g] = fmaf(krn[tid], sa[g], acc[g]);
      }
#pragma unroll
      for (int g = 0; g < GC; ++g) s[g] = kn[tid] * acc[g];
    } else {
#pragma unroll
      for (int g = 0; g < GC; ++g) s[g] = -INFINITY;
    }

    // ---- online softmax: tile max across the CTA, rescale, p_t
#pragma unroll
    for (int g = 0; g < GC; ++g) {
      const float mx = warp_max(s[g]);
      if (lane == 0) red[g * 8 + warp] = mx;
    }
    __syncthreads();
    float alpha[GC];
#pragma unroll
    for (int g = 0; g < GC; ++g) {
      const float mt = fmaxf(fmaxf(red[g * 8], red[g * 8 + 1]), fmaxf(red[g * 8 + 2], red[g * 8 + 3]));
      const float mn = fmaxf(m_run[g], mt);
      alpha[g] = __expf(m_run[g] - mn);
      m_run[g] = mn;
      const float p = __expf(s[g] - mn);
      l_run[g] = fmaf(l_run[g], alpha[g], p);
      const float nv = tid < n ? vn[tid] : 0.f;
      pw[g * kTile + tid] = p * nv;
      if (vprod) pg[g * kTile + tid] = p * nv * (tid < n ? vrn[tid] : 0.f);
    }
    __syncthreads();

    // ---- values, rotated domain: one thread per coordinate (and per QJL row)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int i = tid + r * kThreads;
      if (i < D && vw > 0) {
#pragma unroll
        for (int g = 0; g < GC; ++g) u[r][g] *= alpha[g];
        for (int t = 0; t < n; ++t) {
          const float cv = lutv[get_code(vc + t * vstr, i, vw)];
#pragma unroll
          for (int g = 0; g < GC; ++g) u[r][g] = fmaf(pw[g * kTile + t], cv, u[r][g]);
        }
      }
      if (vprod && i < mv) {
#pragma unroll
        for (int g = 0; g < GC; ++g) w[r][g] *= alpha[g];
        for (int t = 0; t < n; ++t) {
          const bool neg = (vs[t * vsstr + (i >> 3)] >> (i & 7)) & 1;
#pragma unroll
          for (int g = 0; g < GC; ++g) w[r][g] += neg ? -pg[g * kTile + t] : pg[g * kTile + t];
        }
      }
    }
    __syncthreads();
  }

  // ---- partial record per (b, q-head, split): m, l, u'[D], w[mv]
#pragma unroll
  for (int g = 0; g < GC; ++g) {
    const float sl = warp_sum(l_run[g]);
    if (lane == 0) red[g * 8 + 4 + warp] = sl;
  }
  __syncthreads();
  for (int g = 0; g < gcount; ++g) {
    const int hq = h * G + g0 + g;
    float *dst = a.ws + ((static_cast<size_t>(b) * a.Hq + hq) * a.plan.splits + split) * a.plan.ws_stride;
    if (tid == 0) {
      dst[0] = m_run[g];
      dst[1] = red[g * 8 + 4] + red[g * 8 + 5] + red[g * 8 + 6] + red[g * 8 + 7];
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int i = tid + r * kThreads;
      if (i < D) dst[2 + i] = u[r][g];
      if (vprod && i < mv) dst[2 + D + i] = w[r][g];
    }
  }
}

// Merge the split partials of one (b, q-head): global max M, weights e_s = exp(m_s - M),
// L = sum e_s l_s, U = sum e_s u_s (+ W = sum e_s w_s). Compressed cache: add the QJL value
// term sqrt(d) sqrt(pi/2)/m S^T W, apply the inverse rotation D H / d once and divide by L.
template <int D>
__global__ void __launch_bounds__(kThreads) combine_kernel(const float *ws, int splits, int stride,
                                                           int Hq, float *out, int rotate,
                                                           uint64_t seed, const float *Sv, int mv) {
  __shared__ float e[kMaxSplits];
  __shared__ float o[D];
  __shared__ float wsum[kMaxM];
  __shared__ float sL;
  const int tid = threadIdx.x;
  const int hq = blockIdx.x, b = blockIdx.y;
  const float *base = ws + (static_cast<size_t>(b) * Hq + hq) * splits * stride;
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, base[static_cast<size_t>(s) * stride]);
  for (int s = tid; s < splits; s += kThreads) e[s] = __expf(base[static_cast<size_t>(s) * stride] - M);
  __syncthreads();
  if (tid == 0) {
    float l = 0.f;
    for (int s = 0; s < splits; ++s) l = fmaf(e[s], base[static_cast<size_t>(s) * stride + 1], l);
    sL = l;
  }
  for (int i = tid; i < D; i += kThreads) {
    float acc = 0.f;
    for (int s = 0; s < splits; ++s) acc = fmaf(e[s], base[static_cast<size_t>(s) * stride + 2 + i], acc);
    o[i] = acc;
  }
  for (int j = tid; j < mv; j += kThreads) {
    float acc = 0.f;
    for (int s = 0; s < splits; ++s)
      acc = fmaf(e[s], base[static_cast<size_t>(s) * stride + 2 + D + j], acc);
    wsum[j] = acc;
  }
  __syncthreads();
  if (mv > 0) {
    const float cw = sqrtf(static_cast<float>(D)) * kSqrtHalfPi / static_cast<float>(mv);
    for (int i = tid; i < D; i += kThreads) {
      float acc = 0.f;
      for (int j = 0; j < mv; ++j) acc = fmaf(__ldg(Sv + static_cast<size_t>(j) * D + i), wsum[j], acc);
      o[i] = fmaf(cw, acc, o[i]);
    }
    __syncthreads();
  }
  float *dst = out + (static_cast<size_t>(b) * Hq + hq) * D;
  if (rotate) {
    for (int hs = 1; hs < D; hs <<= 1) {
      for (int k = tid; k < D / 2; k += kThreads) {
        const int i = (k / hs) * 2 * hs + (k % hs);
        const float x0 = o[i], x1 = o[i + hs];
        o[i] = x0 + x1;
        o[i + hs] = x0 - x1;
      }
      __syncthreads();
    }
    const float inv = 1.0f / (static_cast<float>(D) * sL);
    for (int i = tid; i < D; i += kThreads) {
      const float v = o[i] * inv;
      dst[i] = sign_is_neg(seed, i) ? -v : v;
    }
  } else {
    const float inv = 1.0f / sL;
    for (int i = tid; i < D; i += kThreads) dst[i] = o[i] * inv;
  }
}

// ------------------------------------------------------------------ bf16 comparator
template <int D, int GC>
__global__ void __launch_bounds__(kThreads) decode_bf16_kernel(const DecodeBf16Args a) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int ROW = D * 2 + 16; // staged bf16 row stride (bytes): 16-byte aligned, bank-skewed
  float *q = reinterpret_cast<float *>(smem);
  uint8_t *kt = smem + GC * D * 4;
  uint8_t *vt = kt + kTile * ROW;
  float *pw = reinterpret_cast<float *>(vt + kTile * ROW);
  float *red = pw + GC * kTile;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = a.Hq / a.Hkv;
  const int ngrp = (G + GC - 1) / GC;
  const int h = blockIdx.y / ngrp, grp = blockIdx.y - h * ngrp;
  const int g0 = grp * GC;
  const int gcount = min(GC, G - g0);
  const int b = blockIdx.z, split = blockIdx.x;
  const int t_begin = split * a.plan.chunk;
  const int t_end = min(a.T_len, t_begin + a.plan.chunk);
  const size_t bh = static_cast<size_t>(b) * a.Hkv + h;

  for (int idx = tid; idx < GC * D; idx += kThreads) {
    const int g = idx / D, i = idx - g * D;
    q[idx] = g < gcount ? a.scale * load_scalar(a.q, TQ_BF16, (static_cast<size_t>(b) * a.Hq + h * G + g0 + g) * D + i)
                        : 0.f;
  }
  float m_run[GC], l_run[GC], u[2][GC];
#pragma unroll
  for (int g = 0; g < GC; ++g) {
    m_run[g] = -INFINITY;
    l_run[g] = 0.f;
    u[0][g] = u[1][g] = 0.f;
  }
  __syncthreads();
  for (int t0 = t_begin; t0 < t_end; t0 += kTile) {
    const int n = min(kTile, t_end - t0);
    const uint8_t *ksrc = static_cast<const uint8_t *>(a.K) + (bh * a.T_cap + t0) * D * 2;
    const uint8_t *vsrc = static_cast<const uint8_t *>(a.V) + (bh * a.T_cap + t0) * D * 2;
    constexpr int PER = D * 2 / 16;
    for (int idx = tid; idx < n * PER; idx += kThreads) {
      const int r = idx / PER, c = idx - r * PER;
      *reinterpret_cast<uint4 *>(kt + r * ROW + c * 16) =
          __ldg(reinterpret_cast<const uint4 *>(ksrc + static_cast<size_t>(r) * D * 2) + c);
      *reinterpret_cast<uint4 *>(vt + r * ROW + c * 16) =
          __ldg(reinterpret_cast<const uint4 *>(vsrc + static_cast<size_t>(r) * D * 2) + c);
    }
    __syncthreads();
    float s[GC];
    if (tid < n) {
      float acc[GC];
#pragma unroll
      for (int g = 0; g < GC; ++g) acc[g] = 0.f;
      const uint4 *row = reinterpret_cast<const uint4 *>(kt + tid * ROW);
      for (int c = 0; c < PER; ++c) {
        const uint4 v = row[c];
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float k0 = bf16_lo(wv[e]), k1 = bf16_hi(wv[e]);
#pragma unroll
          for (int g = 0; g < GC; ++g) {
            acc[g] = fmaf(q[g * D + c * 8 + 2 * e], k0, acc[g]);
            acc[g] = fmaf(q[g * D + c * 8 + 2 * e + 1], k1, acc[g]);
          }
        }
      }
#pragma unroll
      for (int g = 0; g < GC; ++g) s[g] = acc[g];
    } else {
#pragma unroll
      for (int g = 0; g < GC; ++g) s[g] = -INFINITY;
    }
#pragma unroll
    for (int g = 0; g < GC; ++g) {
      const float mx = warp_max(s[g]);
      if (lane == 0) red[g * 8 + warp] = mx;
    }
    __syncthreads();
    float alpha[GC];
#pragma unroll
    for (int g = 0; g < GC; ++g) {
      const float mt = fmaxf(fmaxf(red[g * 8], red[g * 8 + 1]), fmaxf(red[g * 8 + 2], red[g * 8 + 3]));
      const float mn = fmaxf(m_run[g], mt);
      alpha[g] = __expf(m_run[g] - mn);
      m_run[g] = mn;
      const float p = __expf(s[g] - mn);
      l_run[g] = fmaf(l_run[g], alpha[g], p);
      pw[g * kTile + tid] = p;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int i = tid + r * kThreads;
      if (i < D) {
#pragma unroll
        for (int g = 0; g < GC; ++g) u[r][g] *= alpha[g];
        for (int t = 0; t < n; ++t) {
          const float vv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(vt + t * ROW + 2 * i));
#pragma unroll
          for (int g = 0; g < GC; ++g) u[r][g] = fmaf(pw[g * kTile + t], vv, u[r][g]);
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int g = 0; g < GC; ++g) {
    const float sl = warp_sum(l_run[g]);
    if (lane == 0) red[g * 8 + 4 + warp] = sl;
  }
  __syncthreads();
  for (int g = 0; g < gcount; ++g) {
    const int hq = h * G + g0 + g;
    float *dst = a.ws + ((static_cast<size_t>(b) * a.Hq + hq) * a.plan.splits + split) * a.plan.ws_stride;
    if (tid == 0) {
      dst[0] = m_run[g];
      dst[1] = red[g * 8 + 4] + red[g * 8 + 5] + red[g * 8 + 6] + red[g * 8 + 7];
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int i = tid + r * kThreads;
      if (i < D) dst[2 + i] = u[r][g];
    }
  }
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int D, int GC>
cudaError_t run_decode(const DecodeArgs &a, cudaStream_t s) {
  const SmemLayout L = make_layout(D, GC, a.k, a.v);
  const int G = a.Hq / a.Hkv;
  const int ngrp = (G + GC - 1) / GC;
  dim3 grid(a.plan.splits, a.Hkv * ngrp, a.B);
  cudaError_t e = set_smem(decode_split_kernel<D, GC>, L.total);
  if (e != cudaSuccess) return e;
  decode_split_kernel<D, GC><<<grid, kThreads, L.total, s>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  combine_kernel<D><<<dim3(a.Hq, a.B), kThreads, 0, s>>>(a.ws, a.plan.splits, a.plan.ws_stride, a.Hq,
                                                        a.out, 1, a.seed, a.v.S, a.v.m);
  return cudaGetLastError();
}

template <int D, int GC>
cudaError_t run_decode_bf16(const DecodeBf16Args &a, cudaStream_t s) {
  const int bytes = GC * D * 4 + 2 * kTile * (D * 2 + 16) + GC * kTile * 4 + GC * 8 * 4;
  const int G = a.Hq / a.Hkv;
  const int ngrp = (G + GC - 1) / GC;
  dim3 grid(a.plan.splits, a.Hkv * ngrp, a.B);
  cudaError_t e = set_smem(decode_bf16_kernel<D, GC>, bytes);
  if (e != cudaSuccess) return e;
  decode_bf16_kernel<D, GC><<<grid, kThreads, bytes, s>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  combine_kernel<D><<<dim3(a.Hq, a.B), kThreads, 0, s>>>(a.ws, a.plan.splits, a.plan.ws_stride, a.Hq,
                                                        a.out, 0, 0, nullptr, 0);
  return cudaGetLastError();
}

#define TQ_DISPATCH_GC(RUN, D)                                                 \
  switch (a.plan.gc) {                                                         \
  case 1: return RUN<D, 1>(a, s);                                              \
  case 2: return RUN<D, 2>(a, s);                                              \
  case 4: return RUN<D, 4>(a, s);                                              \
  case 8: return RUN<D, 8>(a, s);                                              \
  case 16: return RUN<D, 16>(a, s);                                            \
  }                                                                            \
  return cudaErrorInvalidValue;

#define TQ_DISPATCH_DEC(RUN)                                                   \
  switch (a.d) {                                                               \
  case 16: TQ_DISPATCH_GC(RUN, 16)                                             \
  case 32: TQ_DISPATCH_GC(RUN, 32)                                             \
  case 64: TQ_DISPATCH_GC(RUN, 64)                                             \
  case 128: TQ_DISPATCH_GC(RUN, 128)                                           \
  case 256: TQ_DISPATCH_GC(RUN, 256)                                           \
  }                                                                            \
  return cudaErrorInvalidValue;

} // namespace

DecodePlan plan_decode(int B, int Hq, int Hkv, int d, int T_len, int v_m, int sm_count, bool bf16,
                       int fast) {
  DecodePlan p{};
  if (bf16 && bf16_decode_supported(d, Hq / Hkv)) {
    plan_bf16_mma(B, Hq, Hkv, T_len, sm_count, &p);
    return p;
  }
  if (fast == kProdFast && !bf16) {
    plan_prod(B, Hq, Hkv, T_len, sm_count, &p);
    return p;
  }
  if (fast && !bf16) {
    plan_fast(B, Hq, Hkv, T_len, sm_count, fast >> 4, fast & 15, &p);
    return p;
  }
  p.path = 0;
  p.tile = kTile;
  const int G = Hq / Hkv;
  int gc = 1;
  while (gc < G && gc < 16) gc <<= 1;
  p.gc = gc;
  const int ngrp = (G + gc - 1) / gc;
  const long long ctas = static_cast<long long>(B) * Hkv * ngrp;
  const long long target = 4ll * sm_count;
  const int max_splits = std::min((T_len + kTile - 1) / kTile, kMaxSplits);
  long long want = (target + ctas - 1) / ctas;
  int splits = static_cast<int>(std::max(1ll, std::min<long long>(want, max_splits)));
  int chunk = round_up((T_len + splits - 1) / splits, kTile);
  splits = (T_len + chunk - 1) / chunk;
  p.splits = splits;
  p.chunk = chunk;
  p.ws_stride = round_up(2 + d + v_m, 4);
  p.ws_bytes = static_cast<size_t>(B) * Hq * splits * p.ws_stride * sizeof(float);
  return p;
}

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s) {
  if (a.plan.path == 1) return launch_fast_decode(a, s);
  if (a.plan.path == 2) return launch_prod_decode(a, s);
  TQ_DISPATCH_DEC(run_decode)
}

cudaError_t launch_decode_bf16(const DecodeBf16Args &a, cudaStream_t s) {
  if (a.plan.path == 3) return launch_bf16_mma(a, s);
  TQ_DISPATCH_DEC(run_decode_bf16)
}

} // namespace tq

// ------------------------------------------------------------------ fixed scratch
// Backing store for tq_decode_attention_noalloc: the split-K partials of one call live in
// this file-scope device array instead of a caller workspace. Every GPU that loads the
// library holds it for the life of the process. Host code must not pass the symbol itself
// to a kernel (in host code it names a host-side stand-in); fixed_scratch() fetches the real
// device address once per device and caches it.
namespace tq {
namespace {
constexpr size_t kFixedScratchBytes = size_t(8) << 20; // 8 MiB
constexpr int kMaxDevices = 64;
} // namespace

static __device__ __align__(256) float g_fixed_scratch[kFixedScratchBytes / sizeof(float)];

cudaError_t fixed_scratch(float **ptr, size_t *bytes) {
  static std::mutex mu;
  static void *addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_fixed_scratch); // with `dev` current
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *ptr = static_cast<float *>(addr[dev]);
  *bytes = kFixedScratchBytes;
  return cudaSuccess;
}

} // namespace tq
