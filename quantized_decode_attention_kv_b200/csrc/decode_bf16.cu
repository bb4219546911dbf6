// Tensor-core decode attention over an uncompressed bf16 K/V cache (head_dim 128, 1..8 query
// heads per KV head): the comparator of the compressed kernels, built the same way (split-K
// over 16-token tiles, per-warp online softmax, CTA merge, one combine), and the kernel for
// layers kept in bf16 ("Where This Fits in the Inference Stack", Decode Throughput vs. TTFT).
//
//   scores  S[16 tokens x 8 heads] = K[16 x 128] . q[128 x 8]  (bf16 x bf16 -> fp32: exact
//           products, so no operand splitting). A lane loads coordinates [32 c, 32 c + 32) of
//           its two tokens with 16-byte loads; with the contraction index permuted the same
//           way for q, those registers already are the A fragments.
//   values  O^T[128 x 8] += V^T[128 x 16 tokens] . P[16 tokens x 8]; one PRMT interleaves two
//           tokens' values of one coordinate into an A register; P is split into a bf16 part
//           and a bf16 residual (two MMAs), as the MMA takes one operand type.
//
// The registers of a tile are pipelined by phase: the next tile's keys load while this tile's
// softmax and values run, the next tile's values while the next scores run; an L2 prefetch
// runs a few tiles further ahead.
#include "mma_ops.cuh"

#include <algorithm>

namespace tq {
namespace {
using namespace mma_ops;

constexpr int kBW = 4; // warps per CTA
constexpr int kBThreads = kBW * 32;
constexpr int kBD = 128;
constexpr int kBStep = kBW * 16; // tokens a warp advances per step
constexpr int kBRow = kBD * 2;   // bytes per token row
constexpr float kBLog2e = 1.4426950408889634f;
#ifndef TQ_BF16_PREFETCH
#define TQ_BF16_PREFETCH 2
#endif
constexpr int kBPrefetch = TQ_BF16_PREFETCH; // L2 prefetch distance in warp steps

__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// bf16 pair (a, b) and the bf16 pair of the rounding residuals
__device__ __forceinline__ void split_bf16(float a, float b, uint32_t &hi, uint32_t &lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  const float2 f = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(a - f.x, b - f.y);
  hi = *reinterpret_cast<const uint32_t *>(&h);
  lo = *reinterpret_cast<const uint32_t *>(&l);
}

__device__ __forceinline__ void ld16(uint32_t *dst, const uint8_t *p) {
  const uint4 v = __ldcs(reinterpret_cast<const uint4 *>(p));
  dst[0] = v.x;
  dst[1] = v.y;
  dst[2] = v.z;
  dst[3] = v.w;
}

struct Bf16Args {
  const uint8_t *q, *K, *V;
  float *part; // partial records [cta][slot][G][stride]
  int Hq, Hkv, G, T_len, T_cap;
  int tiles_per_bh, tiles_per_cta, slots, stride;
  long long total_tiles;
  float qk_scale; // softmax scale * log2(e)
};

__global__ void __launch_bounds__(kBThreads, 3) decode_bf16_mma_kernel(const Bf16Args a) {
  __shared__ float mst[kBW * 8];
  __shared__ float gmx[8];
  __shared__ float lsum[8];
  __shared__ float obuf[8 * kBD];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = lane >> 2, c = lane & 3;
  pdl_wait(); // q and the cache may come from earlier kernels
  pdl_trigger();

  const long long range0 = static_cast<long long>(blockIdx.x) * a.tiles_per_cta;
  const long long range1 = min(a.total_tiles, range0 + a.tiles_per_cta);
  int slot = 0;
  for (long long seg = range0; seg < range1; ++slot) {
    const long long bh = seg / a.tiles_per_bh;
    const long long seg_end = min(range1, (bh + 1) * a.tiles_per_bh);
    const int tile0 = static_cast<int>(seg - bh * a.tiles_per_bh);
    const int ntiles = static_cast<int>(seg_end - seg);
    seg = seg_end;
    const int b = static_cast<int>(bh / a.Hkv), h = static_cast<int>(bh % a.Hkv);

    // B operand of the scores: column r = head r, coordinates [32 c, 32 c + 32)
    uint32_t qb[16];
    if (r < a.G) {
      const uint8_t *qs = a.q + ((static_cast<size_t>(b) * a.Hq + h * a.G + r) * kBD + 32 * c) * 2;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(qs) + k);
        qb[4 * k] = v.x;
        qb[4 * k + 1] = v.y;
        qb[4 * k + 2] = v.z;
        qb[4 * k + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int k = 0; k < 16; ++k) qb[k] = 0u;
    }

    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f}; // heads 2c, 2c + 1
    float o[8][4];
#pragma unroll
    for (int m = 0; m < 8; ++m) o[m][0] = o[m][1] = o[m][2] = o[m][3] = 0.f;

    const size_t rec0 = static_cast<size_t>(bh) * a.T_cap;
    const int tlast = a.T_len - 1;
    const uint8_t *Kb = a.K + rec0 * kBRow + 64 * c; // lane's 64-byte key slice
    const uint8_t *Vb = a.V + rec0 * kBRow + 32 * r; // lane's 32-byte value run
    // L2 prefetch: lane l takes line l of a tile's keys and line l of its values
    int tpf = (tile0 + warp) * 16 + kBPrefetch * kBStep;

    uint32_t kr[2][16]; // keys of tokens r, r + 8 (the A fragments of the score MMA)
    uint32_t vr[4][8];  // values of tokens 2c, 2c+1, 2c+8, 2c+9
    auto load_k = [&](int t0) {
      const int t_a = min(t0 + r, tlast), t_b = min(t0 + r + 8, tlast);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        ld16(&kr[0][4 * k], Kb + static_cast<size_t>(t_a) * kBRow + 16 * k);
        ld16(&kr[1][4 * k], Kb + static_cast<size_t>(t_b) * kBRow + 16 * k);
      }
    };
    auto load_v = [&](int t0) {
      const int tv = t0 + 2 * c;
      const int ts[4] = {min(tv, tlast), min(tv + 1, tlast), min(tv + 8, tlast), min(tv + 9, tlast)};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        ld16(&vr[e][0], Vb + static_cast<size_t>(ts[e]) * kBRow);
        ld16(&vr[e][4], Vb + static_cast<size_t>(ts[e]) * kBRow + 16);
      }
    };
    auto prefetch = [&]() {
      if (tpf + 16 <= a.T_len && tpf < (tile0 + ntiles) * 16) {
        const size_t off = (rec0 + tpf) * kBRow + 128 * lane;
        asm volatile("prefetch.global.L2 [%0];" ::"l"(a.K + off));
        asm volatile("prefetch.global.L2 [%0];" ::"l"(a.V + off));
      }
      tpf += kBStep;
    };

    int jt = warp;
    if (jt < ntiles) {
      load_k((tile0 + jt) * 16);
      load_v((tile0 + jt) * 16);
    }
    while (jt < ntiles) {
      const int t0 = (tile0 + jt) * 16;
      const int jn = jt + kBW;
      prefetch();
      // ---- scores (two accumulator chains)
      float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int s = 0; s < 8; s += 2) {
        mma_bf16(sa, kr[0][2 * s], kr[1][2 * s], kr[0][2 * s + 1], kr[1][2 * s + 1], qb[2 * s], qb[2 * s + 1]);
        mma_bf16(sb, kr[0][2 * s + 2], kr[1][2 * s + 2], kr[0][2 * s + 3], kr[1][2 * s + 3],
                 qb[2 * s + 2], qb[2 * s + 3]);
      }
      if (jn < ntiles) load_k((tile0 + jn) * 16);

      // ---- online softmax (log2 domain); lane (r, c) owns heads 2c, 2c + 1 at tokens r, r + 8
      const bool ok0 = t0 + r < a.T_len, ok1 = t0 + r + 8 < a.T_len;
      uint32_t phi[2], plo[2];
      float alpha[2];
      bool moved = false;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float s0 = ok0 ? (sa[e] + sb[e]) * a.qk_scale : -INFINITY;
        const float s1 = ok1 ? (sa[2 + e] + sb[2 + e]) * a.qk_scale : -INFINITY;
        float mx = fmaxf(s0, s1);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float mn = fmaxf(m_run[e], mx);
        alpha[e] = softmax_exp2(m_run[e] - mn);
        moved |= mn != m_run[e];
        m_run[e] = mn;
        const float p0 = softmax_exp2(s0 - mn), p1 = softmax_exp2(s1 - mn);
        l_run[e] = fmaf(l_run[e], alpha[e], p0 + p1);
        split_bf16(p0, p1, phi[e], plo[e]); // (token r, token r + 8)
      }
      if (moved) {
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          o[m][0] *= alpha[0];
          o[m][1] *= alpha[1];
          o[m][2] *= alpha[0];
          o[m][3] *= alpha[1];
        }
      }
      // ---- P operand (column r = head r): tokens 2c, 2c+1 (b0) and 2c+8, 2c+9 (b1) come from
      //      lanes (2c, r/2) and (2c + 1, r/2), which hold head r as their head r & 1
      const int srca = 8 * c + (r >> 1), srcb = srca + 4;
      const bool odd = r & 1;
      const uint32_t ha0 = __shfl_sync(0xffffffffu, phi[0], srca), ha1 = __shfl_sync(0xffffffffu, phi[1], srca);
      const uint32_t hb0 = __shfl_sync(0xffffffffu, phi[0], srcb), hb1 = __shfl_sync(0xffffffffu, phi[1], srcb);
      const uint32_t la0 = __shfl_sync(0xffffffffu, plo[0], srca), la1 = __shfl_sync(0xffffffffu, plo[1], srca);
      const uint32_t lb0 = __shfl_sync(0xffffffffu, plo[0], srcb), lb1 = __shfl_sync(0xffffffffu, plo[1], srcb);
      uint32_t xa = odd ? ha1 : ha0, xb = odd ? hb1 : hb0, ya = odd ? la1 : la0, yb = odd ? lb1 : lb0;
      if (r >= a.G) xa = xb = ya = yb = 0u;
      const uint32_t ph0 = prmt(xa, xb, 0x5410u), ph1 = prmt(xa, xb, 0x7632u);
      const uint32_t pl0 = prmt(ya, yb, 0x5410u), pl1 = prmt(ya, yb, 0x7632u);

      // ---- values: m-tile m = coordinates 16 r + 2m (rows r) and + 1 (rows r + 8)
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const uint32_t a0 = prmt(vr[0][m], vr[1][m], 0x5410u), a1 = prmt(vr[0][m], vr[1][m], 0x7632u);
        const uint32_t a2 = prmt(vr[2][m], vr[3][m], 0x5410u), a3 = prmt(vr[2][m], vr[3][m], 0x7632u);
        mma_bf16(o[m], a0, a1, a2, a3, ph0, ph1);
        mma_bf16(o[m], a0, a1, a2, a3, pl0, pl1);
      }
      if (jn < ntiles) load_v((tile0 + jn) * 16);
      jt = jn;
    }

    // ---- merge the warps: common max per head, rescale, accumulate in shared memory
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float l = l_run[e];
      l += __shfl_xor_sync(0xffffffffu, l, 4);
      l += __shfl_xor_sync(0xffffffffu, l, 8);
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      l_run[e] = l;
      if (r == 0) mst[warp * 8 + 2 * c + e] = m_run[e];
    }
    for (int idx = tid; idx < a.G * kBD; idx += kBThreads) obuf[idx] = 0.f;
    if (tid < 8) lsum[tid] = 0.f;
    __syncthreads();
    if (tid < 8) {
      float M = -INFINITY;
      for (int w = 0; w < kBW; ++w) M = fmaxf(M, mst[w * 8 + tid]);
      gmx[tid] = M;
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int g = 2 * c + e;
      if (g < a.G) {
        const float f = exp2f(m_run[e] - gmx[g]);
        if (r == 0) atomicAdd(&lsum[g], l_run[e] * f);
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const int i0 = 16 * r + 2 * m;
          atomicAdd(&obuf[g * kBD + i0], o[m][e] * f);
          atomicAdd(&obuf[g * kBD + i0 + 1], o[m][2 + e] * f);
        }
      }
    }
    __syncthreads();
    float *dst = a.part + (static_cast<size_t>(blockIdx.x) * a.slots + slot) * a.G * a.stride;
    for (int idx = tid; idx < a.G * kBD; idx += kBThreads) {
      const int g = idx / kBD, i = idx - g * kBD;
      dst[static_cast<size_t>(g) * a.stride + 2 + i] = obuf[idx];
    }
    if (tid < a.G) {
      dst[static_cast<size_t>(tid) * a.stride] = gmx[tid];
      dst[static_cast<size_t>(tid) * a.stride + 1] = lsum[tid];
    }
    __syncthreads();
  }
}

// Merge the partial records of one (b, q-head) and divide by the softmax sum (the bf16 path
// works in the original domain: no rotation). One warp per (b, q-head), 4 coordinates per lane.
__global__ void __launch_bounds__(128) combine_bf16_kernel(const float *part, int B, int Hkv, int G,
                                                           int tiles_per_bh, int tiles_per_cta,
                                                           int slots, int stride, float *out) {
  const int lane = threadIdx.x & 31;
  const int Hq = Hkv * G;
  const int gw = blockIdx.x * 4 + (threadIdx.x >> 5);
  pdl_wait(); // the partials come from the decode kernel
  if (gw >= B * Hq) return;
  const int b = gw / Hq, hq = gw - b * Hq;
  const int h = hq / G, g = hq - h * G;
  const long long bh = static_cast<long long>(b) * Hkv + h;
  const long long first = bh * tiles_per_bh, last = first + tiles_per_bh - 1;
  const int cta0 = static_cast<int>(first / tiles_per_cta), cta1 = static_cast<int>(last / tiles_per_cta);
  auto rec = [&](int cta) {
    const long long bh0 = static_cast<long long>(cta) * tiles_per_cta / tiles_per_bh;
    return part + ((static_cast<size_t>(cta) * slots + (bh - bh0)) * G + g) * stride;
  };
  float M = -INFINITY;
  for (int c = cta0 + lane; c <= cta1; c += 32) M = fmaxf(M, rec(c)[0]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float L = 0.f;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
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
      const float2 *src = reinterpret_cast<const float2 *>(rec(c0 + k) + 2 + 4 * lane);
      const float2 u0 = src[0], u1 = src[1];
      acc[0] = fmaf(ek, u0.x, acc[0]);
      acc[1] = fmaf(ek, u0.y, acc[1]);
      acc[2] = fmaf(ek, u1.x, acc[2]);
      acc[3] = fmaf(ek, u1.y, acc[3]);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
  const float inv = 1.0f / L;
  reinterpret_cast<float4 *>(out + (static_cast<size_t>(b) * Hq + hq) * kBD)[lane] =
      make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
}

} // namespace

bool bf16_decode_supported(int d, int G) { return d == kBD && G >= 1 && G <= 8; }

void plan_bf16_mma(int B, int Hq, int Hkv, int T_len, int sm_count, DecodePlan *p) {
  const int G = Hq / Hkv;
  p->path = 3;
  p->tile = 16;
  p->gc = G;
  p->ws_stride = 2 + kBD + 2; // 132 floats
  p->tiles_per_bh = (T_len + 15) / 16;
  const long long total = static_cast<long long>(B) * Hkv * p->tiles_per_bh;
  long long ctas = static_cast<long long>(sm_count) * 3;
  ctas = std::min<long long>(ctas, (total + 7) / 8); // at least 8 tiles per CTA
  ctas = std::max<long long>(ctas, 1);
  p->tiles_per_cta = static_cast<int>((total + ctas - 1) / ctas);
  p->ctas = static_cast<int>((total + p->tiles_per_cta - 1) / p->tiles_per_cta);
  p->slots = (p->tiles_per_cta + p->tiles_per_bh - 1) / p->tiles_per_bh + 1;
  p->splits = 0;
  p->chunk = 0;
  p->part_bytes = static_cast<size_t>(p->ctas) * p->slots * G * p->ws_stride * sizeof(float);
  p->part_bytes = (p->part_bytes + 255) / 256 * 256;
  p->ws_bytes = p->part_bytes;
}

cudaError_t launch_bf16_mma(const DecodeBf16Args &a, cudaStream_t s) {
  const DecodePlan &p = a.plan;
  Bf16Args f;
  f.q = static_cast<const uint8_t *>(a.q);
  f.K = static_cast<const uint8_t *>(a.K);
  f.V = static_cast<const uint8_t *>(a.V);
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
  f.qk_scale = a.scale * kBLog2e;
  cudaError_t e = launch_pdl(decode_bf16_mma_kernel, dim3(p.ctas), dim3(kBThreads), 0, s, f);
  if (e != cudaSuccess) return e;
  return launch_pdl(combine_bf16_kernel, dim3((a.B * a.Hq + 3) / 4), dim3(128), 0, s,
                    static_cast<const float *>(a.ws), a.B, a.Hkv, f.G, p.tiles_per_bh,
                    p.tiles_per_cta, p.slots, p.ws_stride, a.out);
}

} // namespace tq
