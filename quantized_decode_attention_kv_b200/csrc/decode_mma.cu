// Tensor-core decode attention over the compressed cache (head_dim 128, TurboQuant_mse with
// 3- or 4-bit keys and 2-, 3- or 4-bit values, up to 8 query heads per KV head).
//
// "Where This Fits in the Inference Stack", TensorRT-LLM section: dequantise in registers
// inside the attention kernel. Here the dequantised codes are written straight into the
// operand registers of warp-level tensor-core MMAs:
//
//   scores  S[16 tokens x 3 per head] = K^[16 x 2*128] . Q[2*128 x 3 per head]
//     (mma.sync m16n8k32, int8 x int8 -> int32). Centroids are 16-bit fixed-point numbers
//     c = 256 c_hi + c_lo, queries 24-bit ones q = 65536 q_hi + 256 q_mid + q_lo, each part an
//     int8. K^ comes from a shared-memory LUT indexed by the codes of two adjacent coordinates
//     (a code byte of 4-bit keys, 6 bits of 3-bit keys) whose 4-byte entry is
//     {hi, hi, lo, lo} of the two centroids, i.e. four consecutive k slots of one A row. Per head three columns take {q_hi, 0}, {q_mid, q_hi} and {q_lo, q_mid} at the
//     {hi, lo} slots, so c.q = 2^24 col0 + 2^16 col1 + 2^8 col2 up to c_lo q_lo (2^-24 of the
//     scale); the rounding of the centroids to 16 bits, at a scale chosen to make it small, is
//     the only other error.
//   values  O^T[128 x heads] += V^T[128 x 16 tokens] . P'^T[16 tokens x heads]
//     2-bit V^: one byte of nibble-interleaved codes (two tokens, two coordinates) indexes a
//     lane-replicated shared table whose 8-byte entry is a pair of operand registers;
//     3/4-bit V^: one table word per token and pair of adjacent coordinates, two PRMTs per
//     pair of operand registers. P' = p * ||v_t|| in fp16.
//
// The contraction order is free along k, so each thread owns a contiguous slice of every key
// record (16 bytes of 4-bit codes, 12 of 3-bit codes) and one or two 32-bit words of every
// value record, and the permutation is undone when the partial accumulators are written.
//
// Work split: the (batch, KV head, 16-token tile) space is flattened and cut into equal
// contiguous ranges, one per persistent CTA (12 warps with 2-bit values or 4-bit keys, else
// 4); within a range each maximal run of one (batch, KV head) is a segment, its tiles dealt
// round-robin to the warps (a paged cache: page-aligned chunks of up to 4 tiles), each warp
// keeping its own online-softmax state (log2 domain); at the end of the segment the warps
// store their rescaled accumulators in their own shared-memory slots, which are summed into
// one partial record per query head.
#include "decode_mse_common.cuh"

#include <algorithm>
#include <vector>
#include <mutex>
#include <type_traits>

namespace tq {
namespace {
using namespace mma_ops;
using namespace mse;

#ifndef TQ_DECODE_PREFETCH
#define TQ_DECODE_PREFETCH 1
#endif
// A warp asks L2 for the tile it will load this many of its own steps later (0: no prefetch):
// loads one step ahead in registers only cover part of the DRAM latency.
constexpr int kPrefetchSteps = TQ_DECODE_PREFETCH;

// Warps per CTA and CTAs per SM. 2-bit values use a 64 KB value table beside the 64 KB key
// table, and 4-bit keys keep the 3/4-bit value table in the unused halves of their 64 KB of
// key rows, so these configurations run one CTA of 12 warps per SM sharing the tables; 3-bit
// keys with 3/4-bit values run three CTAs of 4 warps (12 warps of up to 168 registers per SM
// either way; 16 warps of 128 registers were measured slower).
template <int KB, int VB>
struct Cfg {
  static constexpr bool kOneCta = VB == 2 || KB == 4;
  static constexpr int kWarps = kOneCta ? 12 : 4;
  static constexpr int kCtas = kOneCta ? 1 : 3;
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kStep = kWarps * 16; // tokens a warp advances per step
};

// Per-tile registers of one warp lane for KB-bit keys and VB-bit values (d = 128).
//  keys: the lane's slice [32c, 32c+32) of the coordinates = KB words of each of tokens r, r+8
//  values: the lane's run [16r, 16r+16) of the coordinates of tokens c, c+4, c+8, c+12 (the
//          value MMA's k order, so that each load instruction reads four consecutive records):
//          VB = 2: one word; VB = 3: the two words that hold its 48 bits; VB = 4: two words
template <int KB, int VB>
struct Tile {
  static constexpr int VW = VB == 2 ? 1 : 2;
  uint32_t k[2][KB];
  uint32_t v[4][VW];
  uint16_t kn[2]; // key norms (fp16 bits) of tokens r, r+8
  uint16_t vn[2]; // value norms (fp16 bits) of tokens r, r+8
};

// Shared-memory tables of one configuration. Key rows: one code-pair index (4-bit keys: a
// byte of two codes, 256 rows; 3-bit keys: 6 bits, 64 rows) x 32 lane copies of the 4-byte
// int8 entry {hi, hi, lo, lo}, in a 256-byte row of which the first 128 bytes are used (the
// index lands at bit 8 of the address). Value rows, 2-bit values: one byte holding the codes
// of two adjacent coordinates of two tokens (low nibble the first token) x 32 lane copies of
// the two fp16x2 operand words = 256 bytes; 3/4-bit values: one index (the codes of
// two adjacent coordinates of one token, the first in the low bits) x 32 lane copies of the
// fp16x2 pair of their centroids = 128 bytes (with 4-bit keys: the unused half of key row i).
// The 3-bit key table and the 3/4-bit value tables sit at addresses aligned to their size so
// that an index OR-ed above the lane offset is already the address.
template <int KB, int VB>
struct Lut {
  static constexpr int kRows = KB == 4 ? 256 : 64;
  static constexpr int kBytes = kRows * 256;
  static constexpr int kAlign = KB == 4 ? 16 : kBytes;
  // 4-bit keys with 3/4-bit values: value row i is the second 128 bytes of key row i
  static constexpr bool kVInK = KB == 4 && VB >= 3;
  static constexpr int vRows = VB >= 3 ? 1 << (2 * VB) : 256;
  static constexpr int vBytes = kVInK ? 0 : vRows * (VB >= 3 ? 128 : 256);
  static constexpr int vAlign = VB >= 3 && !kVInK ? vBytes : 16;
  // merge area: per-warp maxima and sums [warps][8] each, merged [8] each, then the per-warp
  // value accumulators [warps][8 m-tiles][32 lanes] float4
  static constexpr int kMergeBytes = (2 * Cfg<KB, VB>::kWarps * 8 + 16) * 4 + Cfg<KB, VB>::kWarps * 256 * 16;
  static constexpr int kSmem = kBytes + kAlign - 16 + vBytes + vAlign - 16 + kMergeBytes;
};

struct FastArgs {
  const uint8_t *kc, *vc;
  const uint16_t *kn, *vn;
  const void *q; // queries [B][Hq][128] of q_dtype, rotated by the kernel itself
  int q_dtype;
  float scale;
  uint64_t seed;
  float *part; // partial records [cta][slot][G][stride]
  int Hq, Hkv, G, T_len, T_cap;
  int tiles_per_bh, tiles_per_cta, slots, stride;
  long long total_tiles;
  float kcent[16];
  float kcsc; // 16-bit fixed-point scale of the key centroids
  float vcent[16];
  uint32_t one;
  int B;
  const int *bt; // paged cache: block table [B][maxp]; record (b, h, t) at page bt[b][t >> pshift]
  int pshift, maxp;
};

// A ragged call's launch parameters: the common ones and the per-sequence lengths (kept out of
// the uniform kernels' parameters, which travel with every launch).
struct FastArgsV {
  FastArgs a;
  VarLen vl;
};
struct NoVarLen {};
__device__ __forceinline__ const FastArgs &base_args(const FastArgs &a) { return a; }
__device__ __forceinline__ const FastArgs &base_args(const FastArgsV &a) { return a.a; }

// MODE 0: dense cache, one T_len; 1: dense cache, per-sequence lengths; 2: paged cache,
// per-sequence lengths.
template <int KB, int VB, int NT, int MODE>
__global__ void __launch_bounds__(Cfg<KB, VB>::kThreads, Cfg<KB, VB>::kCtas)
    decode_mse_kernel(const std::conditional_t<MODE != 0, FastArgsV, FastArgs> args) {
  constexpr bool RAG = MODE != 0, PG = MODE == 2;
  const FastArgs &a = base_args(args);
  using L = Lut<KB, VB>;
  using C = Cfg<KB, VB>;
  constexpr int kWarps = C::kWarps, kThreads = C::kThreads, kStep = C::kStep;
  using TileT = Tile<KB, VB>;
  constexpr int KR = KB * 16, VR = VB * 16; // record bytes
  extern __shared__ __align__(16) uint8_t smem[];
  const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  const uint32_t klut = (sbase + L::kAlign - 1) & ~static_cast<uint32_t>(L::kAlign - 1);
  const uint32_t vlut = (klut + L::kBytes + L::vAlign - 1) & ~static_cast<uint32_t>(L::vAlign - 1);
  uint8_t *const kl_p = smem + (klut - sbase);
  uint8_t *const vl_p = smem + (vlut - sbase);
  float *mst = reinterpret_cast<float *>(vl_p + L::vBytes); // [kWarps][8] running max
  float *lst = mst + kWarps * 8;                            // [kWarps][8] running sum
  float *gmx = lst + kWarps * 8;                            // [8] merged max
  float *lsum = gmx + 8;                                    // [8] merged sum
  float4 *obw = reinterpret_cast<float4 *>(lsum + 8);       // [kWarps][8][32] accumulators

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = lane >> 2, c = lane & 3;

  {
    // key row e (first 128 of its 256 bytes): 32 lane copies of {hi(c0), hi(c1), lo(c0),
    // lo(c1)} for the two codes of index e, the first in the low bits
    uint32_t *kw = reinterpret_cast<uint32_t *>(kl_p);
    for (int idx = tid; idx < L::kRows * 32; idx += kThreads) {
      const int e = idx >> 5, l = idx & 31;
      const float c0 = a.kcent[e & (KB == 4 ? 15 : 7)], c1 = a.kcent[KB == 4 ? e >> 4 : e >> 3];
      const int i0 = __float2int_rn(c0 * a.kcsc), i1 = __float2int_rn(c1 * a.kcsc);
      const int l0 = ((i0 + 128) & 255) - 128, l1 = ((i1 + 128) & 255) - 128;
      const int h0 = (i0 - l0) >> 8, h1 = (i1 - l1) >> 8;
      kw[e * 64 + l] = static_cast<uint32_t>(h0 & 255) | (static_cast<uint32_t>(h1 & 255) << 8) |
                       (static_cast<uint32_t>(l0 & 255) << 16) | (static_cast<uint32_t>(l1 & 255) << 24);
    }
    uint32_t *vw = reinterpret_cast<uint32_t *>(vl_p);
    for (int idx = tid; idx < L::vRows * 32; idx += kThreads) {
      const int e = idx >> 5;
      if constexpr (L::kVInK) {
        kw[e * 64 + 32 + (idx & 31)] = pack_h2(a.vcent[e & ((1 << VB) - 1)], a.vcent[e >> VB]);
      } else if constexpr (VB == 2) {
        // byte e: first token's codes at coordinates j, j+1 in bits 0-1, 2-3, the second
        // token's in bits 4-5, 6-7; words: coordinate j, coordinate j+1 (tokens in halves)
        const int l = idx & 31;
        vw[e * 64 + 2 * l] = pack_h2(a.vcent[e & 3], a.vcent[(e >> 4) & 3]);
        vw[e * 64 + 2 * l + 1] = pack_h2(a.vcent[(e >> 2) & 3], a.vcent[(e >> 6) & 3]);
      } else {
        vw[idx] = pack_h2(a.vcent[e & ((1 << VB) - 1)], a.vcent[e >> VB]);
      }
    }
  }
  const uint32_t lanebase = static_cast<uint32_t>(lane) << 2;
  const uint32_t klane4 = static_cast<uint32_t>(lane) << 2; // lane's 4-byte key entry
  const uint32_t klb = klut | klane4;                          // 3-bit keys: base + lane offset
  const uint32_t vlb = vlut | lanebase;
  [[maybe_unused]] const uint32_t vkb = klut + 128; // value rows inside the key rows
  const uint32_t one = a.one; // 1, opaque to the compiler so the add stays an IMAD
  __syncthreads();
  pdl_wait(); // the prepared queries and the cache are written by earlier kernels
  pdl_trigger();

  // Two copies of the persistent loop: when the 4-bit key table starts at the usual first
  // dynamic shared address (kFixedBase), the table base is an immediate offset of the shared
  // loads and the PRMT that places the code byte above the lane offset is the whole address
  // computation; otherwise an IMAD adds the base.
  auto run = [&](auto fixed_tag) {
    constexpr bool kFixed = decltype(fixed_tag)::value;
    [[maybe_unused]] const uint32_t klane = klane4;
    [[maybe_unused]] const uint32_t vlane8 = static_cast<uint32_t>(lane) << 3; // 2-bit values: 8-byte entry
    const long long range0 = static_cast<long long>(blockIdx.x) * a.tiles_per_cta;
    const long long range1 = min(a.total_tiles, range0 + a.tiles_per_cta);
    int slot = 0;
    [[maybe_unused]] int vb = 0; // ragged calls: the sequence of the current segment
    if constexpr (RAG)
      while (vb + 1 < a.B && args.vl.boff[vb + 1] <= range0) ++vb;
    for (long long seg = range0; seg < range1; ++slot) {
      long long bh, seg_end;
      int tile0, T_len;
      if constexpr (RAG) {
        while (vb + 1 < a.B && args.vl.boff[vb + 1] <= seg) ++vb;
        T_len = args.vl.blen[vb];
        const int tpb = (T_len + 15) >> 4;
        const long long local = seg - args.vl.boff[vb];
        const int hh = static_cast<int>(local / tpb);
        tile0 = static_cast<int>(local - static_cast<long long>(hh) * tpb);
        bh = static_cast<long long>(vb) * a.Hkv + hh;
        seg_end = min(range1, args.vl.boff[vb] + static_cast<long long>(hh + 1) * tpb);
      } else {
        T_len = a.T_len;
        bh = seg / a.tiles_per_bh;
        seg_end = min(range1, (bh + 1) * a.tiles_per_bh);
        tile0 = static_cast<int>(seg - bh * a.tiles_per_bh);
      }
      const int ntiles = static_cast<int>(seg_end - seg);
      seg = seg_end;
      const int b = static_cast<int>(bh / a.Hkv), h = static_cast<int>(bh % a.Hkv);

      // ---- B operands of the score MMA: column n = r of n-tile nt < NT is head 4 nt + r/2,
      //      {q_hi, q_hi, 0, 0} (r even) or {q_mid, q_mid, q_hi, q_hi} (r odd) at the k slots
      //      of each coordinate pair; column r of n-tile NT is head r/2 (r even) or 4 + r/2
      //      (r odd) with {q_lo, q_lo, q_mid, q_mid}. Thread c holds coordinates [32c, 32c+32),
      //      k-step s its pairs 2s (b0) and 2s + 1 (b1).
      // ---- the segment's queries, rotated and split by warps 0 .. G-1 into the merge area
      //      (free between segments), then read as fragments by every warp
      QPrep *qs = reinterpret_cast<QPrep *>(obw);
      for (int g = warp; g < a.G; g += kWarps)
        prep_query(a.q, a.q_dtype, static_cast<size_t>(b) * a.Hq + h * a.G + g, a.scale, a.seed, a.kcsc,
                   qs + g, lane);
      __syncthreads();
      uint32_t qb[NT + 1][16];
      float qscale[NT];
#pragma unroll
      for (int nt = 0; nt <= NT; ++nt) {
        const int g = nt < NT ? nt * 4 + (r >> 1) : (r >> 1) + 4 * (r & 1);
        if (g < a.G) {
          const QPrep *p = qs + g;
          // the parts at the hi and the lo k slots of this column
          const int8_t *xs = nt < NT ? ((r & 1) ? p->mid : p->hi) : p->lo;
          const int8_t *ys = nt < NT ? p->hi : p->mid;
          const bool ylo = nt == NT || (r & 1); // the lo slots are used
          const uint4 *xv4 = reinterpret_cast<const uint4 *>(xs + 32 * c);
          const uint4 *yv4 = reinterpret_cast<const uint4 *>(ys + 32 * c);
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const uint4 xv = xv4[k];
            const uint4 yv = ylo ? yv4[k] : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, yw[4] = {yv.x, yv.y, yv.z, yv.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int s = 4 * k + j; // word s holds coordinates 32c + 4s .. 32c + 4s + 3
              qb[nt][2 * s] = prmt(xw[j], yw[j], 0x5410u);
              qb[nt][2 * s + 1] = prmt(xw[j], yw[j], 0x7632u);
            }
          }
        } else {
#pragma unroll
          for (int k = 0; k < 16; ++k) qb[nt][k] = 0u;
        }
        if (nt < NT) {
          const int gs = nt * 4 + c; // head of this lane's score columns
          qscale[nt] = gs < a.G ? qs[gs].inv * kLog2e : 0.f;
        }
      }

      float m_run[NT], l_run[NT];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        m_run[nt] = -INFINITY;
        l_run[nt] = 0.f;
      }
      float o[8][4];
#pragma unroll
      for (int m = 0; m < 8; ++m) o[m][0] = o[m][1] = o[m][2] = o[m][3] = 0.f;

      const size_t rec0 = PG ? 0 : static_cast<size_t>(bh) * a.T_cap;
      // paged cache: record index of token t0 (a multiple of 16: a tile never straddles a
      // page) on a given page
      [[maybe_unused]] auto page_rec = [&](int page, int t0) -> long long {
        return ((static_cast<long long>(page) * a.Hkv + h) << a.pshift) + (t0 & ((1 << a.pshift) - 1));
      };
      const int tlast = T_len - 1;
      // word offset of this lane's value run within a record (3-bit runs start mid-word for odd r)
      constexpr int kVWordOff = 0;
      const int vwo = VB == 2 ? r : (VB == 4 ? 2 * r : (3 * r) >> 1);
      [[maybe_unused]] const int vsh = VB == 3 ? 16 * (r & 1) : kVWordOff;
      // Lane pointers of the next tile this warp loads; a warp advances kWarps tiles per step.
      int jl = warp;
      const int tw0 = (tile0 + warp) * 16;
      const uint8_t *kp = a.kc + (rec0 + tw0 + r) * KR + 4 * KB * c;
      const uint8_t *vp = a.vc + (rec0 + tw0 + c) * VR + 4 * vwo;
      const uint16_t *knp = a.kn + rec0 + tw0 + r;
      const uint16_t *vnp = a.vn + rec0 + tw0 + r;

      // L2 prefetch lanes: the 128-byte lines of a tile's key codes, then of its value codes,
      // then one lane each for its key and value norms.
      constexpr int KL = 16 * KR / 128, VL = 16 * VR / 128;
      const int tp0 = tw0 + kPrefetchSteps * kWarps * 16;
      const char *pfp;
      size_t pfstep;
      if (lane < KL) {
        pfp = reinterpret_cast<const char *>(a.kc + (rec0 + tp0) * KR + 128 * lane);
        pfstep = kStep * KR;
      } else if (lane < KL + VL) {
        pfp = reinterpret_cast<const char *>(a.vc + (rec0 + tp0) * VR + 128 * (lane - KL));
        pfstep = kStep * VR;
      } else {
        pfp = reinterpret_cast<const char *>((lane == KL + VL ? a.kn : a.vn) + rec0 + tp0);
        pfstep = kStep * 2;
      }
      int tpf = tp0;

      auto load_k = [&](uint32_t (&dst)[KB], const uint8_t *p) {
        if constexpr (KB == 4) {
          const uint4 q = __ldcs(reinterpret_cast<const uint4 *>(p));
          dst[0] = q.x;
          dst[1] = q.y;
          dst[2] = q.z;
          dst[3] = q.w;
        } else {
#pragma unroll
          for (int k = 0; k < KB; ++k) dst[k] = __ldcs(reinterpret_cast<const uint32_t *>(p) + k);
        }
      };
      auto load_v = [&](uint32_t (&dst)[TileT::VW], const uint8_t *p) {
#pragma unroll
        for (int k = 0; k < TileT::VW; ++k) dst[k] = __ldcs(reinterpret_cast<const uint32_t *>(p) + k);
      };

      // One tile from the lane pointers: full tiles load at fixed offsets from them; the ragged
      // last tile of a (batch, KV head) clamps each token to T_len - 1 (those tokens are masked
      // later).
      auto load_tile = [&](TileT &T, int t0) {
        if (t0 + 16 <= T_len) {

          load_k(T.k[0], kp);
          load_k(T.k[1], kp + 8 * KR);
          load_v(T.v[0], vp);
          load_v(T.v[1], vp + 4 * VR);
          load_v(T.v[2], vp + 8 * VR);
          load_v(T.v[3], vp + 12 * VR);
          T.kn[0] = __ldcs(knp);
          T.kn[1] = __ldcs(knp + 8);
          T.vn[0] = __ldcs(vnp);
          T.vn[1] = __ldcs(vnp + 8);
        } else {
          // record of token t (within this tile, so within one page) = base + t
          const long long base = PG ? (knp - a.kn) - r - t0 : static_cast<long long>(rec0);
          const long long tr = base + min(t0 + r, tlast), tr8 = base + min(t0 + r + 8, tlast);
          const uint8_t *kb = a.kc + 4 * KB * c;
          load_k(T.k[0], kb + tr * KR);
          load_k(T.k[1], kb + tr8 * KR);
          const uint8_t *vb = a.vc + 4 * vwo;
          const int tv = t0 + c;
          load_v(T.v[0], vb + (base + min(tv, tlast)) * VR);
          load_v(T.v[1], vb + (base + min(tv + 4, tlast)) * VR);
          load_v(T.v[2], vb + (base + min(tv + 8, tlast)) * VR);
          load_v(T.v[3], vb + (base + min(tv + 12, tlast)) * VR);
          T.kn[0] = __ldcs(a.kn + tr);
          T.kn[1] = __ldcs(a.kn + tr8);
          T.vn[0] = __ldcs(a.vn + tr);
          T.vn[1] = __ldcs(a.vn + tr8);
        }
      };

      // the warp's next tile (dense and per-sequence-length walks: every kWarps-th tile)
      auto load_next = [&](TileT &T) {
        if (kPrefetchSteps > 0) {
          if (lane < KL + VL + 2 && tpf + 16 <= T_len && tpf < (tile0 + ntiles) * 16)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(pfp));
          pfp += pfstep;
          tpf += kWarps * 16;
        }
        const int t0 = (tile0 + jl) * 16;
        load_tile(T, t0);
        kp += kStep * KR;
        vp += kStep * VR;
        knp += kStep;
        vnp += kStep;
        jl += kWarps;
      };

      auto compute = [&](const TileT &T, int t0) {
        // ---- scores. A rows r and r + 8 are tokens r and r + 8; k-step s takes the lane's
        //      coordinate pairs 2s (a0: token r, a1: token r + 8) and 2s + 1 (a2, a3), one
        //      32-bit table load each. With one score n-tile pair the even and odd k-steps
        //      accumulate into separate registers (two dependent MMA chains of four instead of
        //      one of eight), added as integers at the end; with two there is no register room.
        int acc[NT + 1][4], acc2[NT + 1][4];
#pragma unroll
        for (int nt = 0; nt <= NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc[nt][e] = kMagic;
            acc2[nt][e] = 0;
          }
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          uint32_t ad0, ad1, ad2, ad3;
          if constexpr (KB == 4) {
            // table row (code byte << 8) + the lane's 4-byte entry; the base is an immediate
            // offset of the load or is added on the IMAD pipe
            const uint32_t sel0 = 0x7604u | (static_cast<uint32_t>((2 * s) & 3) << 4);
            const uint32_t sel1 = 0x7604u | (static_cast<uint32_t>((2 * s + 1) & 3) << 4);
            if constexpr (kFixed) {
              ad0 = prmt(T.k[0][s >> 1], klane, sel0); // token r
              ad1 = prmt(T.k[1][s >> 1], klane, sel0); // token r+8
              ad2 = prmt(T.k[0][s >> 1], klane, sel1);
              ad3 = prmt(T.k[1][s >> 1], klane, sel1);
            } else {
              ad0 = imad(prmt(T.k[0][s >> 1], klane, sel0), one, klut); // token r
              ad1 = imad(prmt(T.k[1][s >> 1], klane, sel0), one, klut); // token r+8
              ad2 = imad(prmt(T.k[0][s >> 1], klane, sel1), one, klut);
              ad3 = imad(prmt(T.k[1][s >> 1], klane, sel1), one, klut);
            }
          } else {
            // the 6-bit pair index lands at bits 8..13 above the lane offset of the aligned table
            ad0 = lop_and_or(bits_at(T.k[0], 12 * s, 8), 0x3F00u, klb);
            ad1 = lop_and_or(bits_at(T.k[1], 12 * s, 8), 0x3F00u, klb);
            ad2 = lop_and_or(bits_at(T.k[0], 12 * s + 6, 8), 0x3F00u, klb);
            ad3 = lop_and_or(bits_at(T.k[1], 12 * s + 6, 8), 0x3F00u, klb);
          }
          uint32_t e0, e1, e2, e3;
          if constexpr (KB == 4 && kFixed) {
            e0 = lds32_off<kFixedBase>(ad0);
            e1 = lds32_off<kFixedBase>(ad1);
            e2 = lds32_off<kFixedBase>(ad2);
            e3 = lds32_off<kFixedBase>(ad3);
          } else {
            e0 = lds32_off<0>(ad0);
            e1 = lds32_off<0>(ad1);
            e2 = lds32_off<0>(ad2);
            e3 = lds32_off<0>(ad3);
          }
#pragma unroll
          for (int nt = 0; nt <= NT; ++nt)
            imma16832((NT == 1 && (s & 1)) ? acc2[nt] : acc[nt], e0, e1, e2, e3, qb[nt][2 * s], qb[nt][2 * s + 1]);
        }
        if constexpr (NT == 1) {
#pragma unroll
          for (int nt = 0; nt <= NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nt][e] += acc2[nt][e];
        }

        // ---- online softmax (log2 domain); lane (r, c) owns head 4 nt + c, tokens r, r+8
        const float kn0 = f16_bits_to_f32(T.kn[0]);
        const float kn1 = f16_bits_to_f32(T.kn[1]);
        const float vn0 = f16_bits_to_f32(T.vn[0]);
        const float vn1 = f16_bits_to_f32(T.vn[1]);
        const bool ok0 = t0 + r < T_len, ok1 = t0 + r + 8 < T_len;
        // The softmax reference of a head moves only when a score of the tile exceeds it: one
        // vote decides, and only then are the tile's maxima reduced across the row group
        // (three shuffles) and the accumulators rescaled. Otherwise the weights are taken
        // against the current reference directly (they are at most 1 either way).
        float s0[NT], s1[NT];
        bool over = false;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          // token r: columns 2c (2^24 terms) and 2c + 1 (2^16) in acc 0, 1 of n-tile nt and the
          // 2^8 column of the same head in acc nt of n-tile NT; token r + 8 in acc 2, 3 and
          // 2 + nt
          const float d0 = fmaf(__int_as_float(acc[NT][nt]), 1.0f / 65536.0f,
                                fmaf(__int_as_float(acc[nt][1]), 1.0f / 256.0f, __int_as_float(acc[nt][0]) - kMagicAdj));
          const float d1 = fmaf(__int_as_float(acc[NT][2 + nt]), 1.0f / 65536.0f,
                                fmaf(__int_as_float(acc[nt][3]), 1.0f / 256.0f, __int_as_float(acc[nt][2]) - kMagicAdj));
          s0[nt] = ok0 ? kn0 * qscale[nt] * d0 : -INFINITY;
          s1[nt] = ok1 ? kn1 * qscale[nt] * d1 : -INFINITY;
          over |= s0[nt] > m_run[nt] || s1[nt] > m_run[nt];
        }
        if (__any_sync(0xffffffffu, over)) {
          float alpha[NT];
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            float mx = fmaxf(s0[nt], s1[nt]);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float mn = fmaxf(m_run[nt], mx);
            alpha[nt] = softmax_exp2(m_run[nt] - mn);
            l_run[nt] *= alpha[nt];
            m_run[nt] = mn;
          }
          // rescale the value accumulators (lane owns heads 2c, 2c+1)
          float a0[NT], a1[NT];
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            a0[nt] = __shfl_sync(0xffffffffu, alpha[nt], (2 * c) & 3);
            a1[nt] = __shfl_sync(0xffffffffu, alpha[nt], (2 * c + 1) & 3);
          }
          const float al0 = NT == 2 && c >= 2 ? a0[NT - 1] : a0[0];
          const float al1 = NT == 2 && c >= 2 ? a1[NT - 1] : a1[0];
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            o[m][0] *= al0;
            o[m][1] *= al1;
            o[m][2] *= al0;
            o[m][3] *= al1;
          }
        }
        uint32_t pk[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const float p0 = softmax_exp2(s0[nt] - m_run[nt]), p1 = softmax_exp2(s1[nt] - m_run[nt]);
          l_run[nt] += p0 + p1;
          pk[nt] = pack_h2(p0 * vn0, p1 * vn1);
        }

        // ---- P'^T as the B operand: lane (r, c) needs head g = r at k rows 2c, 2c+1, 2c+8, 2c+9,
        //      which hold tokens c, c+4, c+8, c+12
        const int src0 = 4 * c + (r & 3);
        uint32_t x0 = __shfl_sync(0xffffffffu, pk[0], src0);
        uint32_t x1 = __shfl_sync(0xffffffffu, pk[0], src0 + 16);
        if (NT == 2) {
          const uint32_t y0 = __shfl_sync(0xffffffffu, pk[NT - 1], src0);
          const uint32_t y1 = __shfl_sync(0xffffffffu, pk[NT - 1], src0 + 16);
          if (r >= 4) {
            x0 = y0;
            x1 = y1;
          }
        }
        if (r >= a.G) x0 = x1 = 0u;
        const uint32_t pb0 = prmt(x0, x1, 0x5410u); // tokens c, c+4
        const uint32_t pb1 = prmt(x0, x1, 0x7632u); // tokens c+8, c+12

        // ---- values. m-tile m covers the lane's run coordinates 2m (rows r) and 2m + 1
        //      (rows r+8); operand quad (a0, a1, a2, a3) = (2m, 2m+1) x tokens (c, c+4) then
        //      (c+8, c+12).
        if constexpr (VB == 2) {
          // Interleave the nibbles of the two tokens of each k pair: byte k of u holds both
          // tokens' codes at run coordinates 4k, 4k+1 (m-tile 2k), byte k of w those at 4k+2,
          // 4k+3 (m-tile 2k+1); one 64-bit table load per byte is the operand pair (a0, a1)
          // or (a2, a3) of that m-tile.
          const uint32_t u01 = (T.v[0][0] & 0x0F0F0F0Fu) | ((T.v[1][0] << 4) & 0xF0F0F0F0u);
          const uint32_t w01 = ((T.v[0][0] >> 4) & 0x0F0F0F0Fu) | (T.v[1][0] & 0xF0F0F0F0u);
          const uint32_t u23 = (T.v[2][0] & 0x0F0F0F0Fu) | ((T.v[3][0] << 4) & 0xF0F0F0F0u);
          const uint32_t w23 = ((T.v[2][0] >> 4) & 0x0F0F0F0Fu) | (T.v[3][0] & 0xF0F0F0F0u);
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const uint32_t sel = 0x7604u | (static_cast<uint32_t>(m >> 1) << 4);
            const uint32_t x01 = (m & 1) ? w01 : u01, x23 = (m & 1) ? w23 : u23;
            uint2 e01, e23;
            if constexpr (kFixed) {
              e01 = lds64_off<kFixedBase + L::kBytes>(prmt(x01, vlane8, sel));
              e23 = lds64_off<kFixedBase + L::kBytes>(prmt(x23, vlane8, sel));
            } else {
              e01 = lds64_off<0>(imad(prmt(x01, vlane8, sel), one, vlut));
              e23 = lds64_off<0>(imad(prmt(x23, vlane8, sel), one, vlut));
            }
            mma16816(o[m], e01.x, e01.y, e23.x, e23.y, pb0, pb1);
          }
        } else {
          // one lane-replicated table word per token and coordinate pair: the word indexed by a
          // token's codes at run coordinates 2m, 2m+1 holds both centroids (fp16x2); two PRMTs
          // turn the words of the two tokens of a k pair into the operand registers of
          // coordinates 2m and 2m+1
          uint32_t run[4][2];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            if constexpr (VB == 3) {
              run[t][0] = __funnelshift_r(T.v[t][0], T.v[t][1], vsh);
              run[t][1] = T.v[t][1] >> vsh;
            } else {
              run[t][0] = T.v[t][0];
              run[t][1] = T.v[t][1];
            }
          }
          // row index above the lane offset: at bit 7 of a size-aligned table, or at bit 8 (rows
          // 256 bytes apart) in the second halves of the 4-bit key rows
          constexpr int kIxBit = L::kVInK ? 8 : 7;
          constexpr uint32_t MI = ((1u << (2 * VB)) - 1u) << kIxBit;
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            uint32_t w[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              if constexpr (!L::kVInK) {
                w[t] = lds32_off<0>(lop_and_or(bits_at(run[t], 2 * VB * m, kIxBit), MI, vlb));
              } else if constexpr (kFixed) {
                w[t] = lds32_off<kFixedBase + 128>(lop_and_or(bits_at(run[t], 2 * VB * m, kIxBit), MI, lanebase));
              } else {
                w[t] = lds32_off<0>(imad(lop_and_or(bits_at(run[t], 2 * VB * m, kIxBit), MI, lanebase), one, vkb));
              }
            }
            mma16816(o[m], prmt(w[0], w[1], 0x5410u), prmt(w[0], w[1], 0x7632u), prmt(w[2], w[3], 0x5410u),
                     prmt(w[2], w[3], 0x7632u), pb0, pb1);
          }
        }
      };

      // Two tile buffers in turn: the next tile loads while the current one computes.
      TileT ta, tb;
      if constexpr (!PG) {
        int jt = warp;
        if (jl < ntiles) load_next(ta);
        while (jt < ntiles) {
          if (jl < ntiles) load_next(tb);
          compute(ta, (tile0 + jt) * 16);
          jt += kWarps;
          if (jt >= ntiles) break;
          if (jl < ntiles) load_next(ta);
          compute(tb, (tile0 + jt) * 16);
          jt += kWarps;
        }
      } else {
        // Paged cache: the segment's tiles are grouped into aligned chunks of ct = min(tiles
        // per page, 4) tiles, which never straddle a page, and the warps take the chunks in
        // turn, so the block table and the page arithmetic are visited once per chunk; inside
        // a chunk the records are consecutive. Pages are looked up two chunks ahead, and each
        // chunk is prefetched into L2 one chunk ahead.
        const int lc = min(a.pshift - 4, 2), ct = 1 << lc;
        const int tend = tile0 + ntiles; // absolute tile end of the segment
        const int cw = (tile0 >> lc) + warp;
        const int *btrow = a.bt + static_cast<size_t>(b) * a.maxp;
        auto chunk_page = [&](int ch) -> int {
          const int u = ch << lc;
          return u < tend ? __ldg(btrow + (u >> (a.pshift - 4))) : 0;
        };
        auto set_ptrs = [&](int page, int u) {
          const long long rb = page_rec(page, u * 16);
          kp = a.kc + (rb + r) * KR + 4 * KB * c;
          vp = a.vc + (rb + c) * VR + 4 * vwo;
          knp = a.kn + rb + r;
          vnp = a.vn + rb + r;
        };
        auto prefetch_chunk = [&](int ch, int page) {
          const int u = ch << lc;
          if (u >= tend) return;
          const long long rc = page_rec(page, u * 16);
          const int kls = ct * KR / 8, vls = ct * VR / 8; // 128-byte lines of the chunk
          for (int i = lane; i < kls + vls + 2; i += 32) {
            const char *pp = i < kls ? reinterpret_cast<const char *>(a.kc + rc * KR) + 128 * i
                             : i < kls + vls ? reinterpret_cast<const char *>(a.vc + rc * VR) + 128 * (i - kls)
                                             : reinterpret_cast<const char *>((i == kls + vls ? a.kn : a.vn) + rc);
            asm volatile("prefetch.global.L2 [%0];" ::"l"(pp));
          }
        };
        // the tile after u in the warp's walk
        auto nxt = [&](int u) { return ((u + 1) & (ct - 1)) ? u + 1 : u + 1 + (kWarps - 1) * ct; };
        int ul = max(tile0, cw << lc), ut = ul; // next tile to load, next tile to compute
        int pg_b = chunk_page(cw + kWarps), pg_c = chunk_page(cw + 2 * kWarps);
        if (ul < tend) set_ptrs(chunk_page(cw), ul);
        prefetch_chunk(cw + kWarps, pg_b);
        auto load_pg = [&](TileT &T) {
          load_tile(T, ul * 16);
          ul = nxt(ul);
          if ((ul & (ct - 1)) == 0) {
            // the next tile starts the warp's next chunk, on page pg_b
            const int ch = ul >> lc;
            if (ul < tend) set_ptrs(pg_b, ul);
            prefetch_chunk(ch + kWarps, pg_c);
            pg_b = pg_c;
            pg_c = chunk_page(ch + 2 * kWarps);
          } else {
            kp += 16 * KR;
            vp += 16 * VR;
            knp += 16;
            vnp += 16;
          }
        };
        if (ul < tend) load_pg(ta);
        while (ut < tend) {
          if (ul < tend) load_pg(tb);
          compute(ta, ut * 16);
          ut = nxt(ut);
          if (ut >= tend) break;
          if (ul < tend) load_pg(ta);
          compute(tb, ut * 16);
          ut = nxt(ut);
        }
      }

      // ---- merge the warps: common max and sum per head, then each warp stores its rescaled
      //      accumulators in its own slots ([m-tile][lane] float4, conflict-free) and the
      //      threads sum them over the warps into the partial record
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float l = l_run[nt];
        l += __shfl_xor_sync(0xffffffffu, l, 4);
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        if (r == 0) {
          mst[warp * 8 + nt * 4 + c] = m_run[nt];
          lst[warp * 8 + nt * 4 + c] = l;
        }
      }
      __syncthreads();
      if (tid < 8) {
        float M = -INFINITY;
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mst[w * 8 + tid]);
        float Ls = 0.f;
        for (int w = 0; w < kWarps; ++w) {
          const float mw = mst[w * 8 + tid];
          if (mw != -INFINITY) Ls = fmaf(lst[w * 8 + tid], exp2f(mw - M), Ls);
        }
        gmx[tid] = M;
        lsum[tid] = Ls;
      }
      __syncthreads();
      {
        const int g0 = 2 * c, g1 = 2 * c + 1;
        const float f0 = g0 < a.G ? exp2f(mst[warp * 8 + g0] - gmx[g0]) : 0.f;
        const float f1 = g1 < a.G ? exp2f(mst[warp * 8 + g1] - gmx[g1]) : 0.f;
        float4 *ow = obw + warp * 256 + lane;
#pragma unroll
        for (int m = 0; m < 8; ++m)
          ow[32 * m] = make_float4(o[m][0] * f0, o[m][1] * f1, o[m][2] * f0, o[m][3] * f1);
      }
      __syncthreads();
      float *dst = a.part + (static_cast<size_t>(blockIdx.x) * a.slots + slot) * a.G * a.stride;
      for (int idx = tid; idx < 256; idx += kThreads) {
        float4 acc = obw[idx];
        for (int w = 1; w < kWarps; ++w) {
          const float4 x = obw[w * 256 + idx];
          acc.x += x.x;
          acc.y += x.y;
          acc.z += x.z;
          acc.w += x.w;
        }
        // slot (m, lane (rr, cc)): coordinates 16 rr + 2m, +1 of heads 2 cc, 2 cc + 1
        const int m = idx >> 5, rr = (idx >> 2) & 7, cc = idx & 3;
        const int i0 = 16 * rr + 2 * m;
        if (2 * cc < a.G)
          *reinterpret_cast<float2 *>(dst + static_cast<size_t>(2 * cc) * a.stride + 2 + i0) =
              make_float2(acc.x, acc.z);
        if (2 * cc + 1 < a.G)
          *reinterpret_cast<float2 *>(dst + static_cast<size_t>(2 * cc + 1) * a.stride + 2 + i0) =
              make_float2(acc.y, acc.w);
      }
      if (tid < a.G) {
        dst[static_cast<size_t>(tid) * a.stride] = gmx[tid];
        dst[static_cast<size_t>(tid) * a.stride + 1] = lsum[tid];
      }
      __syncthreads();
    }
  };
  if (KB == 4 && klut == kFixedBase)
    run(std::true_type{});
  else
    run(std::false_type{});
}

// Merge the partial records of one (b, q-head) (log2-domain maxima), apply the inverse
// rotation D H / d once and divide by the softmax sum. One warp per (b, q-head): lane k reads
// the maximum and sum of partial k, so the merge weights need one round of loads; lane l then
// owns output coordinates [4 l, 4 l + 4) and the Walsh-Hadamard butterflies of span >= 4 run
// across lanes with shuffles.
template <bool RAG>
__global__ void __launch_bounds__(128) combine_fast_kernel(const float *part, int B, int Hkv, int G,
                                                           int tiles_per_bh, int tiles_per_cta,
                                                           int slots, int stride, uint64_t seed,
                                                           float *out,
                                                           const std::conditional_t<RAG, VarLen, NoVarLen> vl) {
  const int lane = threadIdx.x & 31;
  const int Hq = Hkv * G;
  const int gw = blockIdx.x * 4 + (threadIdx.x >> 5); // (b, q-head) of this warp
  pdl_wait(); // the partials come from the decode kernel
  pdl_trigger(); // the next kernel's prologue may overlap this one (it waits for its end)
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
  // inverse rotation: butterflies within the lane, then across lanes
  {
    const float a0 = acc[0] + acc[1], a1 = acc[0] - acc[1];
    const float a2 = acc[2] + acc[3], a3 = acc[2] - acc[3];
    acc[0] = a0 + a2;
    acc[2] = a0 - a2;
    acc[1] = a1 + a3;
    acc[3] = a1 - a3;
  }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float o = __shfl_xor_sync(0xffffffffu, acc[e], m);
      acc[e] = upper ? o - acc[e] : acc[e] + o;
    }
  }
  const float sc = 1.0f / (static_cast<float>(kD) * L);
  const uint64_t sw = dev_splitmix64(seed, static_cast<uint64_t>(lane >> 4)); // coordinates 64 k ..
  const int sb = (4 * lane) & 63;
  float4 r;
  r.x = ((sw >> sb) & 1ull) ? -acc[0] * sc : acc[0] * sc;
  r.y = ((sw >> (sb + 1)) & 1ull) ? -acc[1] * sc : acc[1] * sc;
  r.z = ((sw >> (sb + 2)) & 1ull) ? -acc[2] * sc : acc[2] * sc;
  r.w = ((sw >> (sb + 3)) & 1ull) ? -acc[3] * sc : acc[3] * sc;
  reinterpret_cast<float4 *>(out + (static_cast<size_t>(b) * Hq + hq) * kD)[lane] = r;
}

constexpr int kSmemPerSm = 228 * 1024;

template <int KB, int VB>
int ctas_per_sm() {
  return std::max(1, std::min(Cfg<KB, VB>::kCtas, kSmemPerSm / (Lut<KB, VB>::kSmem + 1024)));
}

// CTAs of the tensor-core decode kernel that fit on one SM.
int mse_ctas_per_sm(int kb, int vb) {
  if (kb == 4) return vb == 2 ? ctas_per_sm<4, 2>() : vb == 3 ? ctas_per_sm<4, 3>() : ctas_per_sm<4, 4>();
  return vb == 2 ? ctas_per_sm<3, 2>() : vb == 3 ? ctas_per_sm<3, 3>() : ctas_per_sm<3, 4>();
}

template <int KB, int VB>
cudaError_t run_mse(const FastArgs &f, const VarLen *vl, int ctas, cudaStream_t s) {
  constexpr int smem = Lut<KB, VB>::kSmem;
  cudaError_t e;
  if (vl) {
    auto kern = f.bt ? (f.G <= 4 ? decode_mse_kernel<KB, VB, 1, 2> : decode_mse_kernel<KB, VB, 2, 2>)
                     : (f.G <= 4 ? decode_mse_kernel<KB, VB, 1, 1> : decode_mse_kernel<KB, VB, 2, 1>);
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    FastArgsV fv;
    fv.a = f;
    fv.vl = *vl;
    return launch_pdl(kern, dim3(ctas), dim3(Cfg<KB, VB>::kThreads), smem, s, fv);
  }
  auto kern = f.G <= 4 ? decode_mse_kernel<KB, VB, 1, 0> : decode_mse_kernel<KB, VB, 2, 0>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(ctas), dim3(Cfg<KB, VB>::kThreads), smem, s, f);
}

} // namespace

bool fast_decode_supported(int d, int k_mode, int k_wbits, int v_mode, int v_wbits, int G) {
  return d == kD && k_mode == TQ_MSE && (k_wbits == 3 || k_wbits == 4) && v_mode == TQ_MSE &&
         v_wbits >= 2 && v_wbits <= 4 && G >= 1 && G <= 8;
}

// Layout of the fast path's workspace: the partial records (the kernel prepares its queries in
// shared memory).
void plan_fast(int B, int Hq, int Hkv, int T_len, int sm_count, int kb, int vb, DecodePlan *p,
               const int *T_lens) {
  const int G = Hq / Hkv;
  p->path = 1;
  p->tile = 16;
  p->gc = G;
  p->ws_stride = 2 + kD + 2; // 132 floats
  p->tiles_per_bh = (T_len + 15) / 16;
  long long total = static_cast<long long>(B) * Hkv * p->tiles_per_bh;
  if (T_lens) {
    total = 0;
    for (int b = 0; b < B; ++b) total += static_cast<long long>(Hkv) * ((T_lens[b] + 15) / 16);
  }
  long long ctas = static_cast<long long>(sm_count) * mse_ctas_per_sm(kb, vb);
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
  p->ws_bytes = p->part_bytes; // the decode kernel prepares the queries in shared memory
}

cudaError_t launch_fast_decode(const DecodeArgs &a, cudaStream_t s) {
  const DecodePlan &p = a.plan;
  FastArgs f;
  f.kc = a.k.codes;
  f.vc = a.v.codes;
  f.kn = a.k.norm;
  f.vn = a.v.norm;
  f.q = a.q;
  f.q_dtype = a.q_dtype;
  f.scale = a.scale;
  f.seed = a.seed;
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
  for (int j = 0; j < 16; ++j) f.kcent[j] = a.k.cb.c[j];
  f.kcsc = a.k.cb.fix_scale;
  for (int j = 0; j < 16; ++j) f.vcent[j] = a.v.cb.c[j];
  f.one = 1u;
  f.B = a.B;
  f.bt = a.pg.bt;
  f.pshift = a.pg.pshift;
  f.maxp = a.pg.maxp;
  VarLen vl;
  const VarLen *vlp = nullptr;
  if (a.T_lens) {
    vl.on = 1;
    vl.boff[0] = 0;
    for (int b = 0; b < a.B; ++b) {
      vl.blen[b] = a.T_lens[b];
      vl.boff[b + 1] = vl.boff[b] + a.Hkv * ((a.T_lens[b] + 15) / 16);
    }
    // the ragged tile space ends at boff[B]: the last CTA's range stops there (past it lies no
    // (sequence, KV head), and its records, queries and block-table entries are out of bounds)
    f.total_tiles = vl.boff[a.B];
    vlp = &vl;
  }
  const int kb = a.k.wbits, vb = a.v.wbits;
  cudaError_t e;
  if (kb == 4) e = vb == 2 ? run_mse<4, 2>(f, vlp, p.ctas, s) : vb == 3 ? run_mse<4, 3>(f, vlp, p.ctas, s)
                                                                      : run_mse<4, 4>(f, vlp, p.ctas, s);
  else e = vb == 2 ? run_mse<3, 2>(f, vlp, p.ctas, s) : vb == 3 ? run_mse<3, 3>(f, vlp, p.ctas, s)
                                                               : run_mse<3, 4>(f, vlp, p.ctas, s);
  if (e != cudaSuccess) return e;
  if (vlp)
    return launch_pdl(combine_fast_kernel<true>, dim3((a.B * a.Hq + 3) / 4), dim3(128), 0, s,
                      static_cast<const float *>(a.ws), a.B, a.Hkv, f.G, p.tiles_per_bh,
                      p.tiles_per_cta, p.slots, p.ws_stride, a.seed, a.out, vl);
  return launch_pdl(combine_fast_kernel<false>, dim3((a.B * a.Hq + 3) / 4), dim3(128), 0, s,
                    static_cast<const float *>(a.ws), a.B, a.Hkv, f.G, p.tiles_per_bh,
                    p.tiles_per_cta, p.slots, p.ws_stride, a.seed, a.out, NoVarLen{});
}

} // namespace tq
