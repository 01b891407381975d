// Decode attention from packed codes whose keys are dequantized through a
// table: 3-bit Lloyd-Max keys with the QJL bit (k4v4: m = 128), and the
// MSE-only formats: norm-corrected 3- or 4-bit keys (k3v4_nc, 4bit_nc,
// 3bit_nc) and 8-bit keys (k8v4); values 4 bits (3 bits for 3bit_nc),
// d = 128, any GQA group of 1, 2, 4 or 8, on the tensor cores (sm_100a).
//
// Same quantities as the 2-bit-key kernels ("What is TurboQuant?", "How
// TurboQuant works", closing paragraph; "How to implement" part 1):
//   l_i = |k_i| <q', c_k[idx_i]> (+ sqrt(pi/2)/m * gamma_i <S q', sigma_i>
//   with the QJL stage), online softmax, o = sum p_i |v_i| c_v[vidx_i] in the
// rotated domain; the merge kernel combines the partials by log-sum-exp and
// applies Pi^T.  Norm correction only changes the stored |k_i| and |v_i|
// ("A First Comprehensive Study of TurboQuant", section A3), so these
// kernels read it like any norm.
//
// An 8- or 16-level codebook is not affine in its index bits, so the key
// product dequantizes: two neighbouring coordinates of a token (a 6-bit index
// from their two 2-bit fields and two top bits, or the byte of their two
// 4-bit fields) select a half2 of centroids from a table in shared memory,
// 16 copies (each half-warp lane reads its own, so the 64-bit reads of a
// half-warp hit distinct banks); 8-bit keys take one coordinate per entry,
// 32 copies.  3-bit keys run three CTAs per SM with two pipeline stages per
// warp (their tables are small enough), the others two CTAs.  Each entry holds the
// fp16 head of the centroid pair and its tail x 2^12; the query operand
// likewise carries an fp16 head and tail, and three MMAs per k-step form
// head*head + head*tail + tail*head (~22 bits).  The QJL product, the
// softmax, the value product and the work split are those of the group-8
// kernel for 2-bit keys: balanced CTA ranges of 16-token tiles, query
// operands built once per row piece into shared memory.
//
// Key layouts (d = 128).  3-bit fields: words 0..7 hold the low two bits of
// the indices (16 coordinates per word), words 8..11 the top bits (32 per
// word); thread t of a quad owns coordinates 32t .. 32t+31: 2-bit words 2t,
// 2t+1 and top-bit word t.  4-bit fields: 8 coordinates per word; thread t
// owns words 4t .. 4t+3.  Either way k-step s (0..7) pairs coordinates
// 32t + 2s, +1 (MMA k 2t, 2t+1) and 32t + 16 + 2s, +1 (k 2t+8, 2t+9).
//
// Group 4 uses the same tiles with the columns of query heads 4..7 empty:
// one head MMA instead of two per k-step, and one softmax state per thread.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cmath>

#include "tq_attn_common.cuh"
#include "tq_internal.h"

namespace tqk {
namespace {

constexpr int NSTK = 3;      // pipeline stages per warp
constexpr int QOPK = 8;      // words per lane and key k-step (G = 8: 6 used, G = 4: 4 used)
constexpr int QOPQ = 4;      // words per lane and QJL k-step (2 MMAs x 2)

// Key formats.  3 and 4 bits: a table entry covers two coordinates (8 bytes:
// heads, tails).  8 bits: an entry covers one coordinate (4 bytes: head,
// tail), 32 copies, and staged rows of 36 words keep the 16-byte loads of
// each quarter-warp on distinct banks.
template <int KB>
struct KeyFmt {
  static constexpr int K2W = KB == 3 ? 8 : (KB == 4 ? 16 : 36);   // staged row (words)
  static constexpr int REC = KB == 3 ? 12 : (KB == 4 ? 16 : 32);  // words per key record
  static constexpr int ENT = KB == 3 ? 64 : 256;                  // table entries
  static constexpr int COP = KB == 8 ? 32 : 16;                   // copies of the table
  static constexpr int ESZ = KB == 8 ? 4 : 8;                     // bytes per entry
  static constexpr size_t LUT_BYTES = (size_t)ENT * COP * ESZ;
  static constexpr int NS = KB == 4 ? NSTK : 2;                   // pipeline stages (shared memory)
  static constexpr int CTAS = KB == 3 ? 3 : 2;                    // CTAs per SM
};

// Values: 4-bit fields (16 words per token, rows padded to VROW) or 3-bit
// (2-bit stream of 8 words, then 4 top-bit words: 12-word rows, on which the
// loads of value_tile3 meet distinct banks).
template <int VB>
struct ValFmt {
  static constexpr int REC = VB == 4 ? 16 : 12;       // words per value record
  static constexpr int ROW = VB == 4 ? VROW : 12;     // staged row (words)
  static constexpr int LUTW = VB == 4 ? LUT_WORDS : 64 * 32;
};

template <int KB, bool QJL, int VB>
struct StageL {
  uint32_t k2[MT][KeyFmt<KB>::K2W];   // 2-bit stream (3-bit keys) or the 4- / 8-bit fields
  uint32_t k1[MT][KB == 3 ? 4 : 1];   // top-bit stream (3-bit keys)
  uint32_t q[MT][QJL ? QW : 1];       // QJL words
  float kn[MT];
  float kr[MT];
  float vn[MT];
  alignas(16) uint32_t v[MT][ValFmt<VB>::ROW];
};

template <int KB, bool QJL, int VB>
constexpr size_t smem_lut() {
  return KeyFmt<KB>::LUT_BYTES + (size_t)ValFmt<VB>::LUTW * 4 +
         (size_t)MW * KeyFmt<KB>::NS * sizeof(StageL<KB, QJL, VB>) +
         (size_t)8 * 32 * QOPK * 4 + (QJL ? (size_t)8 * 32 * QOPQ * 4 : 0) + 8 * 16 + MW * 4 + 16 * 4;
}

// 3-bit value table: entry (idx, lane) = half2(cv[ia], cv[ib]) for the codes
// ia, ib of two tokens at one coordinate, idx = lo2(a) | lo2(b) << 2 |
// top(a) << 4 | top(b) << 5.
__device__ __forceinline__ void build_value_lut3(uint32_t* lut, const float* cv, int tid, int nthreads) {
  for (int e = tid; e < 64 * 32; e += nthreads) {
    const int idx = e >> 5;
    const int ia = (idx & 3) | (((idx >> 4) & 1) << 2), ib = ((idx >> 2) & 3) | (((idx >> 5) & 1) << 2);
    lut[e] = pack_half2(cv[ia], cv[ib]);
  }
}

// Bits 0..15 of x spread to the even bit positions.
__device__ __forceinline__ uint32_t spread16(uint32_t x) {
  x = (x | (x << 8)) & 0x00FF00FFu;
  x = (x | (x << 4)) & 0x0F0F0F0Fu;
  x = (x | (x << 2)) & 0x33333333u;
  return (x | (x << 1)) & 0x55555555u;
}

// value_tile for 3-bit value codes: o[mt] += V^T P over one 16-token tile.
// Thread (g, t) covers coordinates 16g .. 16g+15 (2-bit word g, top bits
// 16 (g & 1) .. of word 8 + g/2) of tokens 2t, 2t+1 (k 2t, 2t+1) and 2t+8,
// 2t+9; row g of MMA mt is coordinate 16g + mt, row g+8 is 16g + 8 + mt.
__device__ __forceinline__ void value_tile3(float (&o)[8][4], const uint32_t (*v)[12], uint32_t pb0,
                                            uint32_t pb1, uint32_t lut_lane, int g, int t) {
  const int sh = 16 * (g & 1);
  uint32_t ne[2], no[2], tt[2];
#pragma unroll
  for (int pr = 0; pr < 2; ++pr) {
    const int ra = 2 * t + 8 * pr;
    const uint32_t A = v[ra][g], B = v[ra + 1][g];
    const uint32_t TA = (v[ra][8 + (g >> 1)] >> sh) & 0xFFFFu, TB = (v[ra + 1][8 + (g >> 1)] >> sh) & 0xFFFFu;
    ne[pr] = (A & 0x33333333u) | ((B & 0x33333333u) << 2);   // nibble k: coordinate 2k
    no[pr] = ((A >> 2) & 0x33333333u) | (B & 0xCCCCCCCCu);   // nibble k: coordinate 2k + 1
    tt[pr] = spread16(TA) | (spread16(TB) << 1);             // bits 2j, 2j+1: top bits of a, b
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    uint32_t av[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int pr = r >> 1, j = mt + 8 * (r & 1);
      const uint32_t nib = ((j & 1 ? no[pr] : ne[pr]) >> (4 * (j >> 1))) & 0xFu;
      const uint32_t top = (tt[pr] >> (2 * j)) & 3u;
      av[r] = lds32(((nib | (top << 4)) << 7) + lut_lane);
    }
    mma16816(o[mt], av[0], av[1], av[2], av[3], pb0, pb1);
  }
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0,%1}, [%2];\n" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

// Byte offset of the 3-bit key-table entry of coordinates 2s, 2s+1 of word
// pair (w2, w1 >> sh), without the lane offset: idx * 16 copies * 8 bytes.
template <int S, int SH>
__device__ __forceinline__ uint32_t klut_off(uint32_t w2, uint32_t w1) {
  const uint32_t nib = (w2 >> (4 * S)) & 0xFu;
  const uint32_t top = (w1 >> (SH + 2 * S)) & 3u;
  return (nib | (top << 4)) << 7;
}
// 4-bit keys: byte B of word w indexes the table (16 copies * 8 bytes); 8-bit
// keys likewise (32 copies * 4 bytes).
template <int B>
__device__ __forceinline__ uint32_t klut4_off(uint32_t w) {
  return __byte_perm(w, 0, 0x4440 + B) << 7;
}
// 8-bit keys: the (head, tail) operand pair of coordinates in bytes B, B+1 of w.
template <int B>
__device__ __forceinline__ uint2 k8_pair(uint32_t lane_base, uint32_t w) {
  const uint32_t x0 = lds32(lane_base + klut4_off<B>(w)), x1 = lds32(lane_base + klut4_off<B + 1>(w));
  return make_uint2(__byte_perm(x0, x1, 0x5410), __byte_perm(x0, x1, 0x7632));
}

template <bool PAGED, int KB, bool QJL, int G, int VB>
__global__ void __launch_bounds__(MW * 32, KeyFmt<KB>::CTAS) k_attn_lut(AttnArgs a) {
  static_assert(G == 2 || G == 4 || G == 8, "group template 2 (groups 1, 2), 4 or 8");
  using KF = KeyFmt<KB>;
  using VF = ValFmt<VB>;
  using Stage = StageL<KB, QJL, VB>;
  constexpr int NJ = G == 8 ? 2 : 1;   // head sets per thread: t (and 4 + t)
  const int Gr = G == 2 ? a.G : G;      // heads in the group (1 or 2 under the template 2)
  extern __shared__ __align__(16) unsigned char smem[];
  uint2* klut = reinterpret_cast<uint2*>(smem);                                          // [ENT][COP]
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem + KF::LUT_BYTES);                     // values
  Stage* stages = reinterpret_cast<Stage*>(smem + KF::LUT_BYTES + (size_t)VF::LUTW * 4);
  uint32_t* qopk = reinterpret_cast<uint32_t*>(stages + MW * KF::NS);                    // [8][32][8]
  uint32_t* qopq = qopk + 8 * 32 * QOPK;                                                  // [8][32][4] (QJL)
  float4* s_head = reinterpret_cast<float4*>(qopq + (QJL ? 8 * 32 * QOPQ : 0));          // [8]
  float* s_vmax = reinterpret_cast<float*>(s_head + 8);                                  // [MW]
  int* s_scale = reinterpret_cast<int*>(s_vmax + MW);                                    // [16]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const bool hv0 = t < Gr;              // this thread's head t exists

  if (VB == 4)
    build_value_lut(lut, a.cv, tid, MW * 32);
  else
    build_value_lut3(lut, a.cv, tid, MW * 32);
  // Key table: entry (idx, copy) = (fp16 heads, fp16 tails x 2^12) of the
  // centroids of two coordinates; idx = f0 | f1 << 2 | top0 << 4 | top1 << 5
  // (3-bit: f = 2-bit field, top = third index bit) or the byte f0 | f1 << 4
  // (4-bit fields).
  for (int e = tid; e < KF::ENT * KF::COP; e += MW * 32) {
    const int idx = e / KF::COP;
    if (KB == 8) {   // one coordinate: (head, tail x 2^12)
      const float c0 = a.ck[idx];
      const float h0 = __half2float(__float2half_rn(c0));
      reinterpret_cast<uint32_t*>(klut)[e] = pack_half2(h0, (c0 - h0) * 4096.f);
      continue;
    }
    int i0, i1;
    if (KB == 3) {
      i0 = (idx & 3) | (((idx >> 4) & 1) << 2);
      i1 = ((idx >> 2) & 3) | (((idx >> 5) & 1) << 2);
    } else {
      i0 = idx & 15;
      i1 = idx >> 4;
    }
    const float c0 = a.ck[i0], c1 = a.ck[i1];
    const float h0 = __half2float(__float2half_rn(c0)), h1 = __half2float(__float2half_rn(c1));
    klut[e] = make_uint2(pack_half2(h0, h1), pack_half2((c0 - h0) * 4096.f, (c1 - h1) * 4096.f));
  }
  __syncthreads();

  const int64_t* P = a.tiles;
  const int64_t W = P[a.B];
  const int64_t NC = min((int64_t)gridDim.x, W);
  const int64_t cta = blockIdx.x;
  if (cta >= NC) return;   // uniform over the CTA
  int64_t x = cta * W / NC;
  const int64_t x1 = (cta + 1) * W / NC;
  int b = locate_sequence(P, a.B, x);

  const uint32_t klut_lane = (uint32_t)__cvta_generic_to_shared(klut) + (lane % KF::COP) * KF::ESZ;
  constexpr int NS = KF::NS;
  const uint32_t lut_lane = (uint32_t)__cvta_generic_to_shared(lut) + lane * 4;
  const uint32_t qopk_lane = (uint32_t)__cvta_generic_to_shared(qopk) + lane * QOPK * 4;
  const uint32_t qopq_lane = (uint32_t)__cvta_generic_to_shared(qopq) + lane * QOPQ * 4;
  Stage* my = stages + warp * NS;
  const uint32_t my_s = (uint32_t)__cvta_generic_to_shared(my);

  while (x < x1) {
    while (P[b + 1] <= x) ++b;
    const int64_t tb = (P[b + 1] - P[b]) / a.Hkv;
    const int64_t rel = x - P[b];
    const int kvh = (int)(rel / tb);
    const int64_t tt = rel - (int64_t)kvh * tb;
    const int64_t te = min(tb, tt + (x1 - x));
    const int nt = (int)(te - tt);
    const int64_t slot = 4 * (cta + (int64_t)b * a.Hkv + kvh) + warp;
    x += nt;

    const int64_t len = min((int64_t)max(a.seq_lens[b], 0), a.max_T);
    const int64_t tok0 = tt * MT;
    const int64_t tok1 = min(te * MT, len);
    const int64_t qbase = (int64_t)b * a.Hq + (int64_t)kvh * Gr;

    __syncthreads();   // the previous piece's readers of the operands are done
    // ---- per-head scales (warp w: heads 2w, 2w+1) and the value-norm maximum ----
#pragma unroll
    for (int hsel = 0; hsel < 2; ++hsel) {
      const int h = 2 * warp + hsel;
      if (h >= Gr) continue;   // uniform over the warp
      const float4 q4 = reinterpret_cast<const float4*>(a.qr + (qbase + h) * 128)[lane];
      float mq = fmaxf(fmaxf(fabsf(q4.x), fabsf(q4.y)), fmaxf(fabsf(q4.z), fabsf(q4.w)));
      float ms = 0.f, ss = 0.f;
      if (QJL) {
        const float4 s4 = reinterpret_cast<const float4*>(a.qs + (qbase + h) * 128)[lane];
        ms = fmaxf(fmaxf(fabsf(s4.x), fabsf(s4.y)), fmaxf(fabsf(s4.z), fabsf(s4.w)));
        ss = (s4.x + s4.y) + (s4.z + s4.w);
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        mq = fmaxf(mq, __shfl_xor_sync(0xffffffffu, mq, o));
        if (QJL) {
          ms = fmaxf(ms, __shfl_xor_sync(0xffffffffu, ms, o));
          ss += __shfl_xor_sync(0xffffffffu, ss, o);
        }
      }
      if (lane == 0) {
        const int eq = mq > 0.f ? ilog2f(mq) : 0;
        const int es = ms > 0.f ? ilog2f(ms) : 0;
        s_scale[h] = eq;
        s_scale[8 + h] = es;
        // q' 2^-(eq+1) < 1 in the key operand; S q' as in the 2-bit kernels.
        s_head[h] = make_float4(pow2i(eq + 1) * a.scale_log2, 0.f, 2.f * pow2i(es) * a.cq * a.scale_log2,
                                -ss * a.cq * a.scale_log2);
      }
    }
    {
      float vmax = 0.f;
      for (int64_t j = tok0 + 4 * tid; j < tok1; j += 4 * MW * 32) {
        const int64_t rec = kv_rec<PAGED>(a, b, kvh, j);   // 4 tokens in a row
        if (PAGED && rec < 0) continue;                    // invalid block: masked
        if (a.nf16) {
          const __half* vr = reinterpret_cast<const __half*>(a.vnorm) + rec;
          if (j + 4 <= tok1) {
            const uint2 w = *reinterpret_cast<const uint2*>(vr);
            const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&w.x));
            const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&w.y));
            vmax = fmaxf(vmax, fmaxf(fmaxf(f0.x, f0.y), fmaxf(f1.x, f1.y)));
          } else {
            for (int64_t k = 0; k < tok1 - j; ++k) vmax = fmaxf(vmax, __half2float(vr[k]));
          }
        } else {
          const float* vr = a.vnorm + rec;
          if (j + 4 <= tok1) {
            const float4 v4 = *reinterpret_cast<const float4*>(vr);
            vmax = fmaxf(vmax, fmaxf(fmaxf(v4.x, v4.y), fmaxf(v4.z, v4.w)));
          } else {
            for (int64_t k = 0; k < tok1 - j; ++k) vmax = fmaxf(vmax, vr[k]);
          }
        }
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
      if (lane == 0) s_vmax[warp] = vmax;
    }
    __syncthreads();
    // ---- query operands: warp w builds key k-steps 2w, 2w+1 and QJL k-steps 2w, 2w+1 ----
    {
      const bool odd_col = (g & 1) != 0;
      auto split = [&](float lo, float hi, bool tail) -> uint32_t {
        const __half2 h = __floats2half2_rn(lo, hi);
        if (!tail) return *reinterpret_cast<const uint32_t*>(&h);
        const float2 f = __half22float2(h);
        return pack_half2((lo - f.x) * 4096.f, (hi - f.y) * 4096.f);
      };
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int s = 2 * warp + k;
        // Key k-step s.  MMA 0: heads 0..3, MMA 1 (G = 8): heads 4..7
        // (column g: head g/2 of its set, fp16 head if g is even, tail if
        // odd); MMA 2: the heads of the query times the centroid tails,
        // column g = head g/2 + 4 (g & 1), fp16 head (empty columns for a
        // missing head).  Words: MMA 0, MMA 1, MMA 2 (G = 8); MMA 0, MMA 2 (G = 4).
        constexpr int NM = G == 8 ? 3 : 2;
        uint32_t fr[6];
#pragma unroll
        for (int mi = 0; mi < NM; ++mi) {
          const int m = (G != 8 && mi == 1) ? 2 : mi;
          const int h = m < 2 ? 4 * m + (g >> 1) : (g >> 1) + 4 * (g & 1);
          const bool tail = m < 2 && odd_col;
          if (h < Gr) {
            const float kq = pow2i(-(s_scale[h] + 1));
            const float* row = a.qr + (qbase + h) * 128 + 32 * t;
            fr[2 * mi] = split(row[2 * s] * kq, row[2 * s + 1] * kq, tail);
            fr[2 * mi + 1] = split(row[16 + 2 * s] * kq, row[16 + 2 * s + 1] * kq, tail);
          } else {
            fr[2 * mi] = fr[2 * mi + 1] = 0u;
          }
        }
        uint32_t* dk = qopk + (s * 32 + lane) * QOPK;
        *reinterpret_cast<uint4*>(dk) = make_uint4(fr[0], fr[1], fr[2], fr[3]);
        if (G == 8) *reinterpret_cast<uint2*>(dk + 4) = make_uint2(fr[4], fr[5]);
        if (QJL) {
          // QJL k-step s: fp16 bit operands as in the 2-bit kernels (registers
          // u = 2s, 2s+1 of the sign word), MMA 0 heads 0..3, MMA 1 heads 4..7.
          uint32_t fq[4] = {0u, 0u, 0u, 0u};
#pragma unroll
          for (int m = 0; m < NJ; ++m) {
            const int h = 4 * m + (g >> 1);
            if (h >= Gr) continue;   // empty columns of a missing head
            const float ks = pow2i(-s_scale[8 + h]);
            const float* row = a.qs + (qbase + h) * 128 + 32 * t;
#pragma unroll
            for (int sl = 0; sl < 2; ++sl) {
              const int u = 2 * s + sl;
              const int elo = 10 + u, ehi = (26 + u) & 31;
              const float inv = bit_inv(bit_pos(u)) * ks;
              fq[2 * m + sl] = split(row[elo] * inv, row[ehi] * inv, odd_col);
            }
          }
          *reinterpret_cast<uint4*>(qopq + (s * 32 + lane) * QOPQ) = make_uint4(fq[0], fq[1], fq[2], fq[3]);
        }
      }
    }
    __syncthreads();
    float4 H[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) H[j] = s_head[4 * j + t];
    const float vmax = fmaxf(fmaxf(s_vmax[0], s_vmax[1]), fmaxf(s_vmax[2], s_vmax[3]));
    // p <= 2^8 and |v| 2^-kv < 2^7 keep p |v| 2^-kv below 2^15.
    const int kv = vmax >= FLT_MIN ? max(ilog2f(vmax) - 6, -120) : -120;
    const float vmul = pow2i(-kv);

    // ---- this warp's tiles: i = warp, warp + 4, ... of the piece ------------------
    const int ntw = nt > warp ? (nt - warp + MW - 1) / MW : 0;
    const int64_t rb = kv_base<PAGED>(a, b, kvh);   // row base (0 when paged)
    const char* kbase = reinterpret_cast<const char*>(a.kcodes + rb * KF::REC);
    // 16-byte chunks of one tile: key codes, QJL words, norms (|k|, gamma, |v|
    // or |k|, |v|), value codes.
    constexpr int NKC = MT * KF::REC / 4;
    constexpr int NQC = QJL ? MT : 0;
    constexpr int NNC = (QJL ? 3 : 2) * 4;
    constexpr int NVC = MT * VF::REC / 4;
    constexpr int NCH = NKC + NQC + NNC + NVC;
    uint32_t bad = 0;   // paged: bit (k % 32) set when the warp's k-th tile has an invalid block id
    auto issue = [&](int k, int stage) {
      const int64_t t0 = tok0 + (int64_t)MT * (warp + MW * k);
      int64_t r = kv_off<PAGED>(a, b, kvh, t0);   // records of tokens t0.. (16 in a row)
      // an invalid block copies nothing: every chunk is zero-filled
      const int64_t tend = (PAGED && r < 0) ? t0 : tok1;
      if (PAGED) {   // the bit of ring tile k is rewritten by every issue (tile k + 32 reuses it)
        bad = (bad & ~(1u << (k & 31))) | ((r < 0 ? 1u : 0u) << (k & 31));
        r = r < 0 ? 0 : r;
      }
      const uint32_t sb = my_s + stage * (uint32_t)sizeof(Stage);
#pragma unroll
      for (int i = 0; i < (NCH + 31) / 32; ++i) {
        const int c = lane + 32 * i;
        if (c < NKC) {                         // key codes
          int tok, part;
          uint32_t dst;
          if (KB == 3) {                       // 16 tokens x 3 chunks
            tok = c / 3;
            part = c % 3;
            dst = part < 2 ? (uint32_t)(offsetof(Stage, k2) + tok * 32 + part * 16)
                           : (uint32_t)(offsetof(Stage, k1) + tok * 16);
          } else {                             // 16 tokens x 4 (8) chunks
            tok = c / (KF::REC / 4);
            part = c % (KF::REC / 4);
            dst = (uint32_t)(offsetof(Stage, k2) + tok * (KF::K2W * 4) + part * 16);
          }
          cp16(sb + dst, kbase + (r + tok) * (KF::REC * 4) + part * 16, t0 + tok < tend);
        } else if (c < NKC + NQC) {            // QJL words: 16 tokens x 1 chunk
          const int tok = c - NKC;
          cp16(sb + offsetof(Stage, q) + tok * 16, a.kqjl + (rb + r + tok) * QW, t0 + tok < tend);
        } else if (c < NKC + NQC + NNC) {      // norms: arrays x 4 chunks of 4 tokens
          const int which = (c - NKC - NQC) >> 2, part = (c - NKC - NQC) & 3;
          const int arr = QJL ? which : (which == 0 ? 0 : 2);   // 0 |k|, 1 gamma, 2 |v|
          const float* base = arr == 0 ? a.knorm : (arr == 1 ? a.krnorm : a.vnorm);
          const uint32_t off = arr == 0 ? offsetof(Stage, kn)
                                        : (arr == 1 ? offsetof(Stage, kr) : offsetof(Stage, vn));
          if (!a.nf16) {
            cp16(sb + off + part * 16, base + rb + r + 4 * part, t0 + 4 * part < tend);
          } else if (part < 2) {   // binary16 norms: 8 tokens per chunk
            cp16(sb + off + part * 16, reinterpret_cast<const __half*>(base) + rb + r + 8 * part,
                 t0 + 8 * part < tend);
          }
        } else if (c < NCH) {                  // value codes: 16 tokens x 4 (3) chunks
          const int cc = c - NKC - NQC - NNC, tok = cc / (VF::REC / 4), part = cc % (VF::REC / 4);
          cp16(sb + offsetof(Stage, v) + tok * (VF::ROW * 4) + part * 16,
               a.vcodes + (rb + r + tok) * VF::REC + part * 4, t0 + tok < tend);
        }
      }
    };
#pragma unroll
    for (int k = 0; k < NS - 1; ++k) {
      if (k < ntw) issue(k, k);
      cp_commit();
    }

    float m_run[NJ], l_part[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      m_run[j] = M_EMPTY;
      l_part[j] = 0.f;
    }
    float o[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;

    for (int k = 0; k < ntw; ++k) {
      if (k + NS - 1 < ntw) issue(k + NS - 1, (k + NS - 1) % NS);
      cp_commit();
      cp_wait<NS - 1>();
      __syncwarp();
      const Stage& st = my[k % NS];
      const int64_t t0 = tok0 + (int64_t)MT * (warp + MW * k);

      // ---- logits: heads t (accH0) and 4 + t (accH1), tails (accL), QJL (acs) ----
      float accH0[4] = {0.f, 0.f, 0.f, 0.f}, accH1[4] = {0.f, 0.f, 0.f, 0.f}, accL[4] = {0.f, 0.f, 0.f, 0.f};
      float acs[NJ][4];
#pragma unroll
      for (int j = 0; j < NJ; ++j) acs[j][0] = acs[j][1] = acs[j][2] = acs[j][3] = 0.f;
      {
        auto kstep = [&](int S, uint2 A0, uint2 A1, uint2 A2, uint2 A3) {
          const uint4 ba = lds128(qopk_lane + S * 32 * QOPK * 4);
          mma16816(accH0, A0.x, A1.x, A2.x, A3.x, ba.x, ba.y);
          if (G == 8) {
            const uint2 bb = lds64(qopk_lane + S * 32 * QOPK * 4 + 16);
            mma16816(accH1, A0.x, A1.x, A2.x, A3.x, ba.z, ba.w);
            mma16816(accL, A0.y, A1.y, A2.y, A3.y, bb.x, bb.y);
          } else {
            mma16816(accL, A0.y, A1.y, A2.y, A3.y, ba.z, ba.w);
          }
        };
        if (KB == 3) {
          const uint2 wg2 = *reinterpret_cast<const uint2*>(&st.k2[g][2 * t]);
          const uint2 wh2 = *reinterpret_cast<const uint2*>(&st.k2[g + 8][2 * t]);
          const uint32_t wg1 = st.k1[g][t], wh1 = st.k1[g + 8][t];
#define TQ_K3STEP(S)                                                                              \
  kstep(S, lds64(klut_lane + klut_off<S, 0>(wg2.x, wg1)), lds64(klut_lane + klut_off<S, 0>(wh2.x, wh1)), \
        lds64(klut_lane + klut_off<S, 16>(wg2.y, wg1)), lds64(klut_lane + klut_off<S, 16>(wh2.y, wh1)));
          TQ_K3STEP(0) TQ_K3STEP(1) TQ_K3STEP(2) TQ_K3STEP(3) TQ_K3STEP(4) TQ_K3STEP(5)
          TQ_K3STEP(6) TQ_K3STEP(7)
#undef TQ_K3STEP
        } else if (KB == 8) {
          // k-step s: bytes 2 (s & 1), +1 of word s >> 1 of the first and of
          // the second 16 coordinates (words 8t + (s >> 1), 8t + 4 + (s >> 1)).
          const uint4 ga = *reinterpret_cast<const uint4*>(&st.k2[g][8 * t]);
          const uint4 gb = *reinterpret_cast<const uint4*>(&st.k2[g][8 * t + 4]);
          const uint4 ha = *reinterpret_cast<const uint4*>(&st.k2[g + 8][8 * t]);
          const uint4 hb = *reinterpret_cast<const uint4*>(&st.k2[g + 8][8 * t + 4]);
#define TQ_K8STEP(S, W)                                                                           \
  kstep(S, k8_pair<2 * ((S) & 1)>(klut_lane, ga.W), k8_pair<2 * ((S) & 1)>(klut_lane, ha.W),     \
        k8_pair<2 * ((S) & 1)>(klut_lane, gb.W), k8_pair<2 * ((S) & 1)>(klut_lane, hb.W));
          TQ_K8STEP(0, x) TQ_K8STEP(1, x) TQ_K8STEP(2, y) TQ_K8STEP(3, y)
          TQ_K8STEP(4, z) TQ_K8STEP(5, z) TQ_K8STEP(6, w) TQ_K8STEP(7, w)
#undef TQ_K8STEP
        } else {
          const uint4 wg = *reinterpret_cast<const uint4*>(&st.k2[g][4 * t]);
          const uint4 wh = *reinterpret_cast<const uint4*>(&st.k2[g + 8][4 * t]);
          // k-step s: byte s & 3 of word s >> 2 (coordinates 32t + 2s, +1) and
          // of word 2 + (s >> 2) (coordinates 32t + 16 + 2s, +1).
#define TQ_K4STEP(S, WA, WB)                                                                      \
  kstep(S, lds64(klut_lane + klut4_off<(S) & 3>(wg.WA)), lds64(klut_lane + klut4_off<(S) & 3>(wh.WA)), \
        lds64(klut_lane + klut4_off<(S) & 3>(wg.WB)), lds64(klut_lane + klut4_off<(S) & 3>(wh.WB)));
          TQ_K4STEP(0, x, z) TQ_K4STEP(1, x, z) TQ_K4STEP(2, x, z) TQ_K4STEP(3, x, z)
          TQ_K4STEP(4, y, w) TQ_K4STEP(5, y, w) TQ_K4STEP(6, y, w) TQ_K4STEP(7, y, w)
#undef TQ_K4STEP
        }
        if (QJL) {
          const Rot4 Q0 = rotations(st.q[g][t]), Q8 = rotations(st.q[g + 8][t]);
#define TQ_QSTEP8(S)                                                                              \
  {                                                                                               \
    const uint4 bq = lds128(qopq_lane + (S) * 32 * QOPQ * 4);                                     \
    const uint32_t x0 = bit_half2<2 * (S)>(Q0), x1 = bit_half2<2 * (S)>(Q8);                       \
    const uint32_t x2 = bit_half2<2 * (S) + 1>(Q0), x3 = bit_half2<2 * (S) + 1>(Q8);              \
    mma16816(acs[0], x0, x1, x2, x3, bq.x, bq.y);                                                 \
    if (NJ == 2) mma16816(acs[NJ - 1], x0, x1, x2, x3, bq.z, bq.w);                               \
  }
          TQ_QSTEP8(0) TQ_QSTEP8(1) TQ_QSTEP8(2) TQ_QSTEP8(3) TQ_QSTEP8(4) TQ_QSTEP8(5)
          TQ_QSTEP8(6) TQ_QSTEP8(7)
#undef TQ_QSTEP8
        }
      }
      const bool tile_ok = !PAGED || !((bad >> (k & 31)) & 1u);
      const bool v0 = tile_ok && t0 + g < tok1, v8 = tile_ok && t0 + g + 8 < tok1;
      auto snorm = [&](const float* arr, int i) {
        return a.nf16 ? __half2float(reinterpret_cast<const __half*>(arr)[i]) : arr[i];
      };
      const float kn0 = snorm(st.kn, g), kn8 = snorm(st.kn, g + 8);
      float sc[NJ][2];
      {
        // <q', c> of head t (rows g, g+8) and head 4 + t: head products plus
        // (head x tail + tail x head) / 2^12.
        float lm[NJ][2];
        lm[0][0] = accH0[0] + (accH0[1] + accL[0]) * (1.f / 4096.f);
        lm[0][1] = accH0[2] + (accH0[3] + accL[2]) * (1.f / 4096.f);
        if (NJ == 2) {
          lm[NJ - 1][0] = accH1[0] + (accH1[1] + accL[1]) * (1.f / 4096.f);
          lm[NJ - 1][1] = accH1[2] + (accH1[3] + accL[3]) * (1.f / 4096.f);
        }
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
          const bool hv = j > 0 || hv0;
          if (QJL) {
            const float kr0 = st.kr[g], kr8 = st.kr[g + 8];
            const float qj0 = fmaf(acs[j][1], 1.f / 4096.f, acs[j][0]);
            const float qj8 = fmaf(acs[j][3], 1.f / 4096.f, acs[j][2]);
            sc[j][0] = (hv && v0) ? fmaf(kn0 * lm[j][0], H[j].x, kr0 * fmaf(qj0, H[j].z, H[j].w)) : -INFINITY;
            sc[j][1] = (hv && v8) ? fmaf(kn8 * lm[j][1], H[j].x, kr8 * fmaf(qj8, H[j].z, H[j].w)) : -INFINITY;
          } else {
            sc[j][0] = (hv && v0) ? kn0 * lm[j][0] * H[j].x : -INFINITY;
            sc[j][1] = (hv && v8) ? kn8 * lm[j][1] * H[j].x : -INFINITY;
          }
        }
      }

      // ---- online softmax, heads t (and 4 + t) --------------------------------------
      float loc[NJ];
      bool grow = false;
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        loc[j] = fmaxf(sc[j][0], sc[j][1]);
        grow = grow || loc[j] > m_run[j] + LAZY_TAU;
      }
      if (__any_sync(0xffffffffu, grow)) {
        float al[NJ];
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
          float tm = loc[j];
#pragma unroll
          for (int o_ = 4; o_ <= 16; o_ <<= 1) tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, o_));
          const float mn = fmaxf(m_run[j], tm);
          al[j] = mn == -INFINITY ? 1.f : ex2f(m_run[j] - mn);   // -inf only for a missing head
          m_run[j] = mn;
          l_part[j] *= al[j];
        }
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          o[mt][0] *= al[0];
          o[mt][2] *= al[0];
          if (NJ == 2) {
            o[mt][1] *= al[NJ - 1];
            o[mt][3] *= al[NJ - 1];
          }
        }
      }
      float p[2][2] = {{0.f, 0.f}, {0.f, 0.f}};   // [head set][row g, g + 8]
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const bool hv = j > 0 || hv0;
        p[j][0] = hv ? ex2f(sc[j][0] - m_run[j]) : 0.f;
        p[j][1] = hv ? ex2f(sc[j][1] - m_run[j]) : 0.f;
        l_part[j] += p[j][0] + p[j][1];
      }
      // A 16-byte norm copy may reach past the row's end: those norms are not data.
      const float w0s = v0 ? snorm(st.vn, g) * vmul : 0.f, w8s = v8 ? snorm(st.vn, g + 8) * vmul : 0.f;
      const uint32_t pb0 = movtrans(pack_half2(p[0][0] * w0s, p[1][0] * w0s));
      const uint32_t pb1 = movtrans(pack_half2(p[0][1] * w8s, p[1][1] * w8s));
      if constexpr (VB == 4)
        value_tile(o, st.v, pb0, pb1, lut_lane, g, t);
      else
        value_tile3(o, st.v, pb0, pb1, lut_lane, g, t);
      __syncwarp();
    }
    cp_wait<0>();
    __syncwarp();

    // ---- this warp's partial of the piece (heads t and 4 + t) --------------------------
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      l_part[j] += __shfl_xor_sync(0xffffffffu, l_part[j], 4);
      l_part[j] += __shfl_xor_sync(0xffffffffu, l_part[j], 8);
      l_part[j] += __shfl_xor_sync(0xffffffffu, l_part[j], 16);
    }
    const float vback = pow2i(kv);
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      if (4 * j + t >= Gr) continue;   // a missing head
      float* pp = a.part + (slot * Gr + 4 * j + t) * (128 + 2);
      if (g == 0) {
        pp[0] = m_run[j];
        pp[1] = l_part[j];
      }
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        pp[2 + 16 * g + mt] = o[mt][j] * vback;
        pp[2 + 16 * g + 8 + mt] = o[mt][2 + j] * vback;
      }
    }
  }
}

}  // namespace

bool attn_lut_supported(const tq_ctx* c, const AttnArgs& a) {
  if (c->d != D || (a.G != 1 && a.G != 2 && a.G != 4 && a.G != 8)) return false;
  const bool k3q = c->bk_lm == 3 && c->qjl_m == 128 && c->bits_v == 4;
  const bool mse = c->qjl_m == 0 && ((c->bk_lm == 3 && (c->bits_v == 4 || c->bits_v == 3)) ||
                                     ((c->bk_lm == 4 || c->bk_lm == 8) && c->bits_v == 4));
  if (!k3q && !mse) return false;
  if (a.max_T % 4 != 0) return false;
  if (c->norm_f16 && (k3q || a.max_T % 8 != 0)) return false;   // binary16 norms: 8-token chunks
  const uintptr_t al = reinterpret_cast<uintptr_t>(a.kcodes) | reinterpret_cast<uintptr_t>(a.knorm) |
                       reinterpret_cast<uintptr_t>(a.vcodes) | reinterpret_cast<uintptr_t>(a.vnorm) |
                       (k3q ? reinterpret_cast<uintptr_t>(a.kqjl) | reinterpret_cast<uintptr_t>(a.krnorm) : 0);
  return (al & 15) == 0;
}

template <int KB, bool QJL, int VB>
static void lut_launch(const AttnArgs& a, unsigned blocks, cudaStream_t s) {
  constexpr size_t sm = smem_lut<KB, QJL, VB>();
  const bool pg = a.block_table != nullptr;
  if (a.G == 8) {
    if (pg) k_attn_lut<true, KB, QJL, 8, VB><<<blocks, MW * 32, sm, s>>>(a);
    else k_attn_lut<false, KB, QJL, 8, VB><<<blocks, MW * 32, sm, s>>>(a);
  } else if (a.G == 4) {
    if (pg) k_attn_lut<true, KB, QJL, 4, VB><<<blocks, MW * 32, sm, s>>>(a);
    else k_attn_lut<false, KB, QJL, 4, VB><<<blocks, MW * 32, sm, s>>>(a);
  } else {   // groups 1 and 2
    if (pg) k_attn_lut<true, KB, QJL, 2, VB><<<blocks, MW * 32, sm, s>>>(a);
    else k_attn_lut<false, KB, QJL, 2, VB><<<blocks, MW * 32, sm, s>>>(a);
  }
}

cudaError_t launch_attn_lut(const tq_ctx* c, const AttnArgs& a_in, float* out, cudaStream_t s) {
  AttnArgs a = a_in;
  if (!a.tiles || (a.G != 1 && a.G != 2 && a.G != 4 && a.G != 8)) return cudaErrorInvalidValue;
  // CTA-owned ranges of at least four tiles per warp; two CTAs per SM (three
  // for 3-bit keys, whose tables and two-stage rings fit three times).
  const int64_t wmax = (int64_t)a.B * a.Hkv * ((a.max_T + MT - 1) / MT);
  const int64_t per_sm = c->bk_lm == 3 ? 3 : 2;
  int64_t blocks = (wmax + 4 * MW - 1) / (4 * MW);
  blocks = blocks < 1 ? 1 : (blocks > (int64_t)c->sms * per_sm ? (int64_t)c->sms * per_sm : blocks);
  a.nw = (int)blocks;
  a.wpu = MW;
  const unsigned nb = (unsigned)blocks;
  const bool q = c->qjl_m > 0;
  if (q && c->bk_lm == 3 && c->bits_v == 4)
    lut_launch<3, true, 4>(a, nb, s);
  else if (!q && c->bk_lm == 3 && c->bits_v == 4)
    lut_launch<3, false, 4>(a, nb, s);
  else if (!q && c->bk_lm == 4 && c->bits_v == 4)
    lut_launch<4, false, 4>(a, nb, s);
  else if (!q && c->bk_lm == 3 && c->bits_v == 3)
    lut_launch<3, false, 3>(a, nb, s);
  else if (!q && c->bk_lm == 8 && c->bits_v == 4)
    lut_launch<8, false, 4>(a, nb, s);
  else
    return cudaErrorInvalidValue;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_attn_merge(c, a, out, s);
}

template <int KB, bool QJL, int VB>
static cudaError_t lut_configure() {
  const cudaFuncAttribute ms = cudaFuncAttributeMaxDynamicSharedMemorySize;
  constexpr int sm = (int)smem_lut<KB, QJL, VB>();
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(k_attn_lut<false, KB, QJL, 8, VB>, ms, sm)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(k_attn_lut<true, KB, QJL, 8, VB>, ms, sm)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(k_attn_lut<false, KB, QJL, 4, VB>, ms, sm)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(k_attn_lut<true, KB, QJL, 4, VB>, ms, sm)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(k_attn_lut<false, KB, QJL, 2, VB>, ms, sm)) != cudaSuccess) return e;
  return cudaFuncSetAttribute(k_attn_lut<true, KB, QJL, 2, VB>, ms, sm);
}

cudaError_t configure_attn_lut() {
  cudaError_t e;
  if ((e = lut_configure<3, true, 4>()) != cudaSuccess) return e;
  if ((e = lut_configure<3, false, 4>()) != cudaSuccess) return e;
  if ((e = lut_configure<4, false, 4>()) != cudaSuccess) return e;
  if ((e = lut_configure<3, false, 3>()) != cudaSuccess) return e;
  return lut_configure<8, false, 4>();
}

}  // namespace tqk
