// Decode attention from packed 2-bit keys with the key product on int8
// tensor-core MMAs (sm_100a).
//
// For every query head h of a KV group of sequence b this computes the softmax
// state over a piece of the context ("What is TurboQuant?", "How TurboQuant
// works", closing paragraph: the logits come straight from the compressed
// indices; "How to implement" part 1: the query is rotated once and dotted
// with centroid values):
//   l_i  = |k_i| <q', c_k[idx_i]> + sqrt(pi/2)/m * gamma_i <S q', sigma_i>
//   s_i  = scale * l_i,   m = max s,   l = sum exp(s - m),
//   o    = sum exp(s_i - m) |v_i| c_v[vidx_i]          (rotated domain)
// The merge kernel combines the pieces by log-sum-exp and applies Pi^T once.
//
// Format: d = 128, keys 2 Lloyd-Max bits + 128 QJL rows, values 4 bits, GQA
// group 1, 2 or 4.  The 16-token tiles of all (sequence, kv head) rows are
// split into balanced contiguous ranges, one per warp; a warp streams its
// tiles through its own cp.async ring and keeps an online softmax.
//
// Key product: mma.sync m16n8k32 with u8 A and s8 B, int32 accumulation.
// A symmetric 2-bit codebook is affine in the index bits (c[i0 + 2 i1] =
// c0 + w0 i0 + w1 i1) and <s, sigma> = 2 <s, bit> - sum s, so both logit
// terms are sums of query terms over the set code bits.  The A operand is the
// code word itself, masked: word & (0x01010101 << p) holds bits p, p+8, p+16,
// p+24 as bytes of value 2^p, one logic instruction per four operand bytes.
// The B operand (built once per query by the pre-rotation kernel) holds, for
// each code-bit position, round(2^(S-p) w q') as four balanced signed-byte
// digits in four columns, so the products are exact integers and the limbs
// recombine in fp32 to ~24 bits of the query.  Two N tiles (8 columns each)
// carry four heads x four digits; 8 k-steps cover the 256 key bits and 4 the
// 128 QJL bits: 24 MMAs per tile.
//
// Values: mma.sync m16n8k16 (fp16), A = dequantized values (16 dims x 16
// tokens, from a per-lane 256-entry half2 table of code pairs), B = p |v|.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cmath>

#include "tq_attn_common.cuh"
#include "tq_internal.h"

namespace tqk {
namespace {

constexpr int MWI = 12;    // warps per CTA (one CTA per SM: the value table is shared)
constexpr int NSI = 5;     // pipeline stages per warp
constexpr int KWI = 8;     // key code words per token (2-bit fields)
constexpr int KROW = 12;   // padded key row in shared memory: the 32-bit loads of words t and t + 4
                           // by the lanes (g, t) of a warp hit 32 distinct banks
struct StageI {
  uint32_t k[MT][KROW];    // 768 B
  uint32_t q[MT][QW];      // 256 B
  float kn[MT];            // 64 B
  float kr[MT];            // 64 B
  float vn[MT];            // 64 B
  uint32_t pad_[4];        // keep v 16-byte aligned
  uint32_t v[MT][VROW];    // 1280 B
};
static_assert(sizeof(StageI) % 16 == 0, "stage alignment");
static_assert(offsetof(StageI, v) % 16 == 0, "value rows alignment");

constexpr size_t SMEM_I8 = (size_t)WLUT_BYTES + (size_t)MWI * NSI * sizeof(StageI);

__device__ __forceinline__ void imma16832(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Four int32 limb sums (digits 0..3 of one head and token) as one fp32 value:
// lo = d0 + 256 d1 and hi = d2 + 256 d3 are exact in int32 (|d| < 2^20).
__device__ __forceinline__ float limbs(int d0, int d1, int d2, int d3) {
  const int lo = d0 + d1 * 256, hi = d2 + d3 * 256;
  return fmaf((float)hi, 65536.f, (float)lo);
}

// ---------------------------------------------------------------------------
// Tile ranges: the 16-token tiles of all (sequence, kv head) rows form one
// sequence of W tiles (row-major over b, kv head, tile; a.tiles[b] counts the
// tiles of rows before sequence b).  Warp w takes [w W / N, (w + 1) W / N),
// N = min(warps, W), and writes one partial (m, l, o) per head and row piece
// to slot w + b Hkv + kv head (unique: consecutive rows' pieces come from
// non-decreasing warps); the merge finds a row's slots from the same
// arithmetic.
//
// Softmax: the running maximum moves only when a tile exceeds it by more than
// 2^8 (exp2 units), so probabilities stay below 2^8; the value norms of a
// piece are scaled once from the piece's largest norm so that p |v| stays
// below 2^15 in fp16.
//
// Paged caches: a tile whose block id is outside [0, num_blocks) is masked
// (zero-filled copies, no weight); the issuing warp keeps one bit per ring
// position.
// ---------------------------------------------------------------------------
template <int G, bool PAGED>
__global__ void __launch_bounds__(MWI * 32, 1) k_attn_i8(AttnArgs a) {
  static_assert(G <= 4, "four heads per N tile pair");
  extern __shared__ __align__(16) unsigned char smem[];
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem);
  StageI* stages = reinterpret_cast<StageI*>(smem + (size_t)WLUT_BYTES);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;

  build_value_wlut(lut, a.cv, tid, MWI * 32);
  __syncthreads();   // the only block-wide barrier: warps run independently below

  const int64_t* P = a.tiles;
  const int64_t W = P[a.B];
  const int64_t NW = min((int64_t)gridDim.x * MWI, W);
  const int64_t wid = (int64_t)blockIdx.x * MWI + warp;
  if (wid >= NW) return;
  int64_t x = wid * W / NW;
  const int64_t x1 = (wid + 1) * W / NW;
  int b = locate_sequence(P, a.B, x);

  const uint32_t lut_s = (uint32_t)__cvta_generic_to_shared(lut), lane4 = 4u * lane;
  StageI* my = stages + warp * NSI;
  const uint32_t my_s = (uint32_t)__cvta_generic_to_shared(my);
  const bool own_head = t < G;   // accumulator columns 2t, 2t+1 belong to head t
  const bool col_ok = (g >> 1) < G;   // this lane's B column belongs to a head of the group

  while (x < x1) {
    while (P[b + 1] <= x) ++b;
    const int64_t tb = (P[b + 1] - P[b]) / a.Hkv;
    const int64_t rel = x - P[b];
    const int kvh = (int)(rel / tb);
    const int64_t tt = rel - (int64_t)kvh * tb;
    const int64_t te = min(tb, tt + (x1 - x));
    const int nt = (int)(te - tt);
    const int64_t slot = wid + (int64_t)b * a.Hkv + kvh;
    x += nt;

    const int64_t len = min((int64_t)max(a.seq_lens[b], 0), a.max_T);
    const int64_t tok0 = tt * MT;
    const int64_t tok1 = min(te * MT, len);

    // ---- cp.async ring: lane assignment fixed for the piece -------------------
    // Chunk 0 = key codes (token lane/2, half lane%2), chunks 1-2 = value codes,
    // chunk 3 = QJL words (lanes 0-15) or norms (lanes 16-27).
    const int64_t rb = kv_base<PAGED>(a, b, kvh);   // row base (0 when paged)
    const char* p0 = reinterpret_cast<const char*>(a.kcodes + rb * KWI) + lane * 16;
    const char* p1 = reinterpret_cast<const char*>(a.vcodes + rb * VW) + lane * 16;
    const char* p2 = p1 + 8 * 64;
    const char* p3;
    int stride3, tok3;
    uint32_t d3;
    if (lane < 16) {
      p3 = reinterpret_cast<const char*>(a.kqjl + rb * QW) + lane * 16;
      stride3 = 16; tok3 = lane; d3 = offsetof(StageI, q) + lane * 16;
    } else if (lane < 28) {
      const int which = (lane - 16) >> 2, part = (lane - 16) & 3;
      const float* base = which == 0 ? a.knorm : (which == 1 ? a.krnorm : a.vnorm);
      p3 = reinterpret_cast<const char*>(base + rb) + part * 16;
      stride3 = 4; tok3 = 4 * part;
      d3 = (which == 0 ? offsetof(StageI, kn) : (which == 1 ? offsetof(StageI, kr) : offsetof(StageI, vn))) +
           part * 16;
    } else {
      p3 = nullptr; stride3 = 0; tok3 = 1 << 30; d3 = 0;
    }
    const uint32_t d0 = offsetof(StageI, k) + (lane >> 1) * (KROW * 4) + (lane & 1) * 16;
    const uint32_t d1 = offsetof(StageI, v) + (lane >> 2) * (VROW * 4) + (lane & 3) * 16;
    const uint32_t d2 = d1 + 8 * (VROW * 4);
    uint32_t bad = 0;   // paged: bit (i % 32) set when tile i's block id is invalid
    auto issue = [&](int i, int stage) {
      const int64_t t0 = tok0 + (int64_t)MT * i;
      const uint32_t sb = my_s + stage * (uint32_t)sizeof(StageI);
      int64_t r = kv_off<PAGED>(a, b, kvh, t0);   // records of tokens t0.. (16 in a row)
      if (PAGED) {   // the bit of tile i is rewritten by every issue (tile i + 32 reuses it)
        bad = (bad & ~(1u << (i & 31))) | ((r < 0 ? 1u : 0u) << (i & 31));
      }
      if (PAGED && r < 0) {   // invalid block: nothing copied, the tile is masked
        r = 0;
      } else if (t0 + MT <= tok1) {   // a full tile: no predicates
        cp16(sb + d0, p0 + r * 32, true);
        cp16(sb + d1, p1 + r * 64, true);
        cp16(sb + d2, p2 + r * 64, true);
        if (lane < 28) cp16(sb + d3, p3 + r * stride3, true);
        return;
      }
      const bool ok = !(PAGED && ((bad >> (i & 31)) & 1u));
      cp16(sb + d0, p0 + r * 32, ok && t0 + (lane >> 1) < tok1);
      cp16(sb + d1, p1 + r * 64, ok && t0 + (lane >> 2) < tok1);
      cp16(sb + d2, p2 + r * 64, ok && t0 + 8 + (lane >> 2) < tok1);
      if (lane < 28) cp16(sb + d3, p3 + r * stride3, ok && t0 + tok3 < tok1);
    };
#pragma unroll
    for (int i = 0; i < NSI - 1; ++i) {
      if (i < nt) issue(i, i);
      cp_commit();
    }

    // ---- query operands: int8 digit images and head constants ----------------
    const unsigned char* img = a.qimg + ((int64_t)b * a.Hkv + kvh) * (int64_t)kQopBytes;
    uint4 bq[12];
#pragma unroll
    for (int k = 0; k < 12; ++k) {
      const uint4 v = reinterpret_cast<const uint4*>(img)[k * 32 + lane];
      bq[k] = col_ok ? v : make_uint4(0u, 0u, 0u, 0u);
    }
    const float4 H = own_head ? reinterpret_cast<const float4*>(img + kQopRegs * 32 * 4)[t]
                              : make_float4(0.f, 0.f, 0.f, 0.f);

    // ---- value-norm scale of the piece ---------------------------------------
    float vmax = 0.f;
    {
      for (int64_t j = tok0 + 4 * lane; j < tok1; j += 128) {
        const int64_t rec = kv_rec<PAGED>(a, b, kvh, j);   // 4 tokens in a row
        if (PAGED && rec < 0) continue;
        const float* vr = a.vnorm + rec;
        if (j + 4 <= tok1) {
          const float4 v4 = *reinterpret_cast<const float4*>(vr);
          vmax = fmaxf(vmax, fmaxf(fmaxf(v4.x, v4.y), fmaxf(v4.z, v4.w)));
        } else {
          for (int64_t k = 0; k < tok1 - j; ++k) vmax = fmaxf(vmax, vr[k]);
        }
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    }
    // p <= 2^8 and |v| 2^-kv < 2^7 keep p |v| 2^-kv below 2^15.
    const int kv = vmax >= FLT_MIN ? max(ilog2f(vmax) - 6, -120) : -120;
    const float vmul = pow2i(-kv);

    float m_run = own_head ? M_EMPTY : 0.f;
    float l_part = 0.f;
    float o[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;

    for (int i = 0; i < nt; ++i) {
      if (i + NSI - 1 < nt) issue(i + NSI - 1, (i + NSI - 1) % NSI);
      cp_commit();
      cp_wait<NSI - 1>();
      __syncwarp();
      const StageI& st = my[i % NSI];
      const int64_t t0 = tok0 + (int64_t)MT * i;

      // ---- logits -----------------------------------------------------------
      int ak0[4] = {0, 0, 0, 0}, ak1[4] = {0, 0, 0, 0}, aq0[4] = {0, 0, 0, 0}, aq1[4] = {0, 0, 0, 0};
      {
        const uint32_t kw0 = st.k[g][t], kw1 = st.k[g][t + 4];
        const uint32_t kx0 = st.k[g + 8][t], kx1 = st.k[g + 8][t + 4];
        const uint32_t qw = st.q[g][t], qx = st.q[g + 8][t];
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const uint32_t msk = 0x01010101u << s;
          const uint32_t a0 = kw0 & msk, a1 = kx0 & msk, a2 = kw1 & msk, a3 = kx1 & msk;
          imma16832(ak0, a0, a1, a2, a3, bq[s].x, bq[s].y);
          imma16832(ak1, a0, a1, a2, a3, bq[s].z, bq[s].w);
          if (s < 4) {
            const uint32_t m0 = 0x01010101u << (2 * s), m1 = m0 << 1;
            const uint32_t c0 = qw & m0, c1 = qx & m0, c2 = qw & m1, c3 = qx & m1;
            imma16832(aq0, c0, c1, c2, c3, bq[8 + s].x, bq[8 + s].y);
            imma16832(aq1, c0, c1, c2, c3, bq[8 + s].z, bq[8 + s].w);
          }
        }
      }
      // Rows g and g + 8 are tokens; N tile 0 holds digits 0, 1 and N tile 1
      // digits 2, 3 of head t in columns 2t, 2t + 1.
      const bool tile_ok = !PAGED || !((bad >> (i & 31)) & 1u);
      const bool v0 = tile_ok && t0 + g < tok1, v8 = tile_ok && t0 + g + 8 < tok1;
      const float lk0 = limbs(ak0[0], ak0[1], ak1[0], ak1[1]), lk8 = limbs(ak0[2], ak0[3], ak1[2], ak1[3]);
      const float lq0 = limbs(aq0[0], aq0[1], aq1[0], aq1[1]), lq8 = limbs(aq0[2], aq0[3], aq1[2], aq1[3]);
      const float sc0 = (own_head && v0) ? fmaf(st.kn[g], fmaf(lk0, H.x, H.y), st.kr[g] * fmaf(lq0, H.z, H.w))
                                         : -INFINITY;
      const float sc1 = (own_head && v8)
                            ? fmaf(st.kn[g + 8], fmaf(lk8, H.x, H.y), st.kr[g + 8] * fmaf(lq8, H.z, H.w))
                            : -INFINITY;

      // ---- online softmax, head t ---------------------------------------------
      const float loc = fmaxf(sc0, sc1);
      if (__any_sync(0xffffffffu, loc > m_run + LAZY_TAU)) {
        float tmax = loc;
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 4));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 8));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
        const float mnew = fmaxf(m_run, tmax);
        const float alpha = ex2f(m_run - mnew);   // 0 on the first update, 1 if unchanged
        m_run = mnew;
        l_part *= alpha;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          o[mt][0] *= alpha;
          o[mt][2] *= alpha;
        }
      }
      const float p0 = ex2f(sc0 - m_run), p1 = ex2f(sc1 - m_run);
      l_part += p0 + p1;
      // P tile (16 tokens x 8 columns): column 2t = head t, odd columns zero.
      // A 16-byte norm copy may reach past the row's end: those norms are not data.
      const float vn0 = v0 ? st.vn[g] : 0.f, vn8 = v8 ? st.vn[g + 8] : 0.f;
      const uint32_t pb0 = movtrans(pack_half2(p0 * (vn0 * vmul), 0.f));
      const uint32_t pb1 = movtrans(pack_half2(p1 * (vn8 * vmul), 0.f));

      value_tile_w(o, st.v, pb0, pb1, lut_s, lane4, g, t);
      __syncwarp();
    }
    cp_wait<0>();
    __syncwarp();   // the next piece's ring refills stages this one read

    // ---- partial of the piece ------------------------------------------------
    l_part += __shfl_xor_sync(0xffffffffu, l_part, 4);
    l_part += __shfl_xor_sync(0xffffffffu, l_part, 8);
    l_part += __shfl_xor_sync(0xffffffffu, l_part, 16);
    if (own_head) {
      float* pp = a.part + (slot * G + t) * (128 + 2);
      const float vback = pow2i(kv);
      if (g == 0) {
        pp[0] = m_run;
        pp[1] = l_part;
      }
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        pp[2 + 16 * g + mt] = o[mt][0] * vback;
        pp[2 + 16 * g + 8 + mt] = o[mt][2] * vback;
      }
    }
  }
}

}  // namespace

bool attn_i8_supported(const tq_ctx* c, const AttnArgs& a) {
  if (c->norm_f16) return false;   // QJL formats keep fp32 norms
  if (c->d != D || c->bk_lm != 2 || c->bits_v != 4 || c->qjl_m != 128) return false;
  if (!(a.G == 1 || a.G == 2 || a.G == 4)) return false;
  if (a.max_T % 4 != 0) return false;
  const uintptr_t al = reinterpret_cast<uintptr_t>(a.kcodes) | reinterpret_cast<uintptr_t>(a.kqjl) |
                       reinterpret_cast<uintptr_t>(a.knorm) | reinterpret_cast<uintptr_t>(a.krnorm) |
                       reinterpret_cast<uintptr_t>(a.vcodes) | reinterpret_cast<uintptr_t>(a.vnorm);
  return (al & 15) == 0;
}

QopPlan attn_i8_qop(const tq_ctx* c, const AttnArgs& a, unsigned char* img) {
  QopPlan q{};
  q.img = img;
  q.Hq = a.Hq;
  q.G = a.G;
  q.scale_log2 = a.scale_log2;
  q.cq = a.cq;
  // The fp32 roundings of the key centroids, as in the device tables.
  q.c0 = (float)c->ck[0];
  q.c1 = (float)c->ck[1];
  q.c2 = (float)c->ck[2];
  return q;
}

cudaError_t launch_attn_i8(const tq_ctx* c, const AttnArgs& a_in, float* out, cudaStream_t s) {
  AttnArgs a = a_in;
  if (!a.tiles || !a.qimg) return cudaErrorInvalidValue;
  // One CTA of twelve warps per SM (at least four tiles per warp); the
  // kernel trims the warp count to the real tile count.
  const int64_t wmax = (int64_t)a.B * a.Hkv * ((a.max_T + MT - 1) / MT);
  int64_t blocks = (wmax + 4 * MWI - 1) / (4 * MWI);
  blocks = blocks < 1 ? 1 : (blocks > (int64_t)c->sms ? (int64_t)c->sms : blocks);
  a.nw = (int)(blocks * MWI);
  a.wpu = 1;
  const bool paged = a.block_table != nullptr;
  switch (a.G * 2 + (paged ? 1 : 0)) {
    case 2: k_attn_i8<1, false><<<(unsigned)blocks, MWI * 32, SMEM_I8, s>>>(a); break;
    case 3: k_attn_i8<1, true><<<(unsigned)blocks, MWI * 32, SMEM_I8, s>>>(a); break;
    case 4: k_attn_i8<2, false><<<(unsigned)blocks, MWI * 32, SMEM_I8, s>>>(a); break;
    case 5: k_attn_i8<2, true><<<(unsigned)blocks, MWI * 32, SMEM_I8, s>>>(a); break;
    case 8: k_attn_i8<4, false><<<(unsigned)blocks, MWI * 32, SMEM_I8, s>>>(a); break;
    case 9: k_attn_i8<4, true><<<(unsigned)blocks, MWI * 32, SMEM_I8, s>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_attn_merge(c, a, out, s);
}

cudaError_t configure_attn_i8() {
  const int b = (int)SMEM_I8;
  const cudaFuncAttribute ms = cudaFuncAttributeMaxDynamicSharedMemorySize;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(k_attn_i8<1, false>, ms, b))) return e;
  if ((e = cudaFuncSetAttribute(k_attn_i8<1, true>, ms, b))) return e;
  if ((e = cudaFuncSetAttribute(k_attn_i8<2, false>, ms, b))) return e;
  if ((e = cudaFuncSetAttribute(k_attn_i8<2, true>, ms, b))) return e;
  if ((e = cudaFuncSetAttribute(k_attn_i8<4, false>, ms, b))) return e;
  return cudaFuncSetAttribute(k_attn_i8<4, true>, ms, b);
}

}  // namespace tqk
