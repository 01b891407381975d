// Decode attention from packed codes on the tensor cores (sm_100a).
//
// Computes, for every query head h of a KV group of sequence b, the softmax
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
// group size 8 (groups of at most four heads take the int8 key product of
// tq_attn_i8.cu).  Work is split into balanced contiguous ranges of 16-token
// tiles over all (sequence, kv head) rows.  Per tile:
//  * logits: mma.sync m16n8k16, A = key code bits as exact fp16 powers of two
//    (16 tokens x 16 bit-planes), B = pre-rotated query (fp16 head and tail
//    per head), fp32 accumulate; the centroid values enter through an affine
//    identity in fp32.  A second product takes the QJL sign bits against S q'.
//  * the 16x8 probability tile is transposed into the B operand of the value
//    product with movmatrix.
//  * values: mma.sync m16n8k16, A = dequantized values (16 dims x 16 tokens),
//    B = p * |v| (16 tokens x 8 columns).  A 4-bit code pair (two tokens, one
//    dim) indexes a 256-entry half2 table in shared memory, one copy per
//    lane so that every lookup of a warp hits 32 different banks.
// The head dimension is permuted inside the tiles (a thread owns contiguous
// code words); the permutation is undone when the partials are written.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cmath>

#include "tq_attn_common.cuh"
#include "tq_internal.h"

namespace tqk {
namespace {

constexpr int KW = 8;           // key code words per token (2-bit fields)
struct Stage {
  uint32_t k[MT][KW];           // 512 B
  uint32_t q[MT][QW];           // 256 B
  float kn[MT];                 // 64 B
  float kr[MT];                 // 64 B
  float vn[MT];                 // 64 B
  uint32_t pad_[4];             // keep v 16-byte aligned
  uint32_t v[MT][VROW];         // 1280 B
};
static_assert(sizeof(Stage) % 16 == 0, "stage alignment");



// ---------------------------------------------------------------------------
// Group size 8.  Eight heads with fp16 head and tail columns need sixteen B
// columns (two MMAs per k-step), and the query operands of all k-steps would
// take 96 registers per thread; they live in shared memory instead, built once
// per row piece by the whole CTA.  So the CTA, not the warp, owns a tile range
// ([c W / N, (c + 1) W / N), N = min(CTAs, W)); tile i of a row piece goes to
// warp i mod 4, and every warp writes its own partial per piece (an empty one,
// m = -inf, if it had no tile), to slot 4 (c + b Hkv + kv head) + warp.
//
// Thread (g, t) owns heads t and 4 + t: the first MMA of a k-step carries
// heads 0..3 (columns 2h, 2h+1 = fp16 head, tail), the second heads 4..7.
// In the value product, column 2t of P carries head t and column 2t+1 head
// 4 + t.
// ---------------------------------------------------------------------------
constexpr int NST8 = 3;                       // pipeline stages per warp
constexpr int QOP_STEPS = 24;                 // 16 key k-steps + 8 QJL k-steps
constexpr size_t SMEM8_BYTES = (size_t)LUT_WORDS * 4 + (size_t)MW * NST8 * sizeof(Stage) +
                               (size_t)QOP_STEPS * 32 * 16 + 8 * 16 + MW * 4 + 16 * 4;

template <bool PAGED>
__global__ void __launch_bounds__(MW * 32, 3) k_attn_seg8(AttnArgs a) {
  constexpr int G = 8;
  extern __shared__ __align__(16) unsigned char smem[];
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem);
  Stage* stages = reinterpret_cast<Stage*>(smem + (size_t)LUT_WORDS * 4);
  uint32_t* qop = reinterpret_cast<uint32_t*>(smem + (size_t)LUT_WORDS * 4 +
                                              (size_t)MW * NST8 * sizeof(Stage));   // [24][32][4]
  float4* s_head = reinterpret_cast<float4*>(qop + QOP_STEPS * 32 * 4);           // [8] KA, KB, QA, QB
  float* s_vmax = reinterpret_cast<float*>(s_head + 8);                             // [MW]
  int* s_scale = reinterpret_cast<int*>(s_vmax + MW);                               // [16] q', S q' exponents

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;

  build_value_lut(lut, a.cv, tid, MW * 32);
  __syncthreads();

  const int64_t* P = a.tiles;
  const int64_t W = P[a.B];
  const int64_t NC = min((int64_t)gridDim.x, W);
  const int64_t cta = blockIdx.x;
  if (cta >= NC) return;   // uniform over the CTA
  int64_t x = cta * W / NC;
  const int64_t x1 = (cta + 1) * W / NC;
  int b = locate_sequence(P, a.B, x);

  const float c0 = a.ck[0], w0 = a.ck[1] - a.ck[0], w1 = a.ck[2] - a.ck[0];
  const int ew = ilog2f(fmaxf(fabsf(w0), fabsf(w1)));
  const uint32_t lut_lane = (uint32_t)__cvta_generic_to_shared(lut) + lane * 4;
  const uint32_t qop_lane = (uint32_t)__cvta_generic_to_shared(qop) + lane * 16;
  Stage* my = stages + warp * NST8;
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
    const int64_t qbase = (int64_t)b * a.Hq + (int64_t)kvh * G;

    __syncthreads();   // the previous piece's readers of qop / s_head are done
    // ---- per-head operand scales (warp w: heads 2w, 2w+1) and value-norm max ----
#pragma unroll
    for (int hsel = 0; hsel < 2; ++hsel) {
      const int h = 2 * warp + hsel;
      const float4 q4 = reinterpret_cast<const float4*>(a.qr + (qbase + h) * 128)[lane];
      const float4 s4 = reinterpret_cast<const float4*>(a.qs + (qbase + h) * 128)[lane];
      float mq = fmaxf(fmaxf(fabsf(q4.x), fabsf(q4.y)), fmaxf(fabsf(q4.z), fabsf(q4.w)));
      float ms = fmaxf(fmaxf(fabsf(s4.x), fabsf(s4.y)), fmaxf(fabsf(s4.z), fabsf(s4.w)));
      float sq = (q4.x + q4.y) + (q4.z + q4.w), ss = (s4.x + s4.y) + (s4.z + s4.w);
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        mq = fmaxf(mq, __shfl_xor_sync(0xffffffffu, mq, o));
        ms = fmaxf(ms, __shfl_xor_sync(0xffffffffu, ms, o));
        sq += __shfl_xor_sync(0xffffffffu, sq, o);
        ss += __shfl_xor_sync(0xffffffffu, ss, o);
      }
      if (lane == 0) {
        const int eq = mq > 0.f ? ilog2f(mq) : 0;
        const int es = ms > 0.f ? ilog2f(ms) : 0;
        s_scale[h] = eq;
        s_scale[8 + h] = es;
        s_head[h] = make_float4(pow2i(eq + ew + 1) * a.scale_log2, c0 * sq * a.scale_log2,
                                2.f * pow2i(es) * a.cq * a.scale_log2, -ss * a.cq * a.scale_log2);
      }
    }
    {
      float vmax = 0.f;
      for (int64_t j = tok0 + 4 * tid; j < tok1; j += 4 * MW * 32) {
        const int64_t rec = kv_rec<PAGED>(a, b, kvh, j);   // 4 tokens in a row
        if (PAGED && rec < 0) continue;                    // invalid block: masked
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
      if (lane == 0) s_vmax[warp] = vmax;
    }
    __syncthreads();
    // ---- query operands: warp w builds key k-steps 4w..4w+3, QJL k-steps 2w, 2w+1 ----
    {
      const int hcol = g >> 1;           // head within the MMA's group of four
      const bool tail_col = (g & 1) != 0;
      auto operand = [&](float lo, float hi) -> uint32_t {
        const __half2 h = __floats2half2_rn(lo, hi);
        if (!tail_col) return *reinterpret_cast<const uint32_t*>(&h);
        const float2 f = __half22float2(h);
        return pack_half2((lo - f.x) * 4096.f, (hi - f.y) * 4096.f);
      };
#pragma unroll
      for (int k = 0; k < 6; ++k) {
        const bool key = k < 4;
        const int s = key ? 4 * warp + k : 2 * warp + (k - 4);
        uint32_t fr[4];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int h = 4 * j + hcol;
          const float* row = (key ? a.qr : a.qs) + (qbase + h) * 128 + 32 * t;
          const float kq = key ? pow2i(-(s_scale[h] + ew + 1)) : pow2i(-s_scale[8 + h]);
#pragma unroll
          for (int sl = 0; sl < 2; ++sl) {
            const int u = key ? 2 * (s & 7) + sl : 2 * s + sl;
            const int elo = 10 + u, ehi = (26 + u) & 31;
            const float inv = bit_inv(bit_pos(u)) * kq;
            float vlo, vhi;
            if (key) {
              vlo = row[16 * (s >> 3) + (elo >> 1)] * ((elo & 1) ? w1 : w0) * inv;
              vhi = row[16 * (s >> 3) + (ehi >> 1)] * ((ehi & 1) ? w1 : w0) * inv;
            } else {
              vlo = row[elo] * inv;
              vhi = row[ehi] * inv;
            }
            fr[2 * j + sl] = operand(vlo, vhi);
          }
        }
        const int step = key ? s : 16 + s;
        *reinterpret_cast<uint4*>(qop + (step * 32 + lane) * 4) = make_uint4(fr[0], fr[1], fr[2], fr[3]);
      }
    }
    __syncthreads();
    const float4 H0 = s_head[t], H1 = s_head[4 + t];
    const float vmax = fmaxf(fmaxf(s_vmax[0], s_vmax[1]), fmaxf(s_vmax[2], s_vmax[3]));
    const int kv = vmax >= FLT_MIN ? max(ilog2f(vmax) - 6, -120) : -120;
    const float vmul = pow2i(-kv);

    // ---- this warp's tiles: i = warp, warp + 4, ... of the piece ------------------
    const int ntw = nt > warp ? (nt - warp + MW - 1) / MW : 0;
    const int64_t rb = kv_base<PAGED>(a, b, kvh);   // row base (0 when paged)
    const char* p0 = reinterpret_cast<const char*>(a.kcodes + rb * KW) + lane * 16;
    const char* p1 = reinterpret_cast<const char*>(a.vcodes + rb * VW) + lane * 16;
    const char* p2 = p1 + 8 * 64;
    const char* p3;
    int stride3, tok3;
    uint32_t d3;
    if (lane < 16) {
      p3 = reinterpret_cast<const char*>(a.kqjl + rb * QW) + lane * 16;
      stride3 = 16; tok3 = lane; d3 = offsetof(Stage, q) + lane * 16;
    } else if (lane < 28) {
      const int which = (lane - 16) >> 2, part = (lane - 16) & 3;
      const float* base = which == 0 ? a.knorm : (which == 1 ? a.krnorm : a.vnorm);
      p3 = reinterpret_cast<const char*>(base + rb) + part * 16;
      stride3 = 4; tok3 = 4 * part;
      d3 = (which == 0 ? offsetof(Stage, kn) : (which == 1 ? offsetof(Stage, kr) : offsetof(Stage, vn))) + part * 16;
    } else {
      p3 = nullptr; stride3 = 0; tok3 = 1 << 30; d3 = 0;
    }
    const uint32_t d0 = offsetof(Stage, k) + lane * 16;
    const uint32_t d1 = offsetof(Stage, v) + (lane >> 2) * (VROW * 4) + (lane & 3) * 16;
    const uint32_t d2 = d1 + 8 * (VROW * 4);
    uint32_t bad = 0;   // paged: bit (k % 32) set when the warp's k-th tile has an invalid block id
    auto issue = [&](int k, int stage) {
      const int64_t t0 = tok0 + (int64_t)MT * (warp + MW * k);
      const uint32_t sb = my_s + stage * (uint32_t)sizeof(Stage);
      int64_t r = kv_off<PAGED>(a, b, kvh, t0);   // records of tokens t0.. (16 in a row)
      bool ok = true;
      if (PAGED) {   // the bit of ring tile k is rewritten by every issue (tile k + 32 reuses it)
        ok = r >= 0;
        bad = (bad & ~(1u << (k & 31))) | ((ok ? 0u : 1u) << (k & 31));
        r = ok ? r : 0;
      }
      cp16(sb + d0, p0 + r * 32, ok && t0 + (lane >> 1) < tok1);
      cp16(sb + d1, p1 + r * 64, ok && t0 + (lane >> 2) < tok1);
      cp16(sb + d2, p2 + r * 64, ok && t0 + 8 + (lane >> 2) < tok1);
      if (lane < 28) cp16(sb + d3, p3 + r * stride3, ok && t0 + tok3 < tok1);
    };
#pragma unroll
    for (int k = 0; k < NST8 - 1; ++k) {
      if (k < ntw) issue(k, k);
      cp_commit();
    }

    float m_run[2] = {M_EMPTY, M_EMPTY};
    float l_part[2] = {0.f, 0.f};
    float o[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;

    for (int k = 0; k < ntw; ++k) {
      if (k + NST8 - 1 < ntw) issue(k + NST8 - 1, (k + NST8 - 1) % NST8);
      cp_commit();
      cp_wait<NST8 - 1>();
      __syncwarp();
      const Stage& st = my[k % NST8];
      const int64_t t0 = tok0 + (int64_t)MT * (warp + MW * k);

      // ---- logits: acc[j] for heads 4j + t ----------------------------------------
      float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      float acs[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      {
        const uint2 kg0 = *reinterpret_cast<const uint2*>(&st.k[g][2 * t]);
        const uint2 kg8 = *reinterpret_cast<const uint2*>(&st.k[g + 8][2 * t]);
        const Rot4 R00 = rotations(kg0.x), R01 = rotations(kg0.y);
        const Rot4 R80 = rotations(kg8.x), R81 = rotations(kg8.y);
#define TQ_KSTEP8(S)                                                                              \
  {                                                                                               \
    const uint4 bq = lds128(qop_lane + (S) * 512);                                                \
    const uint32_t x0 = bit_half2<2 * ((S) & 7)>((S) < 8 ? R00 : R01);                            \
    const uint32_t x1 = bit_half2<2 * ((S) & 7)>((S) < 8 ? R80 : R81);                            \
    const uint32_t x2 = bit_half2<2 * ((S) & 7) + 1>((S) < 8 ? R00 : R01);                        \
    const uint32_t x3 = bit_half2<2 * ((S) & 7) + 1>((S) < 8 ? R80 : R81);                        \
    mma16816(acc[0], x0, x1, x2, x3, bq.x, bq.y);                                                 \
    mma16816(acc[1], x0, x1, x2, x3, bq.z, bq.w);                                                 \
  }
        TQ_KSTEP8(0) TQ_KSTEP8(1) TQ_KSTEP8(2) TQ_KSTEP8(3) TQ_KSTEP8(4) TQ_KSTEP8(5)
        TQ_KSTEP8(6) TQ_KSTEP8(7) TQ_KSTEP8(8) TQ_KSTEP8(9) TQ_KSTEP8(10) TQ_KSTEP8(11)
        TQ_KSTEP8(12) TQ_KSTEP8(13) TQ_KSTEP8(14) TQ_KSTEP8(15)
#undef TQ_KSTEP8
        const Rot4 Q0 = rotations(st.q[g][t]), Q8 = rotations(st.q[g + 8][t]);
#define TQ_QSTEP8(S)                                                                              \
  {                                                                                               \
    const uint4 bq = lds128(qop_lane + (16 + (S)) * 512);                                         \
    const uint32_t x0 = bit_half2<2 * (S)>(Q0), x1 = bit_half2<2 * (S)>(Q8);                      \
    const uint32_t x2 = bit_half2<2 * (S) + 1>(Q0), x3 = bit_half2<2 * (S) + 1>(Q8);              \
    mma16816(acs[0], x0, x1, x2, x3, bq.x, bq.y);                                                 \
    mma16816(acs[1], x0, x1, x2, x3, bq.z, bq.w);                                                 \
  }
        TQ_QSTEP8(0) TQ_QSTEP8(1) TQ_QSTEP8(2) TQ_QSTEP8(3) TQ_QSTEP8(4) TQ_QSTEP8(5)
        TQ_QSTEP8(6) TQ_QSTEP8(7)
#undef TQ_QSTEP8
      }
      const bool tile_ok = !PAGED || !((bad >> (k & 31)) & 1u);
      const bool v0 = tile_ok && t0 + g < tok1, v8 = tile_ok && t0 + g + 8 < tok1;
      const float kn0 = st.kn[g], kn8 = st.kn[g + 8], kr0 = st.kr[g], kr8 = st.kr[g + 8];
      float sc[2][2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float4 Hj = j ? H1 : H0;
        const float lm0 = fmaf(acc[j][1], 1.f / 4096.f, acc[j][0]);
        const float lm8 = fmaf(acc[j][3], 1.f / 4096.f, acc[j][2]);
        const float qj0 = fmaf(acs[j][1], 1.f / 4096.f, acs[j][0]);
        const float qj8 = fmaf(acs[j][3], 1.f / 4096.f, acs[j][2]);
        sc[j][0] = v0 ? fmaf(kn0, fmaf(lm0, Hj.x, Hj.y), kr0 * fmaf(qj0, Hj.z, Hj.w)) : -INFINITY;
        sc[j][1] = v8 ? fmaf(kn8, fmaf(lm8, Hj.x, Hj.y), kr8 * fmaf(qj8, Hj.z, Hj.w)) : -INFINITY;
      }

      // ---- online softmax, heads t and 4 + t ----------------------------------------
      const float loc0 = fmaxf(sc[0][0], sc[0][1]), loc1 = fmaxf(sc[1][0], sc[1][1]);
      if (__any_sync(0xffffffffu, loc0 > m_run[0] + LAZY_TAU || loc1 > m_run[1] + LAZY_TAU)) {
        float tm0 = loc0, tm1 = loc1;
#pragma unroll
        for (int o_ = 4; o_ <= 16; o_ <<= 1) {
          tm0 = fmaxf(tm0, __shfl_xor_sync(0xffffffffu, tm0, o_));
          tm1 = fmaxf(tm1, __shfl_xor_sync(0xffffffffu, tm1, o_));
        }
        const float mn0 = fmaxf(m_run[0], tm0), mn1 = fmaxf(m_run[1], tm1);
        const float al0 = ex2f(m_run[0] - mn0), al1 = ex2f(m_run[1] - mn1);
        m_run[0] = mn0;
        m_run[1] = mn1;
        l_part[0] *= al0;
        l_part[1] *= al1;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          o[mt][0] *= al0; o[mt][2] *= al0;
          o[mt][1] *= al1; o[mt][3] *= al1;
        }
      }
      const float p00 = ex2f(sc[0][0] - m_run[0]), p01 = ex2f(sc[0][1] - m_run[0]);
      const float p10 = ex2f(sc[1][0] - m_run[1]), p11 = ex2f(sc[1][1] - m_run[1]);
      l_part[0] += p00 + p01;
      l_part[1] += p10 + p11;
      // A 16-byte norm copy may reach past the row's end: those norms are not data.
      const float w0s = v0 ? st.vn[g] * vmul : 0.f, w8s = v8 ? st.vn[g + 8] * vmul : 0.f;
      const uint32_t pb0 = movtrans(pack_half2(p00 * w0s, p10 * w0s));
      const uint32_t pb1 = movtrans(pack_half2(p01 * w8s, p11 * w8s));

      value_tile(o, st.v, pb0, pb1, lut_lane, g, t);
      __syncwarp();
    }
    cp_wait<0>();
    __syncwarp();

    // ---- this warp's partial of the piece (heads t and 4 + t) --------------------------
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      l_part[j] += __shfl_xor_sync(0xffffffffu, l_part[j], 4);
      l_part[j] += __shfl_xor_sync(0xffffffffu, l_part[j], 8);
      l_part[j] += __shfl_xor_sync(0xffffffffu, l_part[j], 16);
    }
    const float vback = pow2i(kv);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float* pp = a.part + (slot * G + 4 * j + t) * (128 + 2);
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

bool attn_mma_supported(const tq_ctx* c, const AttnArgs& a) {
  if (c->norm_f16) return false;   // QJL formats keep fp32 norms
  if (c->d != D || c->bk_lm != 2 || c->bits_v != 4 || c->qjl_m != 128) return false;
  if (a.G != 8) return false;
  if (a.max_T % 4 != 0) return false;
  const uintptr_t al = reinterpret_cast<uintptr_t>(a.kcodes) | reinterpret_cast<uintptr_t>(a.kqjl) |
                       reinterpret_cast<uintptr_t>(a.knorm) | reinterpret_cast<uintptr_t>(a.krnorm) |
                       reinterpret_cast<uintptr_t>(a.vcodes) | reinterpret_cast<uintptr_t>(a.vnorm);
  return (al & 15) == 0;
}

// Three 4-warp CTAs per SM (the register limit of the segment kernel).
int64_t attn_seg_max_warps(const tq_ctx* c) { return (int64_t)c->sms * 3 * MW; }

cudaError_t launch_attn_mma(const tq_ctx* c, const AttnArgs& a_in, float* out, cudaStream_t s) {
  AttnArgs a = a_in;
  if (a.G != 8 || !a.tiles) return cudaErrorInvalidValue;
  // CTA-owned ranges of at least four tiles per warp.
  const int64_t wmax = (int64_t)a.B * a.Hkv * ((a.max_T + MT - 1) / MT);
  int64_t blocks = (wmax + 4 * MW - 1) / (4 * MW);
  blocks = blocks < 1 ? 1 : (blocks > (int64_t)c->sms * 3 ? (int64_t)c->sms * 3 : blocks);
  a.nw = (int)blocks;
  a.wpu = MW;
  if (a.block_table)
    k_attn_seg8<true><<<(unsigned)blocks, MW * 32, SMEM8_BYTES, s>>>(a);
  else
    k_attn_seg8<false><<<(unsigned)blocks, MW * 32, SMEM8_BYTES, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_attn_merge(c, a, out, s);
}

cudaError_t configure_attn_mma() {
  const int b8 = (int)SMEM8_BYTES;
  const cudaFuncAttribute ms = cudaFuncAttributeMaxDynamicSharedMemorySize;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(k_attn_seg8<false>, ms, b8))) return e;
  return cudaFuncSetAttribute(k_attn_seg8<true>, ms, b8);
}

}  // namespace tqk
