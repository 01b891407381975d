// Query-operand images of the int8 key product (sm_100a device helpers).
//
// For one KV group (G <= 4 query heads) the image holds the B fragments of
// mma.sync m16n8k32 (s8) for every code-bit position of a 128-dim key:
//   key bits:  bit p of byte e of code word w carries index bit pl = bit % 2
//              of coordinate j = 16 w + bit / 2 (bit = 8 e + p); its weight is
//              w_pl q'_j (w0 = c1 - c0, w1 = c2 - c0 of the 2-bit codebook),
//   QJL bits:  bit p of byte e of QJL word j / 32 is sigma_j; weight s_j = (S q')_j.
// Each weight (an fp32 product) becomes Q = round(2^(S - p) weight), S from
// the largest |weight| of the head so that |Q| < 2^30 at p = 0, written as
// four balanced signed-byte digits, digit l in column 2 hg + l % 2 of N tile
// l / 2 (hg = head within the group).
// Register rr of lane ln holds bytes e = 0..3 of fragment rows; the image is
// [12 uint4 per lane][32 lanes] followed by one float4 of head constants per
// head: (2^-S scale, c0 sum q' scale, 2^(1-S') cq scale, -sum s cq scale),
// scale = softmax scale * log2(e), so that
//   logit * scale = |k| (K 2^-S + c0 sum q') scale + |r| cq (2 <s, bit> - sum s) scale.
#pragma once

#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "tq_internal.h"

namespace tqk {

struct QopExp {
  int S, S2;   // key and QJL digit scales
};

// Digit scales from the head's largest |q'_j| (mq) and |s_j| (ms).
__device__ __forceinline__ QopExp qop_exponents(const QopPlan& P, float mq, float ms) {
  const double c0 = P.c0, w0 = (double)P.c1 - c0, w1 = (double)P.c2 - c0;
  const double wmax = fmax(fabs(w0), fabs(w1));
  const double mk = wmax * mq;
  QopExp e;
  // 2^e <= max |w q'| < 2^(e+1), S = 29 - e: |Q| < 2^30 at p = 0.
  e.S = mk > 0.0 ? 29 - ilogb(mk) : 0;
  e.S2 = ms > 0.f ? 29 - ilogb((double)ms) : 0;
  return e;
}

// The image bytes of coordinate j of head hg: two key weights and one QJL
// weight, four digits each (12 byte stores into img).  The weights are fp32
// products (24 significant bits, as many as the decode recombines), scaled by
// a power of two and rounded to an int32 (|Q| < 2^30).
__device__ __forceinline__ void qop_put_coord(const QopPlan& P, unsigned char* img, int hg, int j, float qj,
                                              float sj, QopExp ex) {
  const float w0 = (float)((double)P.c1 - (double)P.c0), w1 = (float)((double)P.c2 - (double)P.c0);
  auto put = [&](int reg, int tt, int e, int Q) {
#pragma unroll
    for (int l = 0; l < 4; ++l) {
      const int dg = (int)(signed char)(Q & 0xFF);
      Q = (Q - dg) >> 8;
      const int rr = reg + 2 * (l >> 1);
      const int ln = 4 * (2 * hg + (l & 1)) + tt;
      img[(((rr >> 2) * 32 + ln) * 4 + (rr & 3)) * 4 + e] = (unsigned char)(dg & 0xFF);
    }
  };
#pragma unroll
  for (int pl = 0; pl < 2; ++pl) {
    const int bit = 2 * (j & 15) + pl, w = j >> 4, p = bit & 7;
    const int Q = __float2int_rn(ldexpf((pl ? w1 : w0) * qj, ex.S - p));
    put(4 * p + (w >> 2), w & 3, bit >> 3, Q);
  }
  const int bit = j & 31, p = bit & 7;
  const int Q = __float2int_rn(ldexpf(sj, ex.S2 - p));
  put(32 + 4 * (p >> 1) + (p & 1), j >> 5, bit >> 3, Q);
}

// Head constants of head hg (sq = sum_j q'_j, ss = sum_j s_j).
__device__ __forceinline__ void qop_put_constants(const QopPlan& P, unsigned char* img, int hg, QopExp ex,
                                                  double sq, double ss) {
  const double sl = P.scale_log2, c0 = P.c0;
  float4 cst;
  cst.x = (float)ldexp(sl, -ex.S);
  cst.y = (float)(c0 * sq * sl);
  cst.z = (float)ldexp(2.0 * (double)P.cq * sl, -ex.S2);
  cst.w = (float)(-ss * (double)P.cq * sl);
  reinterpret_cast<float4*>(img + kQopRegs * 32 * 4)[hg] = cst;
}

}  // namespace tqk
