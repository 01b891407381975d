// Device helpers shared by the decode-attention kernels (sm_100a): tile
// constants, mma.sync / movmatrix / cp.async wrappers, the fp16 bit-operand
// encoding of code bits, and the value product of one 16-token tile.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "tq_internal.h"

namespace tqk {
namespace {

constexpr int MW = 4;           // warps per CTA
constexpr int MT = 16;          // tokens per tile
constexpr int D = 128;
constexpr int QW = 4;           // QJL words per token (m = 128)
constexpr int VW = 16;          // value code words per token (4-bit fields)
constexpr int VROW = 20;        // padded value row (words): conflict-free LDS.64
constexpr int LUT_WORDS = 256 * 32;   // value table: 256 code pairs x 32 lane copies
// The running maximum moves only when a tile exceeds it by 2^8 (exp2 units).
constexpr float LAZY_TAU = 8.f;
// Running maximum before the first valid token: finite, so that a tile whose
// tokens are all masked (logits -inf, e.g. an invalid block of a paged cache)
// gives exp2(-inf - M_EMPTY) = 0 instead of NaN.  A partial that saw no token
// keeps it (with l = 0, o = 0) and gets weight 0 in the merge next to any
// partial that saw one.
constexpr float M_EMPTY = -1e30f;

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t movtrans(uint32_t x) {
  uint32_t y;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void cp16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n));
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];\n" : "=r"(v) : "r"(addr));
  return v;
}

// ---------------------------------------------------------------------------
// Key operands.  A query head takes two B columns of the key MMA: the fp16
// head of its operand and the fp16 tail (x 2^12), so one MMA yields both
// products of every k-step and the fp32 sum restores ~22 bits.
//
// Keys use exact binary A operands.  A symmetric 2-bit codebook is affine in
// the index bits, c[i0 + 2 i1] = c0 + (c1 - c0) i0 + (c2 - c0) i1, so
//   <q', c[idx]> = c0 sum_j q'_j + (c1 - c0) <q', i0> + (c2 - c0) <q', i1>,
// and the QJL term is <s, sigma> = 2 <s, bit> - sum_i s_i.  A bit becomes an
// fp16 operand by masking it into the exponent field: a lone bit at position
// p in 10..14 of a half reads as 2^E(p), E = -14, -13, -11, -7, 1, and the
// B operand carries the inverse power of two.  Four rotations of a 32-bit
// code word and sixteen masks give sixteen half2 registers: register u holds
// bit 10+u in its low half and bit (26+u) mod 32 in its high half.
// ---------------------------------------------------------------------------
__host__ __device__ constexpr int bit_pos(int u) {
  return u < 5 ? 10 + u : (u < 10 ? 5 + u : (u < 15 ? u : 10));
}
__host__ __device__ constexpr int bit_rot(int u) { return u < 5 ? 0 : (u < 10 ? 5 : (u < 15 ? 10 : 15)); }
__device__ __forceinline__ float bit_inv(int p) {
  return p == 10 ? 16384.f : (p == 11 ? 8192.f : (p == 12 ? 2048.f : (p == 13 ? 128.f : 0.5f)));
}

struct Rot4 {
  uint32_t r[4];
};
__device__ __forceinline__ Rot4 rotations(uint32_t w) {
  return Rot4{{w, __funnelshift_r(w, w, 5), __funnelshift_r(w, w, 10), __funnelshift_r(w, w, 15)}};
}
template <int U>
__device__ __forceinline__ uint32_t bit_half2(const Rot4& R) {
  constexpr int p = bit_pos(U);
  return R.r[bit_rot(U) / 5] & ((1u << p) | (1u << (p + 16)));
}

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}
// 2^e for an integer e in the normal fp32 range.
__device__ __forceinline__ float pow2i(int e) { return __int_as_float((e + 127) << 23); }
// floor(log2(x)) for a positive normal float.
__device__ __forceinline__ int ilog2f(float x) { return ((__float_as_int(x) >> 23) & 0xFF) - 127; }

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// Value table: entry (byte, lane) = half2(cv[byte & 15], cv[byte >> 4]).
__device__ __forceinline__ void build_value_lut(uint32_t* lut, const float* cv, int tid, int nthreads) {
  for (int e = tid; e < LUT_WORDS; e += nthreads) {
    const int byte = e >> 5;
    lut[e] = pack_half2(cv[byte & 15], cv[byte >> 4]);
  }
}

// Wide value table for kernels with one CTA per SM: entry (byte, lane) at
// byte offset 256 byte + 4 lane, so one byte permute forms the address from
// the code-pair byte and the lane's offset (64 KB; half of each entry unused).
constexpr int WLUT_BYTES = 256 * 256;
__device__ __forceinline__ void build_value_wlut(uint32_t* lut, const float* cv, int tid, int nthreads) {
  for (int e = tid; e < 256 * 32; e += nthreads) {
    const int byte = e >> 5, ln = e & 31;
    lut[byte * 64 + ln] = pack_half2(cv[byte & 15], cv[byte >> 4]);
  }
}

// o[mt] += V^T P for one 16-token tile: A = dequantized values (16 dims x 16
// tokens per mt), B = [pb0; pb1] (16 tokens x 8 columns).  v holds the tile's
// 16 value-code rows (VROW words each); a code pair (two tokens, one dim)
// indexes the lane's copy of the value table.
__device__ __forceinline__ void value_tile(float (&o)[8][4], const uint32_t (*v)[VROW], uint32_t pb0,
                                           uint32_t pb1, uint32_t lut_lane, int g, int t) {
  const uint2 xa = *reinterpret_cast<const uint2*>(&v[2 * t][2 * g]);
  const uint2 xb = *reinterpret_cast<const uint2*>(&v[2 * t + 1][2 * g]);
  const uint2 xc = *reinterpret_cast<const uint2*>(&v[2 * t + 8][2 * g]);
  const uint2 xd = *reinterpret_cast<const uint2*>(&v[2 * t + 9][2 * g]);
  const uint32_t ye[4] = {(xa.x & 0x0F0F0F0Fu) | ((xb.x << 4) & 0xF0F0F0F0u),
                          (xa.y & 0x0F0F0F0Fu) | ((xb.y << 4) & 0xF0F0F0F0u),
                          (xc.x & 0x0F0F0F0Fu) | ((xd.x << 4) & 0xF0F0F0F0u),
                          (xc.y & 0x0F0F0F0Fu) | ((xd.y << 4) & 0xF0F0F0F0u)};
  const uint32_t yo[4] = {((xa.x >> 4) & 0x0F0F0F0Fu) | (xb.x & 0xF0F0F0F0u),
                          ((xa.y >> 4) & 0x0F0F0F0Fu) | (xb.y & 0xF0F0F0F0u),
                          ((xc.x >> 4) & 0x0F0F0F0Fu) | (xd.x & 0xF0F0F0F0u),
                          ((xc.y >> 4) & 0x0F0F0F0Fu) | (xd.y & 0xF0F0F0F0u)};
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const int k = mt >> 1;
    const uint32_t* y = (mt & 1) ? yo : ye;
    uint32_t av[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) av[r] = lds32(__byte_perm(y[r], 0, 0x4440 + k) * 128u + lut_lane);
    mma16816(o[mt], av[0], av[1], av[2], av[3], pb0, pb1);
  }
}

// value_tile with the wide table at shared address lut_s; lane4 = 4 * lane.
__device__ __forceinline__ void value_tile_w(float (&o)[8][4], const uint32_t (*v)[VROW], uint32_t pb0,
                                             uint32_t pb1, uint32_t lut_s, uint32_t lane4, int g, int t) {
  const uint2 xa = *reinterpret_cast<const uint2*>(&v[2 * t][2 * g]);
  const uint2 xb = *reinterpret_cast<const uint2*>(&v[2 * t + 1][2 * g]);
  const uint2 xc = *reinterpret_cast<const uint2*>(&v[2 * t + 8][2 * g]);
  const uint2 xd = *reinterpret_cast<const uint2*>(&v[2 * t + 9][2 * g]);
  const uint32_t ye[4] = {(xa.x & 0x0F0F0F0Fu) | ((xb.x << 4) & 0xF0F0F0F0u),
                          (xa.y & 0x0F0F0F0Fu) | ((xb.y << 4) & 0xF0F0F0F0u),
                          (xc.x & 0x0F0F0F0Fu) | ((xd.x << 4) & 0xF0F0F0F0u),
                          (xc.y & 0x0F0F0F0Fu) | ((xd.y << 4) & 0xF0F0F0F0u)};
  const uint32_t yo[4] = {((xa.x >> 4) & 0x0F0F0F0Fu) | (xb.x & 0xF0F0F0F0u),
                          ((xa.y >> 4) & 0x0F0F0F0Fu) | (xb.y & 0xF0F0F0F0u),
                          ((xc.x >> 4) & 0x0F0F0F0Fu) | (xd.x & 0xF0F0F0F0u),
                          ((xc.y >> 4) & 0x0F0F0F0Fu) | (xd.y & 0xF0F0F0F0u)};
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const int k = mt >> 1;
    const uint32_t* y = (mt & 1) ? yo : ye;
    uint32_t av[4];
    // byte 0 = 4 lane, byte 1 = code-pair byte k of y, bytes 2-3 = 0
#pragma unroll
    for (int r = 0; r < 4; ++r) av[r] = lds32(lut_s + __byte_perm(lane4, y[r], 0x1140 + 16 * k));
    mma16816(o[mt], av[0], av[1], av[2], av[3], pb0, pb1);
  }
}

// Record index of token t of row (b, kv head): [B][Hkv][max_T] contiguous, or
// paged [blocks][Hkv][block_size] through the block table; -1 when the
// block id is outside [0, num_blocks) (the caller masks those tokens).  For
// t a multiple of 4 (16 when paged with block_size % 16 == 0) the next 3 (15)
// tokens are the next records.
template <bool PAGED>
__device__ __forceinline__ int64_t kv_rec(const AttnArgs& a, int b, int kvh, int64_t t);

// Record base of row (b, kv head) folded into the array pointers (contiguous
// caches), and the per-tile record offset relative to it: t itself, or for
// paged caches the full record index (base 0).
template <bool PAGED>
__device__ __forceinline__ int64_t kv_base(const AttnArgs& a, int b, int kvh) {
  return PAGED ? 0 : ((int64_t)b * a.Hkv + kvh) * a.max_T;
}
template <bool PAGED>
__device__ __forceinline__ int64_t kv_off(const AttnArgs& a, int b, int kvh, int64_t t) {
  return PAGED ? kv_rec<true>(a, b, kvh, t) : t;
}

template <bool PAGED>
__device__ __forceinline__ int64_t kv_rec(const AttnArgs& a, int b, int kvh, int64_t t) {
  if (!PAGED) return ((int64_t)b * a.Hkv + kvh) * a.max_T + t;
  const int ti = (int)t;
  const int64_t blk = a.block_table[(int64_t)b * a.max_blocks + ti / a.block_size];
  if (blk < 0 || blk >= a.num_blocks) return -1;
  return (blk * a.Hkv + kvh) * a.block_size + ti % a.block_size;
}

// Sequence holding tile x of the tile prefix P[0..B]: P[b] <= x < P[b + 1].
__device__ __forceinline__ int locate_sequence(const int64_t* P, int B, int64_t x) {
  int b = 0, hi = B;
  while (hi - b > 1) {
    const int mid = (b + hi) >> 1;
    if (P[mid] <= x) b = mid; else hi = mid;
  }
  return b;
}

}  // namespace
}  // namespace tqk
