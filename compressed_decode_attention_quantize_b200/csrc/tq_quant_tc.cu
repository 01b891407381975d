// Online quantization on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// "What is TurboQuant?", section "How TurboQuant works": stage 1 rotates the
// normalised vector with the random orthogonal Pi and maps every coordinate
// to its Lloyd-Max index; stage 2 keeps sign(S r) of the residual r.  Here
// both products are GEMMs over a tile of 128 vectors:
//   D_rot[v][j] = sum_k x[v][k] Pi'[j][k]      (M = 128 vectors, N = K = 128)
//   D_qjl[v][i] = sum_k r[v][k] S[i][k]
// issued by one thread per tile group with operands in shared memory (128-byte
// swizzled, K-major) and fp32 accumulators in tensor memory.  TMEM lane v
// holds vector v; two threads own it, one per half of the coordinates, so
// index computation and bit packing need no cross-thread exchange (a packed
// word never spans the halves) and only the two norms are combined.
//
// Exactness.  x (bf16 or fp16) is exact in fp16 after a per-vector power of
// two scale.  Pi' = 2^8 Pi is split into an fp16 head and tail; both products
// accumulate into the same TMEM columns, so y carries ~2^-22 relative error,
// far inside the 1e-5 decision band.  r (scaled by 2^14) is likewise fed as an
// fp16 head and tail tile against the exact fp16 S.  A QJL sign is recomputed
// in fp32 whenever |(S r)_i| is within 2^-17 |S_i| |r| of zero, a bound on the
// operand and accumulation rounding of the tensor-core product (a few bits
// per thousand vectors).
//
// Two groups of eight warps per CTA work on different tiles, so one group's
// MMAs overlap the other's epilogue, and sixteen warps per SM hide latency.
// Waits on MMA completion are bounded; on timeout the group waits (with the
// full limit) for the MMAs it issued, the kernel records a fault code,
// releases its tensor memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "tq_internal.h"
#include "tq_tc_common.cuh"

namespace tqk {

__device__ int g_tq_fault = 0;

namespace {

constexpr int TILE = 128;
constexpr uint32_t SMEM_TILE = 32768;            // one 128 x 128 fp16 operand
constexpr uint32_t OFF_PIH = 0, OFF_PIL = SMEM_TILE, OFF_S = 2 * SMEM_TILE;
constexpr uint32_t OFF_A = 3 * SMEM_TILE;        // + wg * 2 * SMEM_TILE: head, tail
constexpr uint32_t OFF_MISC = 7 * SMEM_TILE;
constexpr uint32_t TC_SMEM = OFF_MISC + 1024 + 1024;  // misc + alignment slack
// Instruction descriptor: D f32, A/B f16, both K-major, N = 128, M = 128.
constexpr uint32_t IDESC = tc_idesc_f16(128);

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t accumulate) {
  tc_mma_f16(d_tmem, a, b, IDESC, accumulate);
}

__device__ __forceinline__ void mma_commit(uint32_t bar) { tc_commit(bar); }

// Byte offset of the 16-byte chunk c (8 fp16 values k = 8c..8c+7) of row r in
// a 128 x 128 K-major operand with 128-byte swizzle (two 64-wide K blocks).
__device__ __forceinline__ uint32_t chunk_off(int r, int c) {
  return (uint32_t)((c >> 3) * 16384 + (r >> 3) * 1024 + (r & 7) * 128 + (((c & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ uint32_t h2bits(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float pow2f(int e) { return __int_as_float((e + 127) << 23); }
__device__ __forceinline__ int flog2(float x) { return ((__float_as_int(x) >> 23) & 0xFF) - 127; }

// Output record of vector v (slot pos[b] of row v = b H + g for cache
// appends); -1 (nothing written) when pos[b] is outside [0, max_T).
__device__ __forceinline__ int64_t out_rec(const QuantTcArgs& a, int64_t v) {
  if (a.pos == nullptr) return v;
  const int64_t p = a.pos[v / a.H];
  return (p >= 0 && p < a.max_T) ? v * a.max_T + p : -1;
}

// Lloyd-Max index of y for 2^BITS symmetric levels: binary search over the
// positive boundaries (pb, L/2 - 1 of them, ascending) on |y|, then mirrored.
// The first level compares with a register (pmid = pb[L/4 - 1]); deeper
// levels read the thresholds from shared memory (distinct banks).
template <int BITS>
__device__ __forceinline__ int lm_idx(float y, float pmid, const float* pb) {
  constexpr int H = 1 << (BITS - 1);
  const float a = fabsf(y);
  if constexpr (BITS == 8) {
    // pb: the 127 positive thresholds in breadth-first order of the balanced
    // search tree (node i has children 2i + 1, 2i + 2), so the lanes of one
    // level read a contiguous range of banks.  Leaf i - 127 = the count of
    // thresholds <= |y|.
    int i = 0;
#pragma unroll
    for (int l = 0; l < 7; ++l) i = 2 * i + 1 + (a >= pb[i] ? 1 : 0);
    const int j = i - 127;
    return (y >= 0.f) ? H + j : H - 1 - j;
  }
  int j = 0;
  if (BITS >= 2) j = (a >= pmid) ? (H >> 1) : 0;
  if (BITS >= 4) j += (a >= pb[j + 1]) ? 2 : 0;
  if (BITS >= 3) j += (a >= pb[j]) ? 1 : 0;
  return (y >= 0.f) ? H + j : H - 1 - j;
}

struct Q4 {
  uint32_t w[4];
};

// Exact fp32 signs of the flagged QJL rows (rare), two rows per lane per
// pass; r is rebuilt from the rotation accumulator exactly as in the main
// epilogue.  tcgen05.ld is warp-collective, so whole warps call and loop.
template <int BITS>
__device__ __noinline__ Q4 qjl_fixup(uint32_t taddr, float inv, float pmid, const float* pb,
                                     const float* s_cen, const float* s_f32, Q4 flag, Q4 qw) {
  while (__any_sync(0xffffffffu, (flag.w[0] | flag.w[1] | flag.w[2] | flag.w[3]) != 0u)) {
    int rows[2] = {-1, -1};
#pragma unroll
    for (int q = 0; q < 2; ++q) {
#pragma unroll
      for (int fw = 0; fw < 4; ++fw) {
        if (rows[q] < 0 && flag.w[fw] != 0u) {
          const int bit = __ffs(flag.w[fw]) - 1;
          flag.w[fw] &= flag.w[fw] - 1;
          rows[q] = fw * 32 + bit;
        }
      }
    }
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 1
    for (int ch = 0; ch < 4; ++ch) {
      float d[32];
      tmem_ld32(taddr + ch * 32, d);
      if (rows[0] >= 0) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float y = d[i] * inv;
          const float r = fmaf(y, 16384.f, -s_cen[lm_idx<BITS>(y, pmid, pb)]);
          acc0 = fmaf(__ldg(s_f32 + (size_t)rows[0] * 128 + ch * 32 + i), r, acc0);
          if (rows[1] >= 0) acc1 = fmaf(__ldg(s_f32 + (size_t)rows[1] * 128 + ch * 32 + i), r, acc1);
        }
      }
    }
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      if (rows[q] >= 0) {
        const int fw = rows[q] >> 5, bit = rows[q] & 31;
        const bool pos = (q == 0 ? acc0 : acc1) >= 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w)
          if (w == fw) qw.w[w] = (qw.w[w] & ~(1u << bit)) | ((pos ? 1u : 0u) << bit);
      }
    }
  }
  return qw;
}

// Thread (group gi, half h, row r): two groups of eight warps per CTA work on
// different tiles; within a group, warps w and w + 4 share TMEM lanes 32 (w &
// 3) .. + 31 (one vector per lane) and take coordinate halves h = 0, 1
// (columns 64h .. 64h + 63 of every accumulator).  The two threads of a
// vector exchange partial sums through two TMEM columns of their lane.
__device__ __forceinline__ void tmem_st1(uint32_t taddr, float v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};\n" ::"r"(taddr), "r"(__float_as_uint(v))
               : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ float tmem_sum2(uint32_t taddr) {
  uint32_t r0, r1;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];\n" : "=r"(r0), "=r"(r1) : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
  return __uint_as_float(r0) + __uint_as_float(r1);
}
__device__ __forceinline__ void grp_sync(int gi) { asm volatile("bar.sync %0, 256;\n" ::"r"(1 + gi) : "memory"); }
// True on every thread of the group if any of its threads passes true.
__device__ __forceinline__ bool grp_any(int gi, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, 256, p;\n\tselp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(1 + gi)
      : "memory");
  return r != 0u;
}

template <int BITS, bool QJL>
__global__ void __launch_bounds__(512, 1) k_quant_tc(QuantTcArgs a) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_s = (uint32_t)__cvta_generic_to_shared(smem_raw);
  const uint32_t base_s = (raw_s + 1023u) & ~1023u;
  unsigned char* base = smem_raw + (base_s - raw_s);
  float* s_snorm = reinterpret_cast<float*>(base + OFF_MISC + 64);   // [128]
  float* s_cen = s_snorm + 128;                                        // [16]
  float* s_pb = s_cen + 16;                                            // [8]
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(base + OFF_MISC + 32);
  const uint32_t bar0 = base_s + OFF_MISC;   // 4 barriers: rot g0, rot g1, qjl g0, qjl g1

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gi = tid >> 8, wq = (tid >> 5) & 7, h = wq >> 2;
  const int row = 32 * (wq & 3) + lane;
  constexpr int L = 1 << BITS;
  constexpr int PER = (BITS == 3) ? 16 : 32 / BITS;   // fields per word of the main stream
  constexpr int W_MAIN = 128 / PER;                     // words of the main stream
  constexpr int WORDS = (BITS == 3) ? W_MAIN + 4 : W_MAIN;

  // ---- shared tables: operand images, QJL row norms, codebook --------------------
  {
    const int4* src_pih = reinterpret_cast<const int4*>(a.pi_hi);
    const int4* src_pil = reinterpret_cast<const int4*>(a.pi_lo);
    const int4* src_s = reinterpret_cast<const int4*>(a.s_img);
    int4* dst = reinterpret_cast<int4*>(base);
    for (int e = tid; e < (int)(SMEM_TILE / 16); e += 512) {
      dst[OFF_PIH / 16 + e] = src_pih[e];
      dst[OFF_PIL / 16 + e] = src_pil[e];
      if (QJL) dst[OFF_S / 16 + e] = src_s[e];
    }
    if (tid < 128) s_snorm[tid] = QJL ? a.snorm[tid] : 0.f;
    if (tid < 16) s_cen[tid] = tid < L ? a.cen[tid] * (QJL ? 16384.f : 1.f) : 0.f;
    if (tid < 8) s_pb[tid] = (tid < L / 2 - 1) ? a.bnd[L / 2 + tid] : INFINITY;
  }
  if (tid == 0) {
    for (int i = 0; i < 4; ++i)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(bar0 + 8 * i) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;\n" ::"r"(
                     base_s + OFF_MISC + 32)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  fence_async_smem();
  tc_before_sync();
  __syncthreads();
  tc_after_sync();
  const uint32_t tmem = *s_tmem;
  const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
  const uint32_t d_rot = tmem + (uint32_t)(gi * 256);
  const uint32_t d_qjl = d_rot + 128;
  // Two columns of the QJL accumulator (free outside the QJL product) carry
  // the halves' partial sums.
  const uint32_t x_col = d_qjl + lane_base;
  const uint32_t sA = base_s + OFF_A + gi * 2 * SMEM_TILE;
  unsigned char* A = base + OFF_A + gi * 2 * SMEM_TILE;
  unsigned char* A2 = A + SMEM_TILE;
  const uint32_t bar_rot = bar0 + 8 * gi, bar_q = bar0 + 16 + 8 * gi;
  const bool leader = (tid & 255) == 0;
  const float* pb = s_pb;
  float snorm_max = 0.f;
  if (QJL)
    for (int i = 0; i < 128; ++i) snorm_max = fmaxf(snorm_max, s_snorm[i]);
  const float pmid = BITS >= 2 ? s_pb[(L >> 2) - 1] : 0.f;

  const int64_t ntiles = (a.n + TILE - 1) / TILE;
  const int64_t tstride = (int64_t)gridDim.x * 2;
  const bool is_bf = a.dtype == TQ_BF16;
  auto lo_f = [&](uint32_t w) {
    return is_bf ? __uint_as_float(w << 16) : __half2float(__ushort_as_half((unsigned short)(w & 0xFFFF)));
  };
  auto hi_f = [&](uint32_t w) {
    return is_bf ? __uint_as_float(w & 0xFFFF0000u) : __half2float(__ushort_as_half((unsigned short)(w >> 16)));
  };
  // This half's 64 coordinates of vector `row` of tile t (zeros past the end).
  auto load_x = [&](int64_t t, uint4 (&xr)[8]) {
    const int64_t vv = t * TILE + row;
    if (vv < a.n) {
      const uint4* src =
          reinterpret_cast<const uint4*>(static_cast<const unsigned short*>(a.x) + vv * a.ld + 64 * h);
#pragma unroll
      for (int c = 0; c < 8; ++c) xr[c] = src[c];
    } else {
#pragma unroll
      for (int c = 0; c < 8; ++c) xr[c] = make_uint4(0, 0, 0, 0);
    }
  };
  uint32_t iter = 0;
  bool fault = false;
  for (int64_t tile = (int64_t)blockIdx.x * 2 + gi; tile < ntiles; tile += tstride, ++iter) {
    const int64_t v = tile * TILE + row;
    const bool live = v < a.n;
    uint4 xr[8];
    load_x(tile, xr);
    {
      const int64_t nxt = tile + tstride;
      if (leader && a.ld == 128 && nxt < ntiles) {
        const int64_t rows_left = a.n - nxt * TILE;
        const uint32_t bytes = (uint32_t)((rows_left < TILE ? rows_left : TILE) * 256);
        const void* p = static_cast<const unsigned short*>(a.x) + nxt * TILE * 128;
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(p), "r"(bytes) : "memory");
      }
    }
    // ---- this half's 64 coordinates, the norm, the scaled fp16 operand ---------------
    float ssp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint32_t w4[4] = {xr[c].x, xr[c].y, xr[c].z, xr[c].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float f0 = lo_f(w4[q]), f1 = hi_f(w4[q]);
        ssp[q] = fmaf(f0, f0, ssp[q]);
        ssp[q] = fmaf(f1, f1, ssp[q]);
      }
    }
    tmem_st1(x_col + h, (ssp[0] + ssp[1]) + (ssp[2] + ssp[3]));
    tc_before_sync();
    grp_sync(gi);
    tc_after_sync();
    const float nrm = sqrtf(tmem_sum2(x_col));
    const int e = nrm > 0.f ? 14 - flog2(nrm) : 0;
    const float sc = pow2f(e);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint32_t w4[4] = {xr[c].x, xr[c].y, xr[c].z, xr[c].w};
      uint4 o;
      o.x = h2bits(lo_f(w4[0]) * sc, hi_f(w4[0]) * sc);
      o.y = h2bits(lo_f(w4[1]) * sc, hi_f(w4[1]) * sc);
      o.z = h2bits(lo_f(w4[2]) * sc, hi_f(w4[2]) * sc);
      o.w = h2bits(lo_f(w4[3]) * sc, hi_f(w4[3]) * sc);
      *reinterpret_cast<uint4*>(A + chunk_off(row, 8 * h + c)) = o;
    }
    fence_async_smem();
    tc_before_sync();
    grp_sync(gi);
    // ---- rotation: D_rot = A (Pi'_hi + Pi'_lo)^T -----------------------------------
    if (leader) {
      tc_after_sync();
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const uint32_t koff = (uint32_t)((s >> 2) * 16384 + (s & 3) * 32);
        mma_f16(d_rot, smem_desc(sA + koff), smem_desc(base_s + OFF_PIH + koff), s > 0 ? 1u : 0u);
        mma_f16(d_rot, smem_desc(sA + koff), smem_desc(base_s + OFF_PIL + koff), 1u);
      }
      mma_commit(bar_rot);
    }
    if (grp_any(gi, !mbar_wait(bar_rot, iter & 1, a.wait_limit))) {
      mbar_wait(bar_rot, iter & 1);   // drain: the group's MMAs finish before TMEM is released
      fault = true;
      break;
    }
    tc_after_sync();

    // ---- epilogue 1: indices, packing, residual (this half's two 32-column chunks) ----
    // y = D_rot / (sc * nrm * 2^8); the residual goes out scaled by 2^14.
    const float inv = nrm > 0.f ? 1.f / (sc * nrm * 256.f) : 0.f;
    const int64_t rec0 = live ? out_rec(a, v) : -1;
    const bool writes = rec0 >= 0;   // this vector's record exists
    const int64_t rec = writes ? rec0 : 0;
    uint32_t* crow = a.codes + rec * WORDS;
    float rho2v[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
    for (int ch = 2 * h; ch < 2 * h + 2; ++ch) {
      float d[32];
      tmem_ld32(d_rot + lane_base + ch * 32, d);
      // words of this chunk: b words of b-bit fields (b = 3: two 2-bit words + one bit word)
      uint32_t cw[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float y = d[i] * inv;
        const int idx = lm_idx<BITS>(y, pmid, pb);
        if (BITS == 3) {
          cw[i >> 4] |= (uint32_t)(idx & 3) << (2 * (i & 15));
          cw[2] |= (uint32_t)(idx >> 2) << i;
        } else {
          cw[i / PER] |= (uint32_t)idx << (BITS * (i % PER));
        }
        if (QJL) {
          const float r = fmaf(y, 16384.f, -s_cen[idx]);   // s_cen holds 2^14 c
          rho2v[i & 3] = fmaf(r, r, rho2v[i & 3]);
          d[i] = r;
        }
      }
      if (writes) {
        if (BITS == 4) *reinterpret_cast<uint4*>(crow + 4 * ch) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
        if (BITS == 2) *reinterpret_cast<uint2*>(crow + 2 * ch) = make_uint2(cw[0], cw[1]);
        if (BITS == 1) crow[ch] = cw[0];
        if (BITS == 3) {
          *reinterpret_cast<uint2*>(crow + 2 * ch) = make_uint2(cw[0], cw[1]);
          crow[W_MAIN + ch] = cw[2];
        }
      }
      if (QJL) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t hv[4], lv[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float r0 = d[8 * q + 2 * u], r1 = d[8 * q + 2 * u + 1];
            const __half2 hh = __floats2half2_rn(r0, r1);
            const float2 f = __half22float2(hh);
            hv[u] = *reinterpret_cast<const uint32_t*>(&hh);
            lv[u] = h2bits(r0 - f.x, r1 - f.y);
          }
          *reinterpret_cast<uint4*>(A + chunk_off(row, ch * 4 + q)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
          *reinterpret_cast<uint4*>(A2 + chunk_off(row, ch * 4 + q)) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
        }
      }
    }
    if (writes && h == 0) a.norm[rec] = nrm;
    if (!QJL) {
      tc_before_sync();
      grp_sync(gi);   // A and D_rot are free for the next tile
      continue;
    }
    tmem_st1(x_col + h, (rho2v[0] + rho2v[1]) + (rho2v[2] + rho2v[3]));
    fence_async_smem();
    tc_before_sync();
    grp_sync(gi);
    tc_after_sync();
    const float rho = sqrtf(tmem_sum2(x_col)) * (1.f / 16384.f);
    tc_before_sync();
    grp_sync(gi);   // the partial sums are read before the QJL product overwrites them
    // ---- QJL product: D_qjl = (2^14 r) S^T ----------------------------------------------
    if (leader) {
      tc_after_sync();
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const uint32_t koff = (uint32_t)((s >> 2) * 16384 + (s & 3) * 32);
        mma_f16(d_qjl, smem_desc(sA + koff), smem_desc(base_s + OFF_S + koff), s > 0 ? 1u : 0u);
        mma_f16(d_qjl, smem_desc(sA + SMEM_TILE + koff), smem_desc(base_s + OFF_S + koff), 1u);
      }
      mma_commit(bar_q);
    }
    if (grp_any(gi, !mbar_wait(bar_q, iter & 1, a.wait_limit))) {
      mbar_wait(bar_q, iter & 1);   // drain, as above
      fault = true;
      break;
    }
    tc_after_sync();
    // D = 2^14 (S r); flag |D_i| <= 2^14 * 2^-17 max_i |S_i| rho.
    const float thr = 0.125f * rho * snorm_max;
    uint32_t qw[4] = {0u, 0u, 0u, 0u};
    uint32_t flag[4] = {0u, 0u, 0u, 0u};
    // Bit i = sign bit of D_i (then inverted: 1 <=> D_i >= 0) and of thr - |D_i|
    // (inverted: 1 <=> |D_i| <= thr), shifted in from the top, row 31 first.  A
    // D_i of -0 reads as negative here, but |D_i| <= thr flags it for the exact
    // recomputation below.
#pragma unroll
    for (int c2 = 0; c2 < 2; ++c2) {
      float d[32];
      tmem_ld32(d_qjl + lane_base + (2 * h + c2) * 32, d);
      uint32_t sg = 0u, fl = 0u;
#pragma unroll
      for (int i = 31; i >= 0; --i) {
        sg = __funnelshift_l(__float_as_uint(d[i]), sg, 1);   // (sg << 1) | sign bit
        fl = __funnelshift_l(__float_as_uint(thr - fabsf(d[i])), fl, 1);
      }
      qw[2 * h + c2] = ~sg;
      flag[2 * h + c2] = ~fl;
    }
    if (!writes) flag[0] = flag[1] = flag[2] = flag[3] = 0u;
    if (__any_sync(0xffffffffu, (flag[0] | flag[1] | flag[2] | flag[3]) != 0u)) {
      const Q4 fixed = qjl_fixup<BITS>(d_rot + lane_base, inv, pmid, pb, s_cen, a.s_f32,
                                       Q4{{flag[0], flag[1], flag[2], flag[3]}},
                                       Q4{{qw[0], qw[1], qw[2], qw[3]}});
#pragma unroll
      for (int w = 0; w < 4; ++w) qw[w] = fixed.w[w];
    }
    if (writes) {
      *reinterpret_cast<uint2*>(a.qjl + rec * 4 + 2 * h) = make_uint2(qw[2 * h], qw[2 * h + 1]);
      if (h == 0) a.rnorm[rec] = nrm * rho;
    }
    tc_before_sync();
    grp_sync(gi);
  }
  if (fault) atomicExch(&g_tq_fault, 1);
  tc_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_after_sync();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;\n" ::"r"(tmem) : "memory");
  }
}

// ---------------------------------------------------------------------------
// Warp-specialised form (k_quant_ws): one CTA per SM, persistent over its
// tiles of 128 vectors.  Warp 0 lane 0 loads the raw input tiles (bf16 or
// fp16, no register pass) with TMA into 128B-swizzled slots; warp 1 owns the
// tensor memory and its lane 0 issues the rotations; warp 2 lane 0 issues the
// QJL products; NB epilogue groups of four warps (one thread per vector =
// TMEM lane) take the tiles in turn, tile k in group and rotation buffer
// k % NB (128 TMEM columns each), so NB tiles are in flight.  With QJL, NB =
// 3 and the remaining 128 columns hold the one QJL accumulator, which the
// groups use in tile order; without QJL, NB = 4.
// The rotation multiplies the input as it is stored: bf16 inputs against
// three bf16 terms of 2^8 Pi, fp16 inputs against the fp16 head and tail,
// both to ~24 bits; the norm is taken from the rotated vector (|Pi x| = |x|).
// The epilogue leaves the residual 2^14 r in its rotation columns as fp16
// head and tail, the A operand (from tensor memory) of the QJL product;
// near-zero QJL signs are recomputed in fp32 from head + tail (~22 bits: a
// sign it could still miss lies within 2^-22 |S_i| |r| of zero, inside the
// 1e-5 |r| band of the comparison rule).
// Shared memory: Pi images 96 KB, S 32 KB (with QJL), input slots (three
// with QJL, four without), 1 KB of barriers and tables.
// ---------------------------------------------------------------------------
constexpr uint32_t WS_OFF_S = 3 * SMEM_TILE;
constexpr uint32_t WS_OFF_MISC = 7 * SMEM_TILE;
constexpr uint32_t WS_SMEM = WS_OFF_MISC + 1024 + 1024;   // + 1 KB misc + alignment slack
constexpr uint32_t IDESC_BF16 = tc_idesc_f16(128) | (1u << 7) | (1u << 10);   // A and B bf16
__host__ __device__ constexpr int ws_groups(bool qjl) { return qjl ? 3 : 4; }
__host__ __device__ constexpr int ws_warps(bool qjl) { return 3 + 4 * ws_groups(qjl); }
// barrier slots (8 bytes each) at WS_OFF_MISC: x full / empty [4], rotation
// full / buffer empty / residual ready / QJL done [4 buffers], QJL accumulator
// empty, two drains.  A barrier that several groups wait on at different
// phases would alias its phase parity, so every per-tile signal a group waits
// for has one barrier per buffer (each group waits on its own, in order).
enum : uint32_t { B_XF = 0, B_XE = 4, B_RF = 8, B_TE = 12, B_RR = 16, B_QF = 20, B_QE = 24, B_DONE = 25 };

__device__ __forceinline__ void tma_load_x(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_prefetch_x(const CUtensorMap* map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];\n" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y)
               : "memory");
}

// A bounded wait that also gives up once another role has set *abort.
__device__ __forceinline__ bool ws_wait(uint32_t bar, uint32_t parity, int limit, volatile int* abort) {
  for (int it = 0;; ++it) {
    uint32_t ok;
    if (limit < TC_WAIT_LIMIT)
      asm volatile(
          "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
          "selp.u32 %0, 1, 0, p;\n\t}\n"
          : "=r"(ok)
          : "r"(bar), "r"(parity)
          : "memory");
    else
      asm volatile(
          "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
          "selp.u32 %0, 1, 0, p;\n\t}\n"
          : "=r"(ok)
          : "r"(bar), "r"(parity)
          : "memory");
    if (ok) return true;
    if (*abort != 0 || it + 1 >= limit) return false;
  }
}

// 32 fp32 columns [col, col+32) of this thread's TMEM lane, written.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])),
      "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
      "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])),
      "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
}

// tcgen05.mma kind::f16 with the A operand in tensor memory (lane = row m;
// a K-step of 16 halves in 8 consecutive columns, two per column, the lower
// K index in the low half).
__device__ __forceinline__ void tc_mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %3, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %4, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(accumulate), "r"(idesc));
}

// fp32 signs of the flagged QJL rows from the residual 2^14 r that the
// epilogue left in its rotation columns (taddr) as fp16 head and tail:
// chunk c (coordinates 32 c ..) in columns 32 c .. 32 c + 15 (heads, two per
// column) and 32 c + 16 .. (tails); r = head + tail carries ~22 bits.  Two
// rows per lane per pass; warp-collective like qjl_fixup.
__device__ __noinline__ Q4 qjl_fixup_r(uint32_t taddr, const float* s_f32, Q4 flag, Q4 qw) {
  while (__any_sync(0xffffffffu, (flag.w[0] | flag.w[1] | flag.w[2] | flag.w[3]) != 0u)) {
    int rows[2] = {-1, -1};
#pragma unroll
    for (int q = 0; q < 2; ++q) {
#pragma unroll
      for (int fw = 0; fw < 4; ++fw) {
        if (rows[q] < 0 && flag.w[fw] != 0u) {
          const int bit = __ffs(flag.w[fw]) - 1;
          flag.w[fw] &= flag.w[fw] - 1;
          rows[q] = fw * 32 + bit;
        }
      }
    }
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 1
    for (int ch = 0; ch < 4; ++ch) {
      float d[32];
      tmem_ld32(taddr + ch * 32, d);
      if (rows[0] >= 0) {
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const float2 hh = __half22float2(*reinterpret_cast<const __half2*>(&d[u]));
          const float2 ll = __half22float2(*reinterpret_cast<const __half2*>(&d[16 + u]));
          const float r0 = hh.x + ll.x, r1 = hh.y + ll.y;
          const float* s0 = s_f32 + (size_t)rows[0] * 128 + ch * 32 + 2 * u;
          acc0 = fmaf(__ldg(s0), r0, acc0);
          acc0 = fmaf(__ldg(s0 + 1), r1, acc0);
          if (rows[1] >= 0) {
            const float* s1 = s_f32 + (size_t)rows[1] * 128 + ch * 32 + 2 * u;
            acc1 = fmaf(__ldg(s1), r0, acc1);
            acc1 = fmaf(__ldg(s1 + 1), r1, acc1);
          }
        }
      }
    }
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      if (rows[q] >= 0) {
        const int fw = rows[q] >> 5, bit = rows[q] & 31;
        const bool pos = (q == 0 ? acc0 : acc1) >= 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w)
          if (w == fw) qw.w[w] = (qw.w[w] & ~(1u << bit)) | ((pos ? 1u : 0u) << bit);
      }
    }
  }
  return qw;
}

template <int BITS, bool QJL, bool BF, bool NC = false>
__global__ void __launch_bounds__(ws_warps(QJL) * 32, 1)
    k_quant_ws(const __grid_constant__ CUtensorMap tmx, QuantTcArgs a) {
  static_assert(!(NC && QJL), "norm correction is for MSE-only formats");
  constexpr int NB = ws_groups(QJL);
  constexpr int NPI = BF ? 3 : 2;
  constexpr uint32_t XBASE = QJL ? 4 * SMEM_TILE : 3 * SMEM_TILE;
  constexpr int NX = (int)((WS_OFF_MISC - XBASE) / SMEM_TILE);
  constexpr int L = 1 << BITS;
  constexpr int PER = (BITS == 3) ? 16 : 32 / BITS;
  constexpr int W_MAIN = 128 / PER;
  constexpr int WORDS = (BITS == 3) ? W_MAIN + 4 : W_MAIN;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_s = (uint32_t)__cvta_generic_to_shared(smem_raw);
  const uint32_t base_s = (raw_s + 1023u) & ~1023u;
  unsigned char* base = smem_raw + (base_s - raw_s);
  const uint32_t bars = base_s + WS_OFF_MISC;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(base + WS_OFF_MISC + 256);
  volatile int* s_abort = reinterpret_cast<volatile int*>(base + WS_OFF_MISC + 260);
  float* s_snorm = reinterpret_cast<float*>(base + WS_OFF_MISC + 320);   // [128]
  float* s_cen = s_snorm + 128;                                           // [16]
  float* s_pb = s_cen + 16;                                               // [8]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int NT = ws_warps(QJL) * 32;

  // ---- tables: Pi images, S, QJL row norms, codebook ----------------------------------
  {
    const int4* src_pi = reinterpret_cast<const int4*>(BF ? a.pi_b : a.pi_hi);
    const int4* src_pl = reinterpret_cast<const int4*>(a.pi_lo);
    const int4* src_s = reinterpret_cast<const int4*>(a.s_img);
    int4* dst = reinterpret_cast<int4*>(base);
    constexpr int CH = (int)(SMEM_TILE / 16);
    for (int e = tid; e < CH; e += NT) {
      dst[e] = src_pi[e];
      dst[CH + e] = BF ? src_pi[CH + e] : src_pl[e];
      if (BF) dst[2 * CH + e] = src_pi[2 * CH + e];
      if (QJL) dst[WS_OFF_S / 16 + e] = src_s[e];
    }
    if (tid < 128 && BITS != 8) s_snorm[tid] = QJL ? a.snorm[tid] : 0.f;
    if (tid < 16) s_cen[tid] = tid < L ? a.cen[tid] * (QJL ? 16384.f : 1.f) : 0.f;
    if (BITS <= 4 && tid < 8) s_pb[tid] = (tid < L / 2 - 1) ? a.bnd[L / 2 + tid] : INFINITY;
    if (BITS == 8 && tid < 127) {
      // Breadth-first node tid (level l, position p) holds the threshold of
      // in-order rank (2p + 1) 2^(6 - l) - 1 among the 127 positive ones.
      const int l = 31 - __clz(tid + 1), p = tid + 1 - (1 << l);
      s_snorm[tid] = a.bnd_dev[L / 2 + (2 * p + 1) * (1 << (6 - l)) - 1];
    }
  }
  if (tid == 0) {
    for (int i = 0; i < 4; ++i) {
      mbar_init(bars + 8 * (B_XF + i), 1);
      mbar_init(bars + 8 * (B_XE + i), 1);
      mbar_init(bars + 8 * (B_RF + i), 1);
      mbar_init(bars + 8 * (B_TE + i), 128);
      mbar_init(bars + 8 * (B_RR + i), 128);
      mbar_init(bars + 8 * (B_QF + i), 1);
    }
    mbar_init(bars + 8 * B_QE, 128);
    mbar_init(bars + 8 * B_DONE, 1);
    mbar_init(bars + 8 * (B_DONE + 1), 1);
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;\n" ::"r"(
                     (uint32_t)__cvta_generic_to_shared(s_tmem))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  fence_async_smem();
  tc_before_sync();
  __syncthreads();
  tc_after_sync();
  const uint32_t tmem = *s_tmem;
  const uint32_t d_qjl0 = tmem + 384;   // the QJL accumulator (with QJL)
  const int64_t ntiles = (a.n + TILE - 1) / TILE;
  const int nk = blockIdx.x < ntiles ? (int)((ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x) : 0;
  const int lim = a.wait_limit;
  bool fault = false;

  if (warp == 0) {
    // ---- producer: TMA of the input tiles ------------------------------------------------
    if (lane == 0) {
      int issued = 0;
      for (int k = 0; k < nk && !*s_abort; ++k) {
        const int slot = k % NX;
        if (k >= NX && !ws_wait(bars + 8 * (B_XE + slot), ((k / NX) - 1) & 1, lim, s_abort)) {
          fault = true;
          break;
        }
        const int y = (int)((blockIdx.x + (int64_t)k * gridDim.x) * TILE);
        const uint32_t xf = bars + 8 * (B_XF + slot);
        mbar_expect_tx(xf, SMEM_TILE);
        tma_load_x(base_s + XBASE + slot * SMEM_TILE, &tmx, 0, y, xf);
        tma_load_x(base_s + XBASE + slot * SMEM_TILE + 16384, &tmx, 64, y, xf);
        ++issued;
        if (k + NX < nk) {   // the tile that reuses this slot: into L2 now
          const int y2 = (int)((blockIdx.x + (int64_t)(k + NX) * gridDim.x) * TILE);
          tma_prefetch_x(&tmx, 0, y2);
          tma_prefetch_x(&tmx, 64, y2);
        }
      }
      // drain: the last load of each slot (consumed or not)
      for (int k = issued - 1; k >= 0 && k >= issued - NX; --k)
        mbar_wait(bars + 8 * (B_XF + k % NX), (k / NX) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---- rotation MMAs into buffer k % NB ------------------------------------------------
    if (lane == 0) {
      for (int k = 0; k < nk && !*s_abort; ++k) {
        const int b = k % NB, slot = k % NX;
        if (k >= NB && !ws_wait(bars + 8 * (B_TE + b), ((k / NB) - 1) & 1, lim, s_abort)) {
          fault = true;
          break;
        }
        if (!ws_wait(bars + 8 * (B_XF + slot), (k / NX) & 1, lim, s_abort)) {
          fault = true;
          break;
        }
        tc_after_sync();
        const uint32_t d_rot = tmem + (uint32_t)(b * 128);
        const uint32_t xs = base_s + XBASE + slot * SMEM_TILE;
#pragma unroll
        for (int st = 0; st < 8; ++st) {
          const uint32_t koff = (uint32_t)((st >> 2) * 16384 + (st & 3) * 32);
#pragma unroll
          for (int t = 0; t < NPI; ++t)
            tc_mma_f16(d_rot, smem_desc(xs + koff), smem_desc(base_s + t * SMEM_TILE + koff),
                       BF ? IDESC_BF16 : IDESC, (st | t) ? 1u : 0u);
        }
        tc_commit(bars + 8 * (B_RF + b));
        tc_commit(bars + 8 * (B_XE + slot));
      }
      tc_commit(bars + 8 * B_DONE);   // drain: every MMA issued
      mbar_wait(bars + 8 * B_DONE, 0);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ---- QJL MMAs, tile order, A = the residual in rotation buffer j % NB ----------------
    if (QJL && lane == 0) {
      for (int j = 0; j < nk && !*s_abort; ++j) {
        const int b = j % NB;
        if (!ws_wait(bars + 8 * (B_RR + b), (j / NB) & 1, lim, s_abort) ||
            (j >= 1 && !ws_wait(bars + 8 * B_QE, (j - 1) & 1, lim, s_abort))) {
          fault = true;
          break;
        }
        tc_after_sync();
        const uint32_t a_r = tmem + (uint32_t)(b * 128);
#pragma unroll
        for (int st = 0; st < 8; ++st) {
          const uint32_t koff = (uint32_t)((st >> 2) * 16384 + (st & 3) * 32);
          const uint32_t acol = (uint32_t)(32 * (st >> 1) + 8 * (st & 1));   // heads; tails 16 columns on
          tc_mma_f16_ts(d_qjl0, a_r + acol, smem_desc(base_s + WS_OFF_S + koff), IDESC, st > 0 ? 1u : 0u);
          tc_mma_f16_ts(d_qjl0, a_r + acol + 16, smem_desc(base_s + WS_OFF_S + koff), IDESC, 1u);
        }
        tc_commit(bars + 8 * (B_QF + b));
      }
      tc_commit(bars + 8 * (B_DONE + 1));   // drain
      mbar_wait(bars + 8 * (B_DONE + 1), 0);
    }
    __syncwarp();
  } else {
    // ---- epilogue groups: warps 3 + 4g .. 3 + 4g + 3 take tiles g, g + NB, ... -----------
    const int g = (warp - 3) >> 2, quad = warp & 3;
    const int row = 32 * quad + lane;
    const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
    const float* pb = BITS == 8 ? s_snorm : s_pb;   // 8 bits: the search tree (no QJL rows then)
    const float pmid = (BITS >= 2 && BITS <= 4) ? s_pb[(L >> 2) - 1] : 0.f;
    float snorm_max = 0.f;
    if (QJL)
      for (int i = 0; i < 128; ++i) snorm_max = fmaxf(snorm_max, s_snorm[i]);
    for (int k = g; k < nk; k += NB) {
      const int b = g;
      const int64_t v = (blockIdx.x + (int64_t)k * gridDim.x) * TILE + row;
      const bool live = v < a.n;
      if (__any_sync(0xffffffffu, !ws_wait(bars + 8 * (B_RF + b), (k / NB) & 1, lim, s_abort))) {
        fault = true;
        *s_abort = 1;
        break;
      }
      tc_after_sync();
      const uint32_t d_rot = tmem + (uint32_t)(b * 128) + lane_base;
      float ss[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        float d[32];
        tmem_ld32(d_rot + ch * 32, d);
#pragma unroll
        for (int i = 0; i < 32; ++i) ss[i & 3] = fmaf(d[i], d[i], ss[i & 3]);
      }
      const float nrm_r = sqrtf((ss[0] + ss[1]) + (ss[2] + ss[3]));   // 2^8 |Pi x|
      const float inv = nrm_r > 0.f ? 1.f / nrm_r : 0.f;
      const float nrm = nrm_r * (1.f / 256.f);
      const int64_t rec0 = live ? out_rec(a, v) : -1;
      const bool writes = rec0 >= 0;
      const int64_t rec = writes ? rec0 : 0;
      uint32_t* crow = a.codes + rec * WORDS;
      float rho2v[4] = {0.f, 0.f, 0.f, 0.f};   // |r|^2 with QJL, |c[idx]|^2 under norm correction
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        float d[32];
        tmem_ld32(d_rot + ch * 32, d);
        uint32_t cw[BITS == 8 ? 8 : 4] = {};
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float y = d[i] * inv;
          const int idx = lm_idx<BITS>(y, pmid, pb);
          if (BITS == 3) {
            cw[i >> 4] |= (uint32_t)(idx & 3) << (2 * (i & 15));
            cw[2] |= (uint32_t)(idx >> 2) << i;
          } else {
            cw[i / PER] |= (uint32_t)idx << (BITS * (i % PER));
          }
          if (QJL) {
            const float r = fmaf(y, 16384.f, -s_cen[idx]);   // s_cen holds 2^14 c
            rho2v[i & 3] = fmaf(r, r, rho2v[i & 3]);
            d[i] = r;
          }
          if (NC) {
            const float cj = s_cen[idx];   // s_cen holds c
            rho2v[i & 3] = fmaf(cj, cj, rho2v[i & 3]);
          }
        }
        if (writes) {
          if (BITS == 8) {
            *reinterpret_cast<uint4*>(crow + 8 * ch) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
            *reinterpret_cast<uint4*>(crow + 8 * ch + 4) = make_uint4(cw[4], cw[5], cw[6], cw[7]);
          }
          if (BITS == 4) *reinterpret_cast<uint4*>(crow + 4 * ch) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
          if (BITS == 2) *reinterpret_cast<uint2*>(crow + 2 * ch) = make_uint2(cw[0], cw[1]);
          if (BITS == 1) crow[ch] = cw[0];
          if (BITS == 3) {
            *reinterpret_cast<uint2*>(crow + 2 * ch) = make_uint2(cw[0], cw[1]);
            crow[W_MAIN + ch] = cw[2];
          }
        }
        if (QJL) {
          // The residual as the QJL product's A operand, in place: the chunk's 32 fp32
          // columns become 16 columns of fp16 heads and 16 of tails.
          float o[32];
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const float r0 = d[2 * u], r1 = d[2 * u + 1];
            const __half2 hh = __floats2half2_rn(r0, r1);
            const float2 f = __half22float2(hh);
            o[u] = __uint_as_float(*reinterpret_cast<const uint32_t*>(&hh));
            o[16 + u] = __uint_as_float(h2bits(r0 - f.x, r1 - f.y));
          }
          tmem_st32(d_rot + ch * 32, o);
        }
      }
      if constexpr (!QJL) {
        // Norm correction stores n / |c[idx]|; binary16 norms round the fp32 value.
        const float st = NC ? nrm / sqrtf((rho2v[0] + rho2v[1]) + (rho2v[2] + rho2v[3])) : nrm;
        if (writes) {
          if (a.nf16)
            reinterpret_cast<__half*>(a.norm)[rec] = __float2half_rn(st);
          else
            a.norm[rec] = st;
        }
        tc_before_sync();
        mbar_arrive(bars + 8 * (B_TE + b));
        continue;
      }
      if (writes) a.norm[rec] = nrm;
      tc_before_sync();
      mbar_arrive(bars + 8 * (B_RR + b));   // this lane's residual operand is in place
      const float rho = sqrtf((rho2v[0] + rho2v[1]) + (rho2v[2] + rho2v[3])) * (1.f / 16384.f);
      if (__any_sync(0xffffffffu, !ws_wait(bars + 8 * (B_QF + b), (k / NB) & 1, lim, s_abort))) {
        fault = true;
        *s_abort = 1;
        break;
      }
      tc_after_sync();
      const uint32_t d_q = d_qjl0 + lane_base;
      // D = 2^14 (S r); flag |D_i| <= 2^14 * 2^-17 max_i |S_i| rho (recomputation below).
      const float thr = 0.125f * rho * snorm_max;
      uint32_t qw[4], flag[4];
#pragma unroll 1
      for (int c2 = 0; c2 < 4; ++c2) {
        float d[32];
        tmem_ld32(d_q + c2 * 32, d);
        uint32_t sg = 0u, fl = 0u;
#pragma unroll
        for (int i = 31; i >= 0; --i) {
          sg = __funnelshift_l(__float_as_uint(d[i]), sg, 1);
          fl = __funnelshift_l(__float_as_uint(thr - fabsf(d[i])), fl, 1);
        }
        qw[c2] = ~sg;
        flag[c2] = ~fl;
      }
      tc_before_sync();
      mbar_arrive(bars + 8 * B_QE);   // the QJL accumulator is read: the next tile's product may go
      if (!writes) flag[0] = flag[1] = flag[2] = flag[3] = 0u;
      if (__any_sync(0xffffffffu, (flag[0] | flag[1] | flag[2] | flag[3]) != 0u)) {
        const Q4 fixed = qjl_fixup_r(d_rot, a.s_f32, Q4{{flag[0], flag[1], flag[2], flag[3]}},
                                     Q4{{qw[0], qw[1], qw[2], qw[3]}});
#pragma unroll
        for (int w = 0; w < 4; ++w) qw[w] = fixed.w[w];
      }
      if (writes) {
        *reinterpret_cast<uint4*>(a.qjl + rec * 4) = make_uint4(qw[0], qw[1], qw[2], qw[3]);
        a.rnorm[rec] = nrm * rho;
      }
      tc_before_sync();
      mbar_arrive(bars + 8 * (B_TE + b));
    }
  }
  if (fault) {
    *s_abort = 1;
    atomicExch(&g_tq_fault, 1);
  }
  tc_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_after_sync();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;\n" ::"r"(tmem) : "memory");
  }
}

template <int BITS>
cudaError_t launch_bits(const QuantTcArgs& a, bool qjl, int grid, cudaStream_t s) {
  if (qjl) {
    k_quant_tc<BITS, true><<<grid, 512, TC_SMEM, s>>>(a);
  } else {
    k_quant_tc<BITS, false><<<grid, 512, TC_SMEM, s>>>(a);
  }
  return cudaGetLastError();
}

template <int BITS>
cudaError_t configure_bits() {
  const cudaFuncAttribute ms = cudaFuncAttributeMaxDynamicSharedMemorySize;
  cudaError_t e = cudaFuncSetAttribute(k_quant_tc<BITS, true>, ms, (int)TC_SMEM);
  if (e != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(k_quant_tc<BITS, false>, ms, (int)TC_SMEM))) return e;
  if ((e = cudaFuncSetAttribute(k_quant_ws<BITS, true, true>, ms, (int)WS_SMEM))) return e;
  if ((e = cudaFuncSetAttribute(k_quant_ws<BITS, true, false>, ms, (int)WS_SMEM))) return e;
  if ((e = cudaFuncSetAttribute(k_quant_ws<BITS, false, true>, ms, (int)WS_SMEM))) return e;
  if ((e = cudaFuncSetAttribute(k_quant_ws<BITS, false, false>, ms, (int)WS_SMEM))) return e;
  if ((e = cudaFuncSetAttribute(k_quant_ws<BITS, false, true, true>, ms, (int)WS_SMEM))) return e;
  return cudaFuncSetAttribute(k_quant_ws<BITS, false, false, true>, ms, (int)WS_SMEM);
}

template <int BITS>
cudaError_t launch_ws(const CUtensorMap& map, const QuantTcArgs& a, bool qjl, bool bf, int grid, cudaStream_t s) {
  const dim3 bq(ws_warps(true) * 32), bn(ws_warps(false) * 32);
  if (qjl && bf) k_quant_ws<BITS, true, true><<<grid, bq, WS_SMEM, s>>>(map, a);
  if (qjl && !bf) k_quant_ws<BITS, true, false><<<grid, bq, WS_SMEM, s>>>(map, a);
  const bool nc = a.nc != 0;
  if (!qjl && bf && !nc) k_quant_ws<BITS, false, true><<<grid, bn, WS_SMEM, s>>>(map, a);
  if (!qjl && !bf && !nc) k_quant_ws<BITS, false, false><<<grid, bn, WS_SMEM, s>>>(map, a);
  if (!qjl && bf && nc) k_quant_ws<BITS, false, true, true><<<grid, bn, WS_SMEM, s>>>(map, a);
  if (!qjl && !bf && nc) k_quant_ws<BITS, false, false, true><<<grid, bn, WS_SMEM, s>>>(map, a);
  return cudaGetLastError();
}

cudaError_t launch_ws8(const CUtensorMap& map, const QuantTcArgs& a, bool bf, int grid, cudaStream_t s) {
  const dim3 bn(ws_warps(false) * 32);
  if (bf)
    k_quant_ws<8, false, true><<<grid, bn, WS_SMEM, s>>>(map, a);
  else
    k_quant_ws<8, false, false><<<grid, bn, WS_SMEM, s>>>(map, a);
  return cudaGetLastError();
}

// cuTensorMapEncodeTiled through the runtime's driver entry point.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Input rows [n][ld] (16-bit), the first 128 of each row: boxes of 64 x 128,
// 128-byte swizzle (the K-major operand layout of chunk_off); rows past n read
// as zeros.
bool make_x_map(CUtensorMap* map, const QuantTcArgs& a) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[2] = {128, (cuuint64_t)a.n};
  const cuuint64_t strides[1] = {(cuuint64_t)a.ld * 2};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t es[2] = {1, 1};
  const CUtensorMapDataType t = a.dtype == TQ_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  return fn(map, t, 2, const_cast<void*>(a.x), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t read_and_clear_fault(int* value) {
  cudaError_t e = cudaMemcpyFromSymbol(value, g_tq_fault, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_tq_fault, &zero, sizeof(int));
}

cudaError_t configure_quant_tc() {
  cudaError_t e;
  if ((e = configure_bits<1>()) != cudaSuccess) return e;
  if ((e = configure_bits<2>()) != cudaSuccess) return e;
  if ((e = configure_bits<3>()) != cudaSuccess) return e;
  if ((e = configure_bits<4>()) != cudaSuccess) return e;
  const cudaFuncAttribute ms = cudaFuncAttributeMaxDynamicSharedMemorySize;
  if ((e = cudaFuncSetAttribute(k_quant_ws<8, false, true>, ms, (int)WS_SMEM))) return e;
  return cudaFuncSetAttribute(k_quant_ws<8, false, false>, ms, (int)WS_SMEM);
}

bool quant_ws_eligible(const QuantTcArgs& a) {
  if ((a.nc || a.nf16) && a.m != 0) return false;   // MSE-only variants
  if (a.bits == 8 && (a.m != 0 || a.nc || !a.bnd_dev)) return false;   // 8 bits: plain MSE codes only
  return a.pi_b && (a.dtype == TQ_BF16 || a.dtype == TQ_F16) && (reinterpret_cast<uintptr_t>(a.x) & 15) == 0 &&
         (a.ld * 2) % 16 == 0 && a.n < ((int64_t)1 << 31) - TILE;
}

cudaError_t launch_quant_tc(const QuantTcArgs& a_in, int sms, cudaStream_t s) {
  QuantTcArgs a = a_in;
  if (a.wait_limit <= 0) a.wait_limit = TC_WAIT_LIMIT;
  const int64_t tiles = (a.n + TILE - 1) / TILE;
  CUtensorMap map;
  const bool ws = quant_ws_eligible(a) && make_x_map(&map, a);
  if (a.bits == 8) {   // the warp-specialised kernel only
    if (!ws) return cudaErrorNotSupported;
    const int grid = (int)(tiles < sms ? tiles : sms);
    return launch_ws8(map, a, a.dtype == TQ_BF16, grid, s);
  }
  if (ws) {
    const int grid = (int)(tiles < sms ? tiles : sms);
    const bool qjl = a.m > 0, bf = a.dtype == TQ_BF16;
    switch (a.bits) {
      case 1: return launch_ws<1>(map, a, qjl, bf, grid, s);
      case 2: return launch_ws<2>(map, a, qjl, bf, grid, s);
      case 3: return launch_ws<3>(map, a, qjl, bf, grid, s);
      case 4: return launch_ws<4>(map, a, qjl, bf, grid, s);
      default: return cudaErrorInvalidValue;
    }
  }
  // The register-staged form writes plain fp32 norms only.
  if (a.nc || a.nf16) return cudaErrorNotSupported;
  int64_t grid = (tiles + 1) / 2;
  if (grid > sms) grid = sms;
  if (grid < 1) grid = 1;
  const bool qjl = a.m > 0;
  switch (a.bits) {
    case 1: return launch_bits<1>(a, qjl, (int)grid, s);
    case 2: return launch_bits<2>(a, qjl, (int)grid, s);
    case 3: return launch_bits<3>(a, qjl, (int)grid, s);
    case 4: return launch_bits<4>(a, qjl, (int)grid, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tqk
