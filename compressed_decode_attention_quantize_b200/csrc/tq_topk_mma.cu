// Inner-product top-k over a compressed database on the tensor cores
// (sm_100a, mma.sync).  "What is TurboQuant?", section "Benchmarks": nearest
// neighbour search scores every database vector from its codes,
//   score(q, v) = n_v <q', c[idx_v]> + sqrt(pi/2)/m * gamma_v <S q', sigma_v>,
// and keeps the k best (score descending, then index ascending).
//
// The scores form a dense contraction of the queries with the dequantized
// database: per 64-vector database tile the CTA expands the codes into fp16
// rows [c[idx] (d, padded to 16) | sigma (m, padded to 16)] in shared memory,
// and four warps multiply them with 64 queries ([q' 2^-e_q | S q' 2^-f_q] in
// fp16, loaded once) with mma.sync m16n8k16, two fp32 accumulators (centroid
// part, sign part).  fp16 rounding of q', S q' and the centroids moves a score
// by ~1e-5 |q| |k|, far below the logit tolerance that separates
// interchangeable near-ties.  Each warp keeps a top-k list per query in shared
// memory; a score enters only if it beats the list's current worst, so after
// the first tiles almost every score costs one comparison.  The lists of all
// warps and database chunks are merged by k_topk_final.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>

#include "tq_internal.h"

namespace tqk {
namespace {

constexpr int TKR = 64;     // database vectors per tile
constexpr int TKWARPS = 8;  // warp w: rows 16 (w & 3) .. +15, queries QB/2 (w >> 2) .. + QB/2 - 1
constexpr int TKLISTS = 4;  // lists per query and chunk (the four row groups)

__device__ __forceinline__ bool better_sc(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

__device__ __forceinline__ void cp4(void* dst, const void* src) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(d), "l"(src) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Query operands: row q = [q' 2^-e (KL) | S q' 2^-f (KQ)] in fp16, zero padded,
// and the scales 2^e, 2^f (powers of two: the fp16 values are q' and S q'
// rounded once).  One warp per query.
__global__ void __launch_bounds__(128) k_topk_qprep(const float* qr, const float* qs, int64_t nq, int d,
                                                    int dpad, int m, int KL, int KQ, __half* qh,
                                                    float* qsc) {
  const int64_t q = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (q >= nq) return;
  float mq = 0.f, ms = 0.f;
  for (int j = lane; j < d; j += 32) mq = fmaxf(mq, fabsf(qr[q * dpad + j]));
  for (int j = lane; j < m; j += 32) ms = fmaxf(ms, fabsf(qs[q * dpad + j]));
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    mq = fmaxf(mq, __shfl_xor_sync(0xffffffffu, mq, o));
    ms = fmaxf(ms, __shfl_xor_sync(0xffffffffu, ms, o));
  }
  const int e = mq > 0.f ? ilogbf(mq) : 0, f = ms > 0.f ? ilogbf(ms) : 0;
  const float se = ldexpf(1.f, -e), sf = ldexpf(1.f, -f);
  __half* row = qh + q * (KL + KQ);
  for (int j = lane; j < KL; j += 32) row[j] = __float2half_rn(j < d ? qr[q * dpad + j] * se : 0.f);
  for (int j = lane; j < KQ; j += 32) row[KL + j] = __float2half_rn(j < m ? qs[q * dpad + j] * sf : 0.f);
  if (lane == 0) {
    qsc[2 * q] = ldexpf(1.f, e);
    qsc[2 * q + 1] = ldexpf(1.f, f);
  }
}

struct TopkMmaArgs {
  const __half* qh;
  const float* qsc;
  int64_t nq;
  int d, bk, kw, m, qw, KL, KQ;
  const float* ck;
  float cq;   // sqrt(pi/2) / m
  const uint32_t* codes;
  const uint32_t* qjl;
  const float* norm;
  const float* rnorm;
  int64_t n, chunk;   // database size, vectors per chunk (multiple of TKR)
  int64_t chunks, qblocks;   // work items = qblocks x chunks, taken round-robin
  int K, nlists;
  float* cand_v;
  int* cand_i;
  // Optional starting bar per query: entry (q, K - 1) of bar_v / bar_i
  // ([nq][K], index -1 = none), the k-th best of a sample of the database.
  const float* bar_v;
  const int* bar_i;
};

// Shared memory for QB queries per CTA: B rows [QB][KS] and A rows [TKR][KS]
// in fp16 (KS = KL + KQ + 8: an odd number of 16-byte chunks per row, so
// ldmatrix rows hit distinct banks), two staging buffers of the tile's codes,
// signs and norms, query scales, the pair table (two coordinates' indices ->
// half2 of centroids, up to 256 entries) and the per-warp lists
// [TKWARPS][QB / 2][K] of (score, index).
__host__ __device__ inline size_t topk_mma_smem(int QB, int KL, int KQ, int kw, int qw, int K) {
  const size_t KS = (size_t)KL + KQ + 8;
  return 2 * KS * (QB + TKR) + 2 * (size_t)TKR * (kw + qw + 2) * 4 + (size_t)QB * 2 * 4 + 256 * 4 +
         (size_t)TKWARPS * (QB / 2) * K * 8 + 64;
}

template <int BK, int QB>
__global__ void __launch_bounds__(TKWARPS * 32) k_topk_mma(TopkMmaArgs a) {
  constexpr int QH = QB / 2;     // queries per warp
  constexpr int NTW = QH / 8;    // n-tiles per warp
  constexpr int SL = 2 * NTW;    // (query) slots per thread
  extern __shared__ __align__(16) unsigned char smem[];
  const int KS = a.KL + a.KQ + 8;
  __half* sB = reinterpret_cast<__half*>(smem);
  __half* sA = sB + (size_t)QB * KS;
  // Two staging buffers (tile i and i + 1): codes [TKR][kw], signs [TKR][qw],
  // norms [TKR], rnorms [TKR].
  const int stage_words = TKR * (a.kw + a.qw + 2);
  uint32_t* sStage = reinterpret_cast<uint32_t*>(sA + (size_t)TKR * KS);
  float* sQ = reinterpret_cast<float*>(sStage + 2 * stage_words);       // [QB][2]: 2^e, 2^f
  uint32_t* sP = reinterpret_cast<uint32_t*>(sQ + QB * 2);               // [256] pair table
  float* lv = reinterpret_cast<float*>(sP + 256);                        // [TKWARPS][QH][K]
  int* li = reinterpret_cast<int*>(lv + TKWARPS * QH * a.K);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int rg = warp & 3, qg = warp >> 2;   // row group, query half
  const int KP = a.KL + a.KQ;
  constexpr int bk = BK;
  // Code words: main (b = 3: low-bit) stream of W2 words with `per` fields each.
  constexpr int per = bk == 3 ? 16 : 32 / bk;
  constexpr int fb = bk == 3 ? 2 : bk;       // bits per field in the main stream
  constexpr int pairs_w = per / 2;           // coordinate pairs per word
  const int W2 = (a.d + per - 1) / per;

  // Pair table: entry i -> half2(c[i0], c[i1]); for b = 3, i = f0 | f1 << 2 |
  // t0 << 4 | t1 << 5 (fields, then top bits), else i = i0 | i1 << b.
  for (int e = tid; e < 256; e += TKWARPS * 32) {
    int i0, i1;
    if (bk == 3) {
      i0 = (e & 3) | (((e >> 4) & 1) << 2);
      i1 = ((e >> 2) & 3) | (((e >> 5) & 1) << 2);
    } else {
      i0 = e & ((1 << bk) - 1);
      i1 = (e >> bk) & ((1 << bk) - 1);
    }
    const bool ok = bk == 3 ? e < 64 : e < (1 << (2 * bk));
    const __half2 hv = __floats2half2_rn(ok ? a.ck[i0] : 0.f, ok ? a.ck[i1] : 0.f);
    sP[e] = *reinterpret_cast<const uint32_t*>(&hv);
  }
  // Centroid columns past the code words (d < KL with < 16 fields per word):
  // zero once, no tile writes them.
  for (int e = tid; e < TKR * KS; e += TKWARPS * 32) sA[e] = __float2half_rn(0.f);

  const uint32_t sA_s = (uint32_t)__cvta_generic_to_shared(sA);
  const uint32_t sB_s = (uint32_t)__cvta_generic_to_shared(sB);
  // ldmatrix row addresses: A tiles (rows 0-7 / 8-15) x (k 0-7 / 8-15);
  // B tiles (n-tile nt / nt+1) x (k 0-7 / 8-15) of this warp's 32 queries.
  const int ti = lane >> 3, tr = lane & 7;
  const uint32_t a_row = sA_s + (uint32_t)((16 * rg + tr + 8 * (ti & 1)) * KS + 8 * (ti >> 1)) * 2;
  const uint32_t b_row = sB_s + (uint32_t)((QH * qg + 8 * (ti >> 1) + tr) * KS + 8 * (ti & 1)) * 2;
  float* mylv = lv + warp * QH * a.K;
  int* myli = li + warp * QH * a.K;

  // Persistent CTAs: item = (query block, database chunk).
  const int64_t nitems = a.qblocks * a.chunks;
  for (int64_t item = blockIdx.x; item < nitems; item += gridDim.x) {
  const int64_t q0 = (item / a.chunks) * QB;
  const int64_t chunk_id = item % a.chunks;
  const int64_t n0 = chunk_id * a.chunk;
  const int64_t n1 = min(a.n, n0 + a.chunk);
  __syncthreads();   // the previous item's readers of sB, sQ and the lists are done
  for (int e = tid; e < QB * KP / 8; e += TKWARPS * 32) {
    const int r = e / (KP / 8), c8 = e % (KP / 8);
    uint4 v = make_uint4(0, 0, 0, 0);
    if (q0 + r < a.nq) v = reinterpret_cast<const uint4*>(a.qh + (q0 + r) * KP)[c8];
    *reinterpret_cast<uint4*>(sB + (size_t)r * KS + 8 * c8) = v;
  }
  for (int e = tid; e < QB * 2; e += TKWARPS * 32) sQ[e] = (q0 + e / 2 < a.nq) ? a.qsc[q0 * 2 + e] : 0.f;
  // Lists start at the query's bar: every final top-k entry is at least as
  // good as the k-th best of any subset, so nothing below it can enter.
  auto bar = [&](int64_t q, float& v, int& i) {
    v = -INFINITY;
    i = INT_MAX;
    if (a.bar_v && q < a.nq) {
      const int bi = a.bar_i[q * a.K + a.K - 1];
      if (bi >= 0) {
        v = a.bar_v[q * a.K + a.K - 1];
        i = bi;
      }
    }
  };
  for (int e = tid; e < TKWARPS * QH * a.K; e += TKWARPS * 32) {
    const int ql = (e / a.K) % QH, w = e / (QH * a.K);
    bar(q0 + QH * (w >> 2) + ql, lv[e], li[e]);
  }
  __syncthreads();
  // This thread's SL queries (NTW n-tiles x 2 columns): scales and the current
  // worst entry of their lists.
  float fe[SL], ff[SL], wv[SL];
  int wi[SL];
#pragma unroll
  for (int s = 0; s < SL; ++s) {
    const int ql = QH * qg + 8 * (s >> 1) + 2 * t + (s & 1);
    fe[s] = sQ[2 * ql];
    ff[s] = sQ[2 * ql + 1];
    bar(q0 + ql, wv[s], wi[s]);
  }

  // Copy tile v0's codes, signs and norms (contiguous in memory) into staging
  // buffer buf with 4-byte cp.async: in flight while the previous tile is
  // scored.
  auto stage = [&](int64_t v0, int buf) {
    const int rows = (int)min((int64_t)TKR, n1 - v0);
    uint32_t* dC = sStage + buf * stage_words;
    uint32_t* dS = dC + TKR * a.kw;
    uint32_t* dN = dS + TKR * a.qw;
    for (int e = tid; e < rows * a.kw; e += TKWARPS * 32) cp4(dC + e, a.codes + v0 * a.kw + e);
    for (int e = tid; e < rows * a.qw; e += TKWARPS * 32) cp4(dS + e, a.qjl + v0 * a.qw + e);
    for (int e = tid; e < rows; e += TKWARPS * 32) {
      cp4(dN + e, a.norm + v0 + e);
      if (a.m > 0) cp4(dN + TKR + e, a.rnorm + v0 + e);
    }
    asm volatile("cp.async.commit_group;\n" ::);
  };
  if (n0 < n1) stage(n0, 0);
  int buf = 0;
  for (int64_t v0 = n0; v0 < n1; v0 += TKR, buf ^= 1) {
    const int rows = (int)min((int64_t)TKR, n1 - v0);
    asm volatile("cp.async.wait_group 0;\n" ::: "memory");
    __syncthreads();   // tile v0 staged; the other buffer is free
    if (v0 + TKR < n1) stage(v0 + TKR, buf ^ 1);
    const uint32_t* sC = sStage + buf * stage_words;
    const uint32_t* sS = sC + TKR * a.kw;
    const float* sNn = reinterpret_cast<const float*>(sS + TKR * a.qw);   // norms, then rnorms
    // ---- dequantize: thread -> row tid % 64, code words tid / 64, +4, ... -----------
    {
      const int r = tid & (TKR - 1);
      const bool live = r < rows;
      for (int wd = tid >> 6; wd < W2; wd += TKWARPS * 32 / TKR) {
        uint32_t* dst = reinterpret_cast<uint32_t*>(sA + (size_t)r * KS) + wd * pairs_w;
        const uint32_t w = live ? sC[r * a.kw + wd] : 0u;
        uint32_t tw = 0u;
        if (bk == 3 && live) tw = sC[r * a.kw + W2 + (wd >> 1)] >> (16 * (wd & 1));
        if (live && per * (wd + 1) <= a.d) {   // every coordinate of the word is real
#pragma unroll
          for (int j = 0; j < pairs_w; ++j) {
            uint32_t idx = (w >> (2 * fb * j)) & ((1u << (2 * fb)) - 1u);
            if (bk == 3) idx |= ((tw >> (2 * j)) & 3u) << 4;
            dst[j] = sP[idx];
          }
        } else {
#pragma unroll
          for (int j = 0; j < pairs_w; ++j) {
            const int c = per * wd + 2 * j;   // first coordinate of the pair
            uint32_t idx = (w >> (2 * fb * j)) & ((1u << (2 * fb)) - 1u);
            if (bk == 3) idx |= ((tw >> (2 * j)) & 3u) << 4;
            uint32_t h2 = sP[idx];
            if (!live || c >= a.d) h2 = 0u;
            else if (c + 1 >= a.d) h2 &= 0xFFFFu;
            if (c < a.KL) dst[j] = h2;
          }
        }
      }
      for (int wd = tid >> 6; wd < a.qw; wd += TKWARPS * 32 / TKR) {
        uint32_t* dst = reinterpret_cast<uint32_t*>(sA + (size_t)r * KS + a.KL) + wd * 16;
        const uint32_t bits = live ? sS[r * a.qw + wd] : 0u;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int c = 32 * wd + 2 * j;   // first sketch row of the pair
          const uint32_t b2 = bits >> (2 * j);
          // -1 (0xBC00) per half, +1 where the bit is set: flip the sign bit.
          uint32_t h2 = 0xBC00BC00u ^ ((b2 & 1u) << 15) ^ ((b2 & 2u) << 30);
          if (!live || c >= a.m) h2 = 0u;
          else if (c + 1 >= a.m) h2 &= 0xFFFFu;
          if (c < a.KQ) dst[j] = h2;
        }
      }
    }
    __syncthreads();

    // ---- scores of rows 16 rg .. +15 against queries QH qg .. + QH - 1 -------------------
    float acc[NTW][4], acs[NTW][4];
#pragma unroll
    for (int nt = 0; nt < NTW; ++nt)
#pragma unroll
      for (int r = 0; r < 4; ++r) acc[nt][r] = acs[nt][r] = 0.f;
    for (int ks = 0; ks < a.KL / 16; ++ks) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(a_row + ks * 32, a0, a1, a2, a3);
#pragma unroll
      for (int np = 0; np < NTW / 2; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(b_row + (uint32_t)(16 * np * KS) * 2 + ks * 32, b0, b1, b2, b3);
        mma_f16(acc[2 * np], a0, a1, a2, a3, b0, b1);
        mma_f16(acc[2 * np + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    for (int ks = a.KL / 16; ks < KP / 16; ++ks) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(a_row + ks * 32, a0, a1, a2, a3);
#pragma unroll
      for (int np = 0; np < NTW / 2; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(b_row + (uint32_t)(16 * np * KS) * 2 + ks * 32, b0, b1, b2, b3);
        mma_f16(acs[2 * np], a0, a1, a2, a3, b0, b1);
        mma_f16(acs[2 * np + 1], a0, a1, a2, a3, b2, b3);
      }
    }

    // ---- candidates: slot s = 2 nt + col (query QH qg + 8 nt + 2 t + col) ----------
    const int ra = 16 * rg + g, rb = ra + 8;
    const bool va = ra < rows, vb = rb < rows;
    const float na = va ? sNn[ra] : 0.f, ga = (va && a.m > 0) ? sNn[TKR + ra] * a.cq : 0.f;
    const float nb = vb ? sNn[rb] : 0.f, gb = (vb && a.m > 0) ? sNn[TKR + rb] * a.cq : 0.f;
    float sc[SL][2];
    uint32_t mask = 0u;
#pragma unroll
    for (int nt = 0; nt < NTW; ++nt) {
#pragma unroll
      for (int col = 0; col < 2; ++col) {
        const int s = 2 * nt + col;
        sc[s][0] = va ? fmaf(na * fe[s], acc[nt][col], ga * ff[s] * acs[nt][col]) : -INFINITY;
        sc[s][1] = vb ? fmaf(nb * fe[s], acc[nt][2 + col], gb * ff[s] * acs[nt][2 + col]) : -INFINITY;
        if (va && better_sc(sc[s][0], (int)(v0 + ra), wv[s], wi[s])) mask |= 1u << (2 * s);
        if (vb && better_sc(sc[s][1], (int)(v0 + rb), wv[s], wi[s])) mask |= 1u << (2 * s + 1);
      }
    }
    // Insert the candidates one at a time (rare once the lists fill): the
    // lowest lane holding one and its lowest (slot, row) bit; lane 0 updates
    // the list, and the lanes holding that query take its new worst entry.
    while (__any_sync(0xffffffffu, mask != 0u)) {
      const int leader = __ffs(__ballot_sync(0xffffffffu, mask != 0u)) - 1;
      const int bit = __shfl_sync(0xffffffffu, __ffs(mask) - 1, leader);
      const int s = bit >> 1, row = bit & 1, lt = leader & 3;
      float mine = 0.f;
#pragma unroll
      for (int k = 0; k < 2 * SL; ++k)
        if (k == bit) mine = sc[k >> 1][k & 1];
      const float val = __shfl_sync(0xffffffffu, mine, leader);
      const int idx = (int)(v0 + 16 * rg + (leader >> 2) + 8 * row);
      const int ql = 8 * (s >> 1) + 2 * lt + (s & 1);   // within this warp's QH queries
      if (lane == leader) mask &= mask - 1u;
      float nwv = 0.f;
      int nwi = 0;
      if (lane == 0) {
        float* L = mylv + ql * a.K;
        int* I = myli + ql * a.K;
        int wpos = 0;
        for (int e = 1; e < a.K; ++e)
          if (better_sc(L[wpos], I[wpos], L[e], I[e])) wpos = e;
        if (better_sc(val, idx, L[wpos], I[wpos])) {
          L[wpos] = val;
          I[wpos] = idx;
          wpos = 0;
          for (int e = 1; e < a.K; ++e)
            if (better_sc(L[wpos], I[wpos], L[e], I[e])) wpos = e;
        }
        nwv = L[wpos];
        nwi = I[wpos];
      }
      nwv = __shfl_sync(0xffffffffu, nwv, 0);
      nwi = __shfl_sync(0xffffffffu, nwi, 0);
      if (t == lt) {
        // Raise this query's bar and drop the candidates it no longer passes.
#pragma unroll
        for (int k = 0; k < SL; ++k) {
          if (k == s) {
            wv[k] = nwv;
            wi[k] = nwi;
            if (!better_sc(sc[k][0], (int)(v0 + 16 * rg + g), nwv, nwi)) mask &= ~(1u << (2 * k));
            if (!better_sc(sc[k][1], (int)(v0 + 16 * rg + g + 8), nwv, nwi)) mask &= ~(1u << (2 * k + 1));
          }
        }
      }
      __syncwarp();
    }
    __syncthreads();   // the next tile overwrites sA
  }
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");

  // ---- this warp's lists -> candidates of (query, chunk, row group) ------------------
  const int list = (int)chunk_id * TKLISTS + rg;
  for (int e = lane; e < QH * a.K; e += 32) {
    const int ql = e / a.K, r = e % a.K;
    const int64_t q = q0 + QH * qg + ql;
    if (q < a.nq) {
      const int64_t o = (q * a.nlists + list) * a.K + r;
      a.cand_v[o] = mylv[ql * a.K + r];
      a.cand_i[o] = myli[ql * a.K + r];
    }
  }
  }
}

}  // namespace

TopkPlan topk_mma_plan(const tq_ctx* c, int64_t nq, int64_t n, int k) {
  TopkPlan p{};
  p.KL = (c->d + 15) / 16 * 16;
  p.KQ = (c->qjl_m + 15) / 16 * 16;
  const int qw = (c->qjl_m + 31) / 32;
  // 128 queries per CTA (more products per dequantized tile) when it fits.
  p.qb = topk_mma_smem(128, p.KL, p.KQ, c->wk, qw, k) <= (size_t)227 * 1024 ? 128 : 64;
  const int64_t qblocks = (nq + p.qb - 1) / p.qb;
  // About sixteen (query block, chunk) items per SM for the persistent grid.
  int64_t chunks = (16 * (int64_t)c->sms + qblocks - 1) / (qblocks > 0 ? qblocks : 1);
  const int64_t max_chunks = (n + 8 * TKR - 1) / (8 * TKR);   // at least eight tiles per chunk
  if (chunks > max_chunks) chunks = max_chunks;
  if (chunks < 1) chunks = 1;
  if (chunks > 65535) chunks = 65535;
  p.chunks = chunks;
  p.chunk = ((n + chunks - 1) / chunks + TKR - 1) / TKR * TKR;
  p.chunks = (n + p.chunk - 1) / p.chunk;   // no empty chunk after rounding
  p.qblocks = qblocks;
  p.nlists = (int)(p.chunks * TKLISTS);
  p.qh_bytes = (size_t)nq * (p.KL + p.KQ) * sizeof(__half);
  p.qsc_bytes = (size_t)nq * 2 * sizeof(float);
  p.cand_bytes = (size_t)nq * p.nlists * k * (sizeof(float) + sizeof(int));
  p.smem = topk_mma_smem(p.qb, p.KL, p.KQ, c->wk, qw, k);
  return p;
}

TopkPlan topk_mma_sample_plan(const TopkPlan& full, int64_t n_sample, int sms) {
  TopkPlan p = full;
  int64_t chunks = (sms + p.qblocks - 1) / p.qblocks;   // about one item per SM
  const int64_t max_chunks = (n_sample + 8 * TKR - 1) / (8 * TKR);
  if (chunks > max_chunks) chunks = max_chunks;
  if (chunks < 1) chunks = 1;
  p.chunk = ((n_sample + chunks - 1) / chunks + TKR - 1) / TKR * TKR;
  p.chunks = (n_sample + p.chunk - 1) / p.chunk;
  p.nlists = (int)(p.chunks * TKLISTS);
  return p;
}

cudaError_t launch_topk_qprep(const tq_ctx* c, const TopkPlan& p, const float* qr, const float* qs,
                              int64_t nq, void* qh, float* qsc, cudaStream_t s) {
  k_topk_qprep<<<(unsigned)((nq + 3) / 4), 128, 0, s>>>(qr, qs, nq, c->d, c->dpad, c->qjl_m, p.KL, p.KQ,
                                                          static_cast<__half*>(qh), qsc);
  return cudaGetLastError();
}

cudaError_t launch_topk_mma(const tq_ctx* c, const TopkPlan& p, const void* qh, const float* qsc, int64_t nq,
                            const uint32_t* codes, const uint32_t* qjl, const float* norm,
                            const float* rnorm, int64_t n, int k, const float* bar_v, const int* bar_i,
                            float* cand_v, int* cand_i, cudaStream_t s) {
  TopkMmaArgs a{};
  a.qh = static_cast<const __half*>(qh);
  a.qsc = qsc;
  a.nq = nq;
  a.d = c->d;
  a.bk = c->bk_lm;
  a.kw = c->wk;
  a.m = c->qjl_m;
  a.qw = (c->qjl_m + 31) / 32;
  a.KL = p.KL;
  a.KQ = p.KQ;
  a.ck = c->ck_f;
  a.cq = c->qjl_m > 0 ? (float)(std::sqrt(M_PI / 2.0) / c->qjl_m) : 0.f;
  a.codes = codes;
  a.qjl = qjl;
  a.norm = norm;
  a.rnorm = rnorm;
  a.n = n;
  a.chunk = p.chunk;
  a.K = k;
  a.nlists = p.nlists;
  a.cand_v = cand_v;
  a.cand_i = cand_i;
  a.chunks = p.chunks;
  a.qblocks = p.qblocks;
  a.bar_v = bar_v;
  a.bar_i = bar_i;
  const int64_t items = p.qblocks * p.chunks;
  const unsigned grid = (unsigned)(items < c->sms ? items : c->sms);   // one CTA per SM
  const bool wide = p.qb == 128;
  switch (c->bk_lm * 2 + (wide ? 1 : 0)) {
    case 2: k_topk_mma<1, 64><<<grid, TKWARPS * 32, p.smem, s>>>(a); break;
    case 3: k_topk_mma<1, 128><<<grid, TKWARPS * 32, p.smem, s>>>(a); break;
    case 4: k_topk_mma<2, 64><<<grid, TKWARPS * 32, p.smem, s>>>(a); break;
    case 5: k_topk_mma<2, 128><<<grid, TKWARPS * 32, p.smem, s>>>(a); break;
    case 6: k_topk_mma<3, 64><<<grid, TKWARPS * 32, p.smem, s>>>(a); break;
    case 7: k_topk_mma<3, 128><<<grid, TKWARPS * 32, p.smem, s>>>(a); break;
    case 8: k_topk_mma<4, 64><<<grid, TKWARPS * 32, p.smem, s>>>(a); break;
    case 9: k_topk_mma<4, 128><<<grid, TKWARPS * 32, p.smem, s>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t configure_topk_mma() {
  const int lim = 227 * 1024;   // the plan never asks for more
  const cudaFuncAttribute ms = cudaFuncAttributeMaxDynamicSharedMemorySize;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(k_topk_mma<1, 64>, ms, lim))) return e;
  if ((e = cudaFuncSetAttribute(k_topk_mma<1, 128>, ms, lim))) return e;
  if ((e = cudaFuncSetAttribute(k_topk_mma<2, 64>, ms, lim))) return e;
  if ((e = cudaFuncSetAttribute(k_topk_mma<2, 128>, ms, lim))) return e;
  if ((e = cudaFuncSetAttribute(k_topk_mma<3, 64>, ms, lim))) return e;
  if ((e = cudaFuncSetAttribute(k_topk_mma<3, 128>, ms, lim))) return e;
  if ((e = cudaFuncSetAttribute(k_topk_mma<4, 64>, ms, lim))) return e;
  return cudaFuncSetAttribute(k_topk_mma<4, 128>, ms, lim);
}

}  // namespace tqk
