// Inner-product top-k over a compressed database on the tensor cores
// (sm_100a, mma.sync).  "What is TurboQuant?", section "Benchmarks": nearest
// neighbour search scores every database vector from its codes,
//   score(q, v) = n_v <q', c[idx_v]> + sqrt(pi/2)/m * gamma_v <S q', sigma_v>,
// and keeps the k best (score descending, then index ascending).
//
// The scores form a dense contraction of the queries with the dequantized
// database.  k_topk_dequant expands every vector's codes once into an fp16
// row [c[idx] (d, padded to 16) | sigma (m, padded to 16)] in global memory
// (a pair table maps two coordinates' indices to a half2 of centroids).
// k_topk_gemm streams 32-row tiles of those rows through a three-stage
// cp.async ring into shared memory and multiplies them with up to 128 queries
// ([q' 2^-e_q | S q' 2^-f_q] in fp16, loaded once per work item) with
// mma.sync m16n8k16 into two fp32 accumulators (centroid part, sign part);
// n and sqrt(pi/2)/m gamma are applied per row in fp32.  Work items (query
// block, database chunk) run chunk-major on a persistent grid, so the CTAs
// in flight read the same few chunks and the rows come from L2.  fp16
// rounding of q', S q' and the centroids moves a score by ~1e-5 |q| |k|, far
// below the logit tolerance that separates interchangeable near-ties.  Each
// warp keeps a top-k list per query in shared memory; a score enters only if
// it beats the list's current worst.  The lists of all warps and chunks are
// merged by k_topk_final.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>

#include "tq_internal.h"

namespace tqk {
namespace {

constexpr int TKR = 32;     // database vectors per tile
constexpr int TKWARPS = 8;  // warp w: rows 16 (w & 1) .. +15, queries QB/4 (w >> 1) .. + QB/4 - 1
constexpr int TKLISTS = 2;  // lists per query and chunk (the two row groups)
constexpr int TKST = 3;     // tile stages in flight

__device__ __forceinline__ bool better_sc(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

__device__ __forceinline__ void cp4(void* dst, const void* src, bool valid) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(d), "l"(src), "r"(valid ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cp16z(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
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
  int KL, KQ, m;
  float cq;   // sqrt(pi/2) / m
  const __half* rows;   // dequantized database [n][KL + KQ]
  const float* norm;     // binary16 values when nf16
  const float* rnorm;
  int nf16;
  int64_t n, chunk;   // database size, vectors per chunk (multiple of TKR)
  int64_t chunks, qblocks;   // work items = chunks x qblocks, chunk-major
  int K, nlists;
  float* cand_v;
  int* cand_i;
  // Optional starting bar per query: entry (q, K - 1) of bar_v / bar_i
  // ([nq][K], index -1 = none), the k-th best of a sample of the database.
  const float* bar_v;
  const int* bar_i;
};

// Database rows: thread task (v, w) writes the half2 pairs of code word w of
// vector v (w < W2), the +-1 halves of sign word w - W2 (w < W2 + qw), or
// zeros for centroid columns past the code words (last task).
template <int BK>
__global__ void __launch_bounds__(256) k_topk_dequant(const uint32_t* codes, const uint32_t* qjl, int64_t n,
                                                      int d, int kw, int qw, int m, int KL, int KQ,
                                                      const float* ck, __half* rows) {
  __shared__ uint32_t sP[256];
  constexpr int per = BK == 3 ? 16 : 32 / BK;   // fields per word of the main stream
  constexpr int fb = BK == 3 ? 2 : BK;          // bits per field of the main stream
  constexpr int pairs_w = per / 2;
  // Pair table: entry i -> half2(c[i0], c[i1]); for b = 3, i = f0 | f1 << 2 |
  // t0 << 4 | t1 << 5 (fields, then top bits), else i = i0 | i1 << b.
  for (int e = threadIdx.x; e < 256; e += blockDim.x) {
    int i0, i1;
    if (BK == 3) {
      i0 = (e & 3) | (((e >> 4) & 1) << 2);
      i1 = ((e >> 2) & 3) | (((e >> 5) & 1) << 2);
    } else {
      i0 = e & ((1 << BK) - 1);
      i1 = (e >> BK) & ((1 << BK) - 1);
    }
    const bool ok = BK == 3 ? e < 64 : e < (1 << (2 * BK));
    const __half2 hv = __floats2half2_rn(ok ? ck[i0] : 0.f, ok ? ck[i1] : 0.f);
    sP[e] = *reinterpret_cast<const uint32_t*>(&hv);
  }
  __syncthreads();
  const int W2 = (d + per - 1) / per;
  const int tasks = W2 + qw + 1;
  const int KP = KL + KQ;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n * tasks;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t v = e / tasks;
    const int wd = (int)(e - v * tasks);
    uint32_t* row = reinterpret_cast<uint32_t*>(rows + v * KP);
    if (wd < W2) {
      const uint32_t w = codes[v * kw + wd];
      uint32_t tw = 0u;
      if (BK == 3) tw = codes[v * kw + W2 + (wd >> 1)] >> (16 * (wd & 1));
#pragma unroll
      for (int j = 0; j < pairs_w; ++j) {
        const int c = per * wd + 2 * j;   // first coordinate of the pair
        uint32_t idx = (w >> (2 * fb * j)) & ((1u << (2 * fb)) - 1u);
        if (BK == 3) idx |= ((tw >> (2 * j)) & 3u) << 4;
        uint32_t h2 = sP[idx];
        if (c >= d) h2 = 0u;
        else if (c + 1 >= d) h2 &= 0xFFFFu;
        if (c < KL) row[c / 2] = h2;
      }
    } else if (wd < W2 + qw) {
      const int j0 = wd - W2;
      const uint32_t bits = qjl[v * qw + j0];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int c = 32 * j0 + 2 * j;   // first sketch row of the pair
        const uint32_t b2 = bits >> (2 * j);
        // -1 (0xBC00) per half, +1 where the bit is set: flip the sign bit.
        uint32_t h2 = 0xBC00BC00u ^ ((b2 & 1u) << 15) ^ ((b2 & 2u) << 30);
        if (c >= m) h2 = 0u;
        else if (c + 1 >= m) h2 &= 0xFFFFu;
        if (c < KQ) row[(KL + c) / 2] = h2;
      }
    } else {
      for (int c = per * W2; c < KL; c += 2) row[c / 2] = 0u;
    }
  }
}

// Shared memory for QB queries per CTA: B rows [QB][KS] and TKST stages of A
// rows [TKR][KS] in fp16 (KS = KL + KQ + 8: an odd number of 16-byte chunks
// per row, so ldmatrix rows hit distinct banks), the stages' norms and
// rnorms, query scales and the per-warp lists [TKWARPS][QB / 4][K] of
// (score, index).
__host__ __device__ inline size_t topk_mma_smem(int QB, int KL, int KQ, int K) {
  const size_t KS = (size_t)KL + KQ + 8;
  return 2 * KS * (QB + TKST * TKR) + (size_t)TKST * 2 * TKR * 4 + (size_t)QB * 2 * 4 +
         (size_t)TKWARPS * (QB / 4) * K * 8 + 64;
}

template <int QB>
__global__ void __launch_bounds__(TKWARPS * 32) k_topk_gemm(TopkMmaArgs a) {
  constexpr int QH = QB / 4;     // queries per warp
  constexpr int NTW = QH / 8;    // n-tiles per warp
  constexpr int SL = 2 * NTW;    // (query) slots per thread
  extern __shared__ __align__(16) unsigned char smem[];
  const int KS = a.KL + a.KQ + 8;
  const int KP = a.KL + a.KQ;
  __half* sB = reinterpret_cast<__half*>(smem);
  __half* sA = sB + (size_t)QB * KS;                                          // [TKST][TKR][KS]
  float* sN = reinterpret_cast<float*>(sA + (size_t)TKST * TKR * KS);         // [TKST][2][TKR]
  float* sQ = sN + TKST * 2 * TKR;                                            // [QB][2]: 2^e, 2^f
  float* lv = sQ + QB * 2;                                                    // [TKWARPS][QH][K]
  int* li = reinterpret_cast<int*>(lv + TKWARPS * QH * a.K);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int rg = warp & 1, qg = warp >> 1;   // row group, query quarter

  const uint32_t sA_s = (uint32_t)__cvta_generic_to_shared(sA);
  const uint32_t sB_s = (uint32_t)__cvta_generic_to_shared(sB);
  const uint32_t stage_bytes = (uint32_t)(TKR * KS * 2);
  // ldmatrix row addresses: A tiles (rows 0-7 / 8-15) x (k 0-7 / 8-15);
  // B tiles (n-tile nt / nt+1) x (k 0-7 / 8-15) of this warp's queries.
  const int ti = lane >> 3, tr = lane & 7;
  const uint32_t a_row0 = sA_s + (uint32_t)((16 * rg + tr + 8 * (ti & 1)) * KS + 8 * (ti >> 1)) * 2;
  const uint32_t b_row = sB_s + (uint32_t)((QH * qg + 8 * (ti >> 1) + tr) * KS + 8 * (ti & 1)) * 2;
  float* mylv = lv + warp * QH * a.K;
  int* myli = li + warp * QH * a.K;
  const int c16 = KP / 8;   // 16-byte chunks per row

  // Persistent CTAs: item = (database chunk, query block), chunk-major.
  const int64_t nitems = a.qblocks * a.chunks;
  for (int64_t item = blockIdx.x; item < nitems; item += gridDim.x) {
  const int64_t q0 = (item % a.qblocks) * QB;
  const int64_t chunk_id = item / a.qblocks;
  const int64_t n0 = chunk_id * a.chunk;
  const int64_t n1 = min(a.n, n0 + a.chunk);
  const int ntile = (int)((n1 - n0 + TKR - 1) / TKR);
  __syncthreads();   // the previous item's readers of sB, sA, sQ and the lists are done

  // Tile i of the chunk into stage st: its rows (zero past n1), norms, rnorms.
  auto stage = [&](int i, int st) {
    const int64_t v0 = n0 + (int64_t)i * TKR;
    const uint32_t dst = sA_s + st * stage_bytes;
    for (int e = tid; e < TKR * c16; e += TKWARPS * 32) {
      const int r = e / c16, c = e - r * c16;
      const bool ok = v0 + r < n1;
      cp16z(dst + (uint32_t)(r * KS + 8 * c) * 2, a.rows + (ok ? (v0 + r) * KP + 8 * c : 0), ok);
    }
    if (tid < 2 * TKR) {
      const int r = tid & (TKR - 1);
      const bool ok = v0 + r < n1 && (tid < TKR || a.m > 0);
      if (a.nf16 && tid < TKR) {   // binary16 norms: a plain load (no 2-byte cp.async)
        sN[st * 2 * TKR + tid] = ok ? load_norm(a.norm, v0 + r, 1) : 0.f;
      } else {
        const float* src = tid < TKR ? a.norm : a.rnorm;
        cp4(sN + st * 2 * TKR + tid, ok ? src + v0 + r : a.norm, ok);
      }
    }
  };
#pragma unroll
  for (int i = 0; i < TKST - 1; ++i) {
    if (i < ntile) stage(i, i);
    asm volatile("cp.async.commit_group;\n" ::);
  }
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
    bar(q0 + QH * (w >> 1) + ql, lv[e], li[e]);
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

  for (int i = 0; i < ntile; ++i) {
    const int64_t v0 = n0 + (int64_t)i * TKR;
    const int rows = (int)min((int64_t)TKR, n1 - v0);
    const int st = i % TKST;
    asm volatile("cp.async.wait_group %0;\n" ::"n"(TKST - 2) : "memory");
    __syncthreads();   // tile i landed; every warp is done with tile i - 1's stage
    if (i + TKST - 1 < ntile) stage(i + TKST - 1, (i + TKST - 1) % TKST);
    asm volatile("cp.async.commit_group;\n" ::);
    const float* sNn = sN + st * 2 * TKR;   // norms, then rnorms
    const uint32_t a_row = a_row0 + st * stage_bytes;

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
  // 128 queries per CTA (more products per staged tile) when it fits.
  p.qb = topk_mma_smem(128, p.KL, p.KQ, k) <= (size_t)227 * 1024 ? 128 : 64;
  const int64_t qblocks = (nq + p.qb - 1) / p.qb;
  // About sixteen (chunk, query block) items per SM for the persistent grid.
  int64_t chunks = (16 * (int64_t)c->sms + qblocks - 1) / (qblocks > 0 ? qblocks : 1);
  const int64_t max_chunks = (n + 8 * TKR - 1) / (8 * TKR);   // at least eight tiles per chunk
  if (chunks > max_chunks) chunks = max_chunks;
  if (chunks < 1) chunks = 1;
  if (chunks > 65535) chunks = 65535;
  p.chunk = ((n + chunks - 1) / chunks + TKR - 1) / TKR * TKR;
  p.chunks = (n + p.chunk - 1) / p.chunk;   // no empty chunk after rounding
  p.qblocks = qblocks;
  p.nlists = (int)(p.chunks * TKLISTS);
  p.qh_bytes = (size_t)nq * (p.KL + p.KQ) * sizeof(__half);
  p.qsc_bytes = (size_t)nq * 2 * sizeof(float);
  p.cand_bytes = (size_t)nq * p.nlists * k * (sizeof(float) + sizeof(int));
  p.rows_bytes = (size_t)n * (p.KL + p.KQ) * sizeof(__half);
  p.smem = topk_mma_smem(p.qb, p.KL, p.KQ, k);
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

cudaError_t launch_topk_dequant(const tq_ctx* c, const TopkPlan& p, const uint32_t* codes, const uint32_t* qjl,
                                int64_t n, void* rows, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const int qw = (c->qjl_m + 31) / 32;
  const int per = c->bk_lm == 3 ? 16 : 32 / c->bk_lm;
  const int64_t tasks = n * ((c->d + per - 1) / per + qw + 1);
  int64_t blocks = (tasks + 255) / 256;
  blocks = blocks > (int64_t)c->sms * 16 ? (int64_t)c->sms * 16 : blocks;
  __half* r = static_cast<__half*>(rows);
  const int qwv = qw;
  switch (c->bk_lm) {
    case 1: k_topk_dequant<1><<<(unsigned)blocks, 256, 0, s>>>(codes, qjl, n, c->d, c->wk, qwv, c->qjl_m, p.KL, p.KQ, c->ck_f, r); break;
    case 2: k_topk_dequant<2><<<(unsigned)blocks, 256, 0, s>>>(codes, qjl, n, c->d, c->wk, qwv, c->qjl_m, p.KL, p.KQ, c->ck_f, r); break;
    case 3: k_topk_dequant<3><<<(unsigned)blocks, 256, 0, s>>>(codes, qjl, n, c->d, c->wk, qwv, c->qjl_m, p.KL, p.KQ, c->ck_f, r); break;
    case 4: k_topk_dequant<4><<<(unsigned)blocks, 256, 0, s>>>(codes, qjl, n, c->d, c->wk, qwv, c->qjl_m, p.KL, p.KQ, c->ck_f, r); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_topk_mma(const tq_ctx* c, const TopkPlan& p, const void* qh, const float* qsc, int64_t nq,
                            const void* rows, const float* norm, const float* rnorm, int64_t n, int k,
                            const float* bar_v, const int* bar_i, float* cand_v, int* cand_i, cudaStream_t s) {
  TopkMmaArgs a{};
  a.qh = static_cast<const __half*>(qh);
  a.qsc = qsc;
  a.nq = nq;
  a.KL = p.KL;
  a.KQ = p.KQ;
  a.m = c->qjl_m;
  a.cq = c->qjl_m > 0 ? (float)(std::sqrt(M_PI / 2.0) / c->qjl_m) : 0.f;
  a.rows = static_cast<const __half*>(rows);
  a.norm = norm;
  a.rnorm = rnorm;
  a.nf16 = c->norm_f16 ? 1 : 0;
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
  if (p.qb == 128)
    k_topk_gemm<128><<<grid, TKWARPS * 32, p.smem, s>>>(a);
  else
    k_topk_gemm<64><<<grid, TKWARPS * 32, p.smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t configure_topk_mma() {
  const int lim = 227 * 1024;   // the plan never asks for more
  const cudaFuncAttribute ms = cudaFuncAttributeMaxDynamicSharedMemorySize;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(k_topk_gemm<64>, ms, lim))) return e;
  return cudaFuncSetAttribute(k_topk_gemm<128>, ms, lim);
}

}  // namespace tqk
