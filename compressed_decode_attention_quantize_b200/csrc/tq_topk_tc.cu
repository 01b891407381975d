// Inner-product top-k on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// "What is TurboQuant?", section "Benchmarks": nearest-neighbour search
// scores every database vector from its codes,
//   score(q, v) = n_v <q', c[idx_v]> + sqrt(pi/2)/m * gamma_v <S q', sigma_v>,
// and keeps the k best (score descending, then index ascending).
//
// The database rows [c[idx] | sigma] are dequantized once into fp16
// (k_topk_dequant) and the queries into [q' 2^-e | S q' 2^-f] (k_topk_qprep).
// This kernel is the contraction with a top-k epilogue:
//  - a producer thread streams 64-wide K blocks of 128 database rows with
//    TMA (128-byte swizzle) through a ring of shared-memory stages, and an
//    MMA thread issues tcgen05.mma (M = 128 rows, N = 128 queries, K = 16)
//    into two fp32
//    accumulators in tensor memory (centroid part, sign part); the 128
//    queries of the work item stay in shared memory;
//  - the accumulators are double-buffered, so sixteen epilogue warps read the
//    scores of tile i (tcgen05.ld; warp w: rows 32 (w & 3).., queries
//    32 (w >> 2)..) while the tensor cores compute tile i + 1;
//  - each (row quarter, query) keeps a top-k list (k <= 12) in the registers
//    of one lane; a score enters only if it beats the list's worst entry
//    (the bar, kept in a shared-memory column record).
// Work items (database chunk, query block) run chunk-major on a persistent
// grid, so the CTAs in flight read the same chunks from L2.  Every mbarrier
// wait is bounded; on expiry the kernel records a fault, drains its copies
// and MMAs, frees its tensor memory and returns.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>

#include "tq_internal.h"
#include "tq_tc_common.cuh"

namespace tqk {

__device__ int g_topk_fault = 0;

namespace {

constexpr int TC_ROWS = 128;                // database vectors per tile (TMEM lanes)
constexpr int TC_Q = 128;                   // queries per work item (MMA N)
constexpr uint32_t BLK = 128 * 128;         // one 64-wide K block of 128 rows (fp16): 16 KB
constexpr int EPI_WARPS = 16;               // warp w: rows 32 (w & 3).., queries 32 (w >> 2)..
constexpr int TC_THREADS = (EPI_WARPS + 2) * 32;   // + producer warp + MMA warp
constexpr int TC_LISTS = 4;                 // lists per query and chunk (row quarters)
constexpr int TC_KMAX = 12;                 // largest k kept in registers
constexpr uint32_t IDESC_TK = tc_idesc_f16(TC_Q);

struct TopkTcArgs {
  const float* qsc;   // [nq][2]: 2^e, 2^f
  int64_t nq;
  int KL, KQ, nkb;    // K blocks of 64 covering KL + KQ
  int m;
  float cq;           // sqrt(pi/2) / m
  const float* norm;   // binary16 values when nf16
  const float* rnorm;
  int nf16;
  int64_t n, chunk, chunks, qblocks;
  int K, nlists, stages;
  float* cand_v;
  int* cand_i;
  const float* bar_v;   // optional starting bar: entry (q, K - 1) of [nq][K]
  const int* bar_i;
  int wait_limit;       // polls of the main waits (drains keep the full limit)
};

__device__ __forceinline__ bool better_tc(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// 16 fp32 columns [col, col+16) of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared memory above the 1024-byte aligned base: query K blocks, A stages,
// then barriers, the TMEM address, query scales, bars and lists.
struct TcLayout {
  uint32_t b_off, a_off, bar_off, misc_off, total;
};
__host__ __device__ inline TcLayout tc_layout(int nkb, int stages, int K) {
  TcLayout L;
  L.b_off = 0;
  L.a_off = (uint32_t)nkb * BLK;
  L.bar_off = L.a_off + (uint32_t)stages * BLK;
  // barriers: full[S], empty[S], acc_full[2], acc_empty[2], bfull, done; then tmem slot
  L.misc_off = L.bar_off + (uint32_t)(2 * stages + 6) * 8 + 16;
  const uint32_t misc = EPI_WARPS * 32 * 16;
  (void)K;
  L.total = L.misc_off + misc + 1024;   // + alignment slack
  return L;
}

__global__ void __maxnreg__(96)
    k_topk_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, TopkTcArgs a) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_s = (uint32_t)__cvta_generic_to_shared(smem_raw);
  const uint32_t base_s = (raw_s + 1023u) & ~1023u;
  unsigned char* base = smem_raw + (base_s - raw_s);
  const int S = a.stages;
  const TcLayout LY = tc_layout(a.nkb, S, a.K);
  const uint32_t sB = base_s + LY.b_off, sA = base_s + LY.a_off;
  const uint32_t bar_full = base_s + LY.bar_off, bar_empty = bar_full + 8 * S;
  const uint32_t bar_accf = bar_empty + 8 * S, bar_acce = bar_accf + 16;
  const uint32_t bar_b = bar_acce + 16, bar_done = bar_b + 8;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(base + LY.bar_off + (2 * S + 6) * 8);
  // Per epilogue warp and column: (2^e, 2^f, bar score, bar index bits).
  float4* sCol = reinterpret_cast<float4*>(base + LY.misc_off);        // [EPI_WARPS][32]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == EPI_WARPS * 32) {
    for (int s = 0; s < S; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_accf + 8 * b, 1);
      mbar_init(bar_acce + 8 * b, EPI_WARPS);
    }
    mbar_init(bar_b, 1);
    mbar_init(bar_done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;\n" ::"r"(
                     (uint32_t)__cvta_generic_to_shared(s_tmem))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  tc_before_sync();
  __syncthreads();
  tc_after_sync();
  const uint32_t tmem = *s_tmem;
  const int64_t nitems = a.qblocks * a.chunks;
  const int ksteps = (a.KL + a.KQ) / 16;
  bool fault = false;

  if (warp == EPI_WARPS) {
    // ---- producer: TMA loads of the query blocks and the database K blocks ------------
    if (lane == 0) {
      uint32_t s = 0, up = 0;            // stage ring position and its fill parity
      uint32_t loaded = 0, tiles_before = 0, icount = 0;
      bool b_pending = false;
      uint32_t b_par = 0;                // phase parity of the last query-block load
      for (int64_t item = blockIdx.x; item < nitems && !fault; item += gridDim.x, ++icount) {
        const int64_t q0 = (item % a.qblocks) * TC_Q;
        const int64_t n0 = (item / a.qblocks) * a.chunk;
        const int64_t n1 = min(a.n, n0 + a.chunk);
        const int ntile = (int)((n1 - n0 + TC_ROWS - 1) / TC_ROWS);
        // The previous item's MMAs read the query blocks: let them finish.
        if (tiles_before > 0 &&
            !mbar_wait(bar_accf + 8 * ((tiles_before - 1) & 1), ((tiles_before - 1) >> 1) & 1, a.wait_limit)) {
          fault = true;
          break;
        }
        mbar_expect_tx(bar_b, (uint32_t)a.nkb * BLK);
        for (int kb = 0; kb < a.nkb; ++kb) tma_load_2d(sB + kb * BLK, &tmB, 64 * kb, (int)q0, bar_b);
        b_pending = true;
        b_par = icount & 1;
        for (int t = 0; t < ntile && !fault; ++t) {
          const int y = (int)(n0 + (int64_t)t * TC_ROWS);
          for (int kb = 0; kb < a.nkb; ++kb) {
            // The stage's previous K block has been consumed by its MMAs.
            if (loaded >= (uint32_t)S && !mbar_wait(bar_empty + 8 * s, up ^ 1, a.wait_limit)) {
              fault = true;
              break;
            }
            mbar_expect_tx(bar_full + 8 * s, BLK);
            tma_load_2d(sA + s * BLK, &tmA, 64 * kb, y, bar_full + 8 * s);
            ++loaded;
            if (++s == (uint32_t)S) {
              s = 0;
              up ^= 1;
            }
          }
        }
        tiles_before += ntile;
      }
      // Drain: the last copies issued (whether consumed or not).
      if (b_pending) mbar_wait(bar_b, b_par);
      const uint32_t back = loaded < (uint32_t)S ? loaded : (uint32_t)S;
      for (uint32_t k = 1; k <= back; ++k) {
        const uint32_t idx = loaded - k;
        mbar_wait(bar_full + 8 * (idx % S), (idx / S) & 1);
      }
    }
    __syncwarp();
  } else if (warp == EPI_WARPS + 1) {
    // ---- MMA issue (one thread) --------------------------------------------------------
    if (lane == 0) {
      uint32_t s = 0, up = 0, tcount = 0, icount = 0;
      const uint64_t dA0 = smem_desc(sA), dB0 = smem_desc(sB);
      for (int64_t item = blockIdx.x; item < nitems && !fault; item += gridDim.x, ++icount) {
        const int64_t n0 = (item / a.qblocks) * a.chunk;
        const int64_t n1 = min(a.n, n0 + a.chunk);
        const int ntile = (int)((n1 - n0 + TC_ROWS - 1) / TC_ROWS);
        if (!mbar_wait(bar_b, icount & 1, a.wait_limit)) {
          fault = true;
          break;
        }
        for (int t = 0; t < ntile && !fault; ++t) {
          const uint32_t ab = tcount & 1;
          if (!mbar_wait(bar_acce + 8 * ab, ((tcount >> 1) & 1) ^ 1, a.wait_limit)) {
            fault = true;
            break;
          }
          tc_after_sync();
          const uint32_t d_lm = tmem + ab * 256, d_q = d_lm + 128;
          for (int kb = 0; kb < a.nkb; ++kb) {
            if (!mbar_wait(bar_full + 8 * s, up, a.wait_limit)) {
              fault = true;
              break;
            }
            tc_after_sync();
            // Descriptor start addresses advance by 32 bytes (16 fp16) per k-step.
            const uint64_t da = dA0 + (uint64_t)(s * (BLK >> 4)), db = dB0 + (uint64_t)(kb * (BLK >> 4));
#pragma unroll
            for (int t4 = 0; t4 < 4; ++t4) {
              const int js = 4 * kb + t4;   // k-step: K columns 16 js .. + 15
              if (js < ksteps) {
                const bool lm = 16 * js < a.KL;
                const uint32_t acc = lm ? (js > 0 ? 1u : 0u) : (16 * js > a.KL ? 1u : 0u);
                tc_mma_f16(lm ? d_lm : d_q, da + 2 * t4, db + 2 * t4, IDESC_TK, acc);
              }
            }
            tc_commit(bar_empty + 8 * s);
            if (++s == (uint32_t)S) {
              s = 0;
              up ^= 1;
            }
          }
          if (fault) break;
          tc_commit(bar_accf + 8 * ab);
          ++tcount;
        }
      }
      // Drain: every MMA issued.
      tc_commit(bar_done);
      mbar_wait(bar_done, 0);
    }
    __syncwarp();
  } else {
    // ---- epilogue warps -------------------------------------------------------------
    // Warp w owns the lists of (row quarter w & 3, queries 32 (w >> 2) .. + 31):
    // lane l keeps the list of query 32 (w >> 2) + l in registers, and the
    // column records of those queries sit in shared memory (read by all
    // lanes, written by the owner).  No barrier between warps.
    const int rq = warp & 3, qc = warp >> 2;
    float4* col = sCol + warp * 32;
    uint32_t tcount = 0;
    for (int64_t item = blockIdx.x; item < nitems && !fault; item += gridDim.x) {
      const int64_t q0 = (item % a.qblocks) * TC_Q;
      const int64_t chunk_id = item / a.qblocks;
      const int64_t n0 = chunk_id * a.chunk;
      const int64_t n1 = min(a.n, n0 + a.chunk);
      const int ntile = (int)((n1 - n0 + TC_ROWS - 1) / TC_ROWS);
      // This lane's list starts at its query's bar (the k-th best of a
      // sample bounds the final k-th best from below).
      const int64_t myq = q0 + 32 * qc + lane;
      float lv[TC_KMAX];
      int li[TC_KMAX];
      {
        float v = -INFINITY;
        int ix = INT_MAX;
        if (a.bar_v && myq < a.nq && a.bar_i[myq * a.K + a.K - 1] >= 0) {
          v = a.bar_v[myq * a.K + a.K - 1];
          ix = a.bar_i[myq * a.K + a.K - 1];
        }
#pragma unroll
        for (int r = 0; r < TC_KMAX; ++r) {
          lv[r] = v;
          li[r] = ix;
        }
        const bool in = myq < a.nq;
        __syncwarp();   // every lane is done with the previous item's records
        col[lane] = make_float4(in ? a.qsc[2 * myq] : 0.f, in ? a.qsc[2 * myq + 1] : 0.f, v, __int_as_float(ix));
        __syncwarp();
      }
      // Row norms one tile ahead.
      auto norms = [&](int t, float& nv, float& gv) {
        const int64_t v = n0 + (int64_t)t * TC_ROWS + 32 * rq + lane;
        const bool ok = t < ntile && v < n1;
        nv = ok ? load_norm(a.norm, v, a.nf16) : 0.f;
        gv = (ok && a.m > 0) ? a.rnorm[v] * a.cq : 0.f;
      };
      float nv_next, gv_next;
      norms(0, nv_next, gv_next);
      for (int t = 0; t < ntile; ++t) {
        const int64_t v = n0 + (int64_t)t * TC_ROWS + 32 * rq + lane;   // this lane's database row
        const bool valid = v < n1;
        const float nv = nv_next, gv = gv_next;
        norms(t + 1, nv_next, gv_next);
        const uint32_t ab = tcount & 1;
        if (!mbar_wait(bar_accf + 8 * ab, (tcount >> 1) & 1, a.wait_limit)) {
          fault = true;
          break;
        }
        tc_after_sync();
        const uint32_t t_lm = tmem + ((uint32_t)(32 * rq) << 16) + ab * 256 + 32 * qc;
        // Scores of the 32 columns in two halves of 16 (fewer live registers)
        // and this lane's candidate bits: one 16-byte column record and one
        // comparison per score.
        float sc[32];
        uint32_t cm = 0u;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          float dq[16];
          float* dl = sc + 16 * hf;
          tmem_ld16(t_lm + 16 * hf, dl);
          if (a.m > 0) {
            tmem_ld16(t_lm + 128 + 16 * hf, dq);
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) dq[i] = 0.f;
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float4 ci = col[16 * hf + i];
            dl[i] = valid ? fmaf(nv * ci.x, dl[i], gv * ci.y * dq[i]) : -INFINITY;
            if (valid && better_tc(dl[i], (int)v, ci.z, __float_as_int(ci.w))) cm |= 1u << (16 * hf + i);
          }
        }
        tc_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_acce + 8 * ab);   // the scores are in registers
        ++tcount;
        // Rare once the bars are up: insert column by column; the lane that
        // owns the column's list updates it and its record, every lane
        // re-checks against the new bar.
        uint32_t cols = __reduce_or_sync(0xffffffffu, cm);
        while (cols) {
          const int i = __ffs(cols) - 1;
          cols &= cols - 1u;
          float mine = 0.f;
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (k == i) mine = sc[k];
          bool cand = (cm >> i) & 1u;
          uint32_t mask = __ballot_sync(0xffffffffu, cand);
          while (mask) {
            const int leader = __ffs(mask) - 1;
            const float val = __shfl_sync(0xffffffffu, mine, leader);
            const int idx = __shfl_sync(0xffffffffu, (int)v, leader);
            if (lane == i) {
              // Replace the worst entry, then find the new worst (the bar).
              int wpos = 0;
              float wv = lv[0];
              int wi = li[0];
#pragma unroll
              for (int r = 1; r < TC_KMAX; ++r)
                if (r < a.K && better_tc(wv, wi, lv[r], li[r])) {
                  wpos = r;
                  wv = lv[r];
                  wi = li[r];
                }
              if (better_tc(val, idx, wv, wi)) {
#pragma unroll
                for (int r = 0; r < TC_KMAX; ++r)
                  if (r == wpos) {
                    lv[r] = val;
                    li[r] = idx;
                  }
                wv = lv[0];
                wi = li[0];
#pragma unroll
                for (int r = 1; r < TC_KMAX; ++r)
                  if (r < a.K && better_tc(wv, wi, lv[r], li[r])) {
                    wv = lv[r];
                    wi = li[r];
                  }
              }
              col[i].z = wv;
              col[i].w = __int_as_float(wi);
            }
            __syncwarp();
            if (lane == leader) cand = false;
            const float4 ci = col[i];
            cand = cand && better_tc(mine, (int)v, ci.z, __float_as_int(ci.w));
            mask = __ballot_sync(0xffffffffu, cand);
          }
        }
      }
      if (fault) break;
      // This lane's list -> candidates of (query, chunk, row quarter).
      if (myq < a.nq) {
        const int64_t o = (myq * a.nlists + chunk_id * TC_LISTS + rq) * a.K;
#pragma unroll
        for (int r = 0; r < TC_KMAX; ++r)
          if (r < a.K) {
            a.cand_v[o + r] = lv[r];
            a.cand_i[o + r] = li[r];
          }
      }
    }
  }
  if (fault) atomicExch(&g_topk_fault, 1);
  tc_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_after_sync();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;\n" ::"r"(tmem) : "memory");
  }
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

// fp16 rows [rows][kp] (row pitch kp * 2 bytes), boxes of 64 x 128, 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, int64_t rows, int kp) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)kp, (cuuint64_t)(rows > 0 ? rows : 1)};
  const cuuint64_t strides[1] = {(cuuint64_t)kp * 2};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t es[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

TopkPlan topk_tc_plan(const tq_ctx* c, int64_t nq, int64_t n, int k, int64_t n_sample) {
  TopkPlan p{};
  p.KL = (c->d + 15) / 16 * 16;
  p.KQ = (c->qjl_m + 15) / 16 * 16;
  p.qb = TC_Q;
  p.nkb = (p.KL + p.KQ + 63) / 64;
  const size_t fixed = tc_layout(p.nkb, 0, k).total;
  const size_t room = (size_t)227 * 1024 > fixed ? (size_t)227 * 1024 - fixed : 0;
  p.stages = (int)(room / BLK);
  if (p.stages > 8) p.stages = 8;
  p.use_tc = p.stages >= 3 && k <= TC_KMAX && encode_fn() != nullptr;
  const int64_t qblocks = (nq + TC_Q - 1) / TC_Q;
  const int64_t nn = n_sample > 0 ? n_sample : n;
  // Full pass: about sixteen items per SM; sample pass: about one.
  int64_t chunks = ((n_sample > 0 ? 1 : 16) * (int64_t)c->sms + qblocks - 1) / (qblocks > 0 ? qblocks : 1);
  const int64_t max_chunks = (nn + 4 * TC_ROWS - 1) / (4 * TC_ROWS);   // at least four tiles per chunk
  if (chunks > max_chunks) chunks = max_chunks;
  if (chunks < 1) chunks = 1;
  p.chunk = ((nn + chunks - 1) / chunks + TC_ROWS - 1) / TC_ROWS * TC_ROWS;
  p.chunks = (nn + p.chunk - 1) / p.chunk;
  p.qblocks = qblocks;
  p.nlists = (int)(p.chunks * TC_LISTS);
  p.qh_bytes = (size_t)nq * (p.KL + p.KQ) * sizeof(__half);
  p.qsc_bytes = (size_t)nq * 2 * sizeof(float);
  p.cand_bytes = (size_t)nq * p.nlists * k * (sizeof(float) + sizeof(int));
  p.rows_bytes = (size_t)n * (p.KL + p.KQ) * sizeof(__half);
  p.smem = tc_layout(p.nkb, p.stages, k).total;
  return p;
}

cudaError_t launch_topk_tc(const tq_ctx* c, const TopkPlan& p, const void* qh, const float* qsc, int64_t nq,
                           const void* rows, const float* norm, const float* rnorm, int64_t n, int k,
                           const float* bar_v, const int* bar_i, float* cand_v, int* cand_i, cudaStream_t s) {
  const int kp = p.KL + p.KQ;
  CUtensorMap ma, mb;
  if (!make_map(&ma, rows, n, kp) || !make_map(&mb, qh, nq, kp)) return cudaErrorInvalidValue;
  TopkTcArgs a{};
  a.qsc = qsc;
  a.nq = nq;
  a.KL = p.KL;
  a.KQ = p.KQ;
  a.nkb = p.nkb;
  a.m = c->qjl_m;
  a.cq = c->qjl_m > 0 ? (float)(std::sqrt(M_PI / 2.0) / c->qjl_m) : 0.f;
  a.norm = norm;
  a.rnorm = rnorm;
  a.nf16 = c->norm_f16 ? 1 : 0;
  a.n = n;
  a.chunk = p.chunk;
  a.chunks = p.chunks;
  a.qblocks = p.qblocks;
  a.K = k;
  a.nlists = p.nlists;
  a.stages = p.stages;
  a.cand_v = cand_v;
  a.cand_i = cand_i;
  a.bar_v = bar_v;
  a.bar_i = bar_i;
  a.wait_limit = c->wait_limit > 0 ? c->wait_limit : TC_WAIT_LIMIT;
  const int64_t items = p.qblocks * p.chunks;
  const unsigned grid = (unsigned)(items < c->sms ? items : c->sms);   // one CTA per SM
  k_topk_tc<<<grid, TC_THREADS, p.smem, s>>>(ma, mb, a);
  return cudaGetLastError();
}

cudaError_t configure_topk_tc() {
  return cudaFuncSetAttribute(k_topk_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
}

cudaError_t read_and_clear_topk_fault(int* value) {
  cudaError_t e = cudaMemcpyFromSymbol(value, g_topk_fault, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_topk_fault, &zero, sizeof(int));
}

}  // namespace tqk
