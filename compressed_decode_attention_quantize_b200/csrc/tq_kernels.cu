// CUDA kernels of libtq (sm_100a), plain fp32 versions.
//
// Each kernel states the operation it computes; the method follows "What is
// TurboQuant?" (a2a-mcp.org), section "How TurboQuant works": stage 1 (rotate
// the normalised vector with Pi, Lloyd-Max index per coordinate), stage 2 (1-bit
// QJL sketch of the residual) and the closing paragraph (logits taken from the
// compressed indices without dequantizing the keys).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <climits>
#include <cmath>

#include "tq_internal.h"
#include "tq_qop.cuh"

namespace tqk {

namespace {

constexpr float kNegInf = -INFINITY;

__device__ __forceinline__ float load_elem(const void* p, int dtype, int64_t i) {
  if (dtype == TQ_F32) return static_cast<const float*>(p)[i];
  if (dtype == TQ_BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
  return __half2float(static_cast<const __half*>(p)[i]);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Index of a coordinate: number of boundaries at or below y (ties go up).
// The boundaries ascend, so for the 255 of an 8-bit codebook a bisection for
// the first boundary above y gives the same count.
__device__ __forceinline__ int lm_index(float y, const float* sb, int nb) {
  if (nb > 15) {
    int lo = 0, hi = nb;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (y >= sb[mid]) lo = mid + 1; else hi = mid;
    }
    return lo;
  }
  int idx = 0;
  for (int t = 0; t < nb; ++t) idx += (y >= sb[t]) ? 1 : 0;
  return idx;
}

// Output record of input row v (cache placement when a.pos is set).
// Output record of vector v: v itself, or for cache appends slot pos[b] of
// row v = b H + g (contiguous or paged cache); -1 (nothing written) when
// pos[b] is outside [0, max_T) or its block id is invalid.
__device__ __forceinline__ int64_t out_record(const QuantArgs& a, int64_t v) {
  if (a.pos == nullptr) return v;
  const int64_t b = v / a.H;
  const int64_t p = a.pos[b];
  if (p < 0 || p >= a.max_T) return -1;
  if (a.block_table == nullptr) return v * a.max_T + p;
  // Paged: slot p % block_size of block block_table[b][p / block_size].
  const int64_t blk = a.block_table[b * a.max_blocks + p / a.block_size];
  if (blk < 0 || blk >= a.num_blocks) return -1;
  return (blk * a.H + (v - b * a.H)) * a.block_size + p % a.block_size;
}

// Lloyd-Max index of coordinate j of a packed vector (b-bit fields; for b = 3
// a 2-bit stream of the low bits followed by a 1-bit stream of the top bits).
__device__ __forceinline__ int code_index(const uint32_t* w, int bits, int d, int j) {
  if (bits == 3) {
    const int lo = (w[j >> 4] >> ((j & 15) * 2)) & 3;
    const int hi = (w[((d + 15) >> 4) + (j >> 5)] >> (j & 31)) & 1;
    return lo | (hi << 2);
  }
  const int per = 32 / bits;
  return (w[j / per] >> (bits * (j % per))) & ((1 << bits) - 1);
}

// OR of the b-bit field of each lane placed at its slot, over groups of 32/b
// consecutive lanes (every lane of the group ends with the group's word).
__device__ __forceinline__ uint32_t field_word(uint32_t val, int b, int lane) {
  const int per = 32 / b;
  uint32_t x = val << (b * (lane % per));
  for (int o = 1; o < per; o <<= 1) x |= __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// ----------------------------------------------------------------------------
// Quantize: one warp quantizes QV vectors at a time (quant_qv).  Lane l owns the output
// coordinates j = l + 32 i (i < J), so the Lloyd-Max bits of plane p, word i
// of a vector are one __ballot_sync.  The rotation y = Pi x / |x| and the
// sketch S r are fp32 FMA dot products (PiT and ST are k-major so lanes read
// consecutive words).
// ----------------------------------------------------------------------------
// ----------------------------------------------------------------------------
// Row-batched matrix-vector products for the latency-bound small kernels:
// thread j (blockDim = dpad) computes acc[r] = sum_k M[k][j] x_r[k] for R
// vectors x_r held in shared memory.  M ([d][dpad] fp32) streams through
// shared memory in chunks of MV_KC rows, two chunks in flight (cp.async), so
// the block pays the L2 latency about once per chunk, not once per row.
// ----------------------------------------------------------------------------
constexpr int MV_KC = 32;

__device__ __forceinline__ void mv_cp16(float* dst, const float* src) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(src));
}

__device__ __forceinline__ void mv_issue(const float* M, int d, int dpad, int chunk, float* buf) {
  const int k0 = chunk * MV_KC;
  const int rows = min(MV_KC, d - k0);
  const int pieces = rows * dpad / 4;
  for (int e = threadIdx.x; e < pieces; e += blockDim.x) mv_cp16(buf + 4 * e, M + (size_t)k0 * dpad + 4 * e);
  asm volatile("cp.async.commit_group;\n" ::);
}

// Ms: shared [2][MV_KC][dpad].  Ends with a barrier (Ms and xs reusable).
template <int R>
__device__ __forceinline__ void mv_rows(const float* M, int d, int dpad, const float* xs, float* Ms,
                                        float (&acc)[R]) {
  const int j = threadIdx.x;
#pragma unroll
  for (int r = 0; r < R; ++r) acc[r] = 0.f;
  const int nchunk = (d + MV_KC - 1) / MV_KC;
  mv_issue(M, d, dpad, 0, Ms);
  for (int c = 0; c < nchunk; ++c) {
    if (c + 1 < nchunk) {
      mv_issue(M, d, dpad, c + 1, Ms + ((c + 1) & 1) * MV_KC * dpad);
      asm volatile("cp.async.wait_group 1;\n" ::);
    } else {
      asm volatile("cp.async.wait_group 0;\n" ::);
    }
    __syncthreads();
    const float* mb = Ms + (c & 1) * MV_KC * dpad;
    const int k0 = c * MV_KC, rows = min(MV_KC, d - k0);
    int kk = 0;
    for (; kk + 4 <= rows; kk += 4) {   // x rows read as float4 (k0 + kk is a multiple of 4)
      const float m0 = mb[kk * dpad + j], m1 = mb[(kk + 1) * dpad + j];
      const float m2 = mb[(kk + 2) * dpad + j], m3 = mb[(kk + 3) * dpad + j];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float4 x4 = *reinterpret_cast<const float4*>(xs + r * dpad + k0 + kk);
        acc[r] = fmaf(m0, x4.x, acc[r]);
        acc[r] = fmaf(m1, x4.y, acc[r]);
        acc[r] = fmaf(m2, x4.z, acc[r]);
        acc[r] = fmaf(m3, x4.w, acc[r]);
      }
    }
    for (; kk < rows; ++kk) {
      const float m = mb[kk * dpad + j];
#pragma unroll
      for (int r = 0; r < R; ++r) acc[r] = fmaf(m, xs[r * dpad + k0 + kk], acc[r]);
    }
    __syncthreads();   // the chunk buffer is refilled two chunks later
  }
}

constexpr int QWARPS = 8;
// Vectors per warp: eight up to d = 128; four beyond, where eight would hold
// 8 J accumulators and indices per lane (d = 200: 242 registers, one
// 256-thread CTA per SM) and leave the matrix loads' latency uncovered.
template <int J>
__host__ __device__ constexpr int quant_qv() {
  return J >= 5 ? 4 : 8;
}

template <int J>
__global__ void __launch_bounds__(QWARPS * 32) k_quantize(QuantArgs a) {
  constexpr int DP = J * 32;
  constexpr int QV = quant_qv<J>();
  static_assert(QV % 4 == 0, "x rows are read as float4");
  extern __shared__ float smem[];
  __shared__ float s_cen[kMaxLevels], s_bnd[kMaxLevels];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* sx = smem + warp * (DP * QV);  // [DP][QV]
  for (int e = threadIdx.x; e < kMaxLevels; e += blockDim.x) {
    s_cen[e] = (e < (1 << a.bits)) ? a.cen[e] : 0.f;
    s_bnd[e] = (e < a.nbnd) ? a.bnd[e] : INFINITY;
  }
  __syncthreads();
  const int64_t ngroups = (a.n + QV - 1) / QV;
  const int mwords = (a.m + 31) >> 5;
  for (int64_t g = (int64_t)blockIdx.x * QWARPS + warp; g < ngroups;
       g += (int64_t)gridDim.x * QWARPS) {
    const int64_t v0 = g * QV;
    float ss[QV];
#pragma unroll
    for (int v = 0; v < QV; ++v) {
      ss[v] = 0.f;
#pragma unroll
      for (int i = 0; i < J; ++i) {
        const int k = lane + 32 * i;
        float val = 0.f;
        if (k < a.d && v0 + v < a.n) val = load_elem(a.x, a.dtype, (v0 + v) * a.ld + k);
        sx[k * QV + v] = val;
        ss[v] = fmaf(val, val, ss[v]);
      }
      ss[v] = warp_sum(ss[v]);
    }
    __syncwarp();
    float acc[J][QV];
#pragma unroll
    for (int i = 0; i < J; ++i)
#pragma unroll
      for (int v = 0; v < QV; ++v) acc[i][v] = 0.f;
    for (int k = 0; k < a.d; ++k) {
      float xv[QV];
      if constexpr (QV == 8) {
        const float4 x0 = *reinterpret_cast<const float4*>(sx + k * QV);
        const float4 x1 = *reinterpret_cast<const float4*>(sx + k * QV + 4);
        xv[0] = x0.x, xv[1] = x0.y, xv[2] = x0.z, xv[3] = x0.w;
        xv[4] = x1.x, xv[5] = x1.y, xv[6] = x1.z, xv[7] = x1.w;
      } else {
        const float4 x0 = *reinterpret_cast<const float4*>(sx + k * QV);
        xv[0] = x0.x, xv[1] = x0.y, xv[2] = x0.z, xv[3] = x0.w;
      }
#pragma unroll
      for (int i = 0; i < J; ++i) {
        const float p = __ldg(a.PiT + (size_t)k * DP + lane + 32 * i);
#pragma unroll
        for (int v = 0; v < QV; ++v) acc[i][v] = fmaf(p, xv[v], acc[i][v]);
      }
    }
    // y = Pi x / |x| (0 for a zero vector), then the Lloyd-Max index.
    float nrm[QV];
    unsigned char idx[J][QV];
#pragma unroll
    for (int v = 0; v < QV; ++v) {
      nrm[v] = sqrtf(ss[v]);
#pragma unroll
      for (int i = 0; i < J; ++i) {
        const float y = nrm[v] > 0.f ? acc[i][v] / nrm[v] : 0.f;
        acc[i][v] = y;
        idx[i][v] = (unsigned char)lm_index(y, s_bnd, a.nbnd);
      }
    }
    // Norm correction: the stored scalar is n / |c[idx]| (no QJL stage then,
    // so nrm is not needed afterwards).
    if (a.nc) {
#pragma unroll
      for (int v = 0; v < QV; ++v) {
        float cc = 0.f;
#pragma unroll
        for (int i = 0; i < J; ++i) {
          const float cj = (lane + 32 * i < a.d) ? s_cen[idx[i][v]] : 0.f;
          cc = fmaf(cj, cj, cc);
        }
        nrm[v] = nrm[v] / sqrtf(warp_sum(cc));
      }
    }
    // Field packing: lane owns coordinates lane + 32 i; a group of 32/b lanes
    // fills one word (b = 3: 2-bit stream of low bits, then 1-bit stream).
#pragma unroll
    for (int v = 0; v < QV; ++v) {
      const int64_t rec = v0 + v < a.n ? out_record(a, v0 + v) : -1;
      const bool live = rec >= 0;
      const int64_t base = live ? rec * a.words : 0;
#pragma unroll
      for (int i = 0; i < J; ++i) {
        const uint32_t iv = (lane + 32 * i < a.d) ? idx[i][v] : 0u;
        if (a.bits == 3) {
          const int w2 = (a.d + 15) >> 4;
          const uint32_t lo = field_word(iv & 3u, 2, lane);
          const uint32_t hi = field_word(iv >> 2, 1, lane);
          const int wlo = 2 * i + (lane >> 4);
          if (live && (lane & 15) == 0 && wlo < w2) a.codes[base + wlo] = lo;
          if (live && lane == 0) a.codes[base + w2 + i] = hi;
        } else {
          const int per = 32 / a.bits;
          const uint32_t wv = field_word(iv, a.bits, lane);
          const int wi = a.bits * i + lane / per;
          if (live && lane % per == 0 && wi < a.words) a.codes[base + wi] = wv;
        }
      }
    }
    float my_norm = 0.f;
#pragma unroll
    for (int v = 0; v < QV; ++v)
      if (lane == v) my_norm = nrm[v];
    if (lane < QV && v0 + lane < a.n) {
      const int64_t rec = out_record(a, v0 + lane);
      if (rec >= 0) store_norm(a.norm, rec, my_norm, a.nf16);
    }
    if (a.m == 0) { __syncwarp(); continue; }

    // Stage 2: residual r = y - c[idx], rho = |r|, QJL bits sign(S r).
    __syncwarp();
    float rr[QV];
#pragma unroll
    for (int v = 0; v < QV; ++v) {
      rr[v] = 0.f;
#pragma unroll
      for (int i = 0; i < J; ++i) {
        const int k = lane + 32 * i;
        const float r = (k < a.d) ? acc[i][v] - s_cen[idx[i][v]] : 0.f;
        sx[k * QV + v] = r;
        rr[v] = fmaf(r, r, rr[v]);
      }
      rr[v] = warp_sum(rr[v]);
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < J; ++i)
#pragma unroll
      for (int v = 0; v < QV; ++v) acc[i][v] = 0.f;
    for (int k = 0; k < a.d; ++k) {
      float xv[QV];
      if constexpr (QV == 8) {
        const float4 x0 = *reinterpret_cast<const float4*>(sx + k * QV);
        const float4 x1 = *reinterpret_cast<const float4*>(sx + k * QV + 4);
        xv[0] = x0.x, xv[1] = x0.y, xv[2] = x0.z, xv[3] = x0.w;
        xv[4] = x1.x, xv[5] = x1.y, xv[6] = x1.z, xv[7] = x1.w;
      } else {
        const float4 x0 = *reinterpret_cast<const float4*>(sx + k * QV);
        xv[0] = x0.x, xv[1] = x0.y, xv[2] = x0.z, xv[3] = x0.w;
      }
#pragma unroll
      for (int i = 0; i < J; ++i) {
        const float p = __ldg(a.ST + (size_t)k * DP + lane + 32 * i);
#pragma unroll
        for (int v = 0; v < QV; ++v) acc[i][v] = fmaf(p, xv[v], acc[i][v]);
      }
    }
#pragma unroll
    for (int v = 0; v < QV; ++v) {
      uint32_t mine = 0;
#pragma unroll
      for (int i = 0; i < J; ++i) {
        const bool bit = (acc[i][v] >= 0.f) && (lane + 32 * i < a.m);
        const uint32_t w = __ballot_sync(0xffffffffu, bit);
        if (lane == i) mine = w;
      }
      if (v0 + v < a.n && lane < mwords) {
        const int64_t rec = out_record(a, v0 + v);
        if (rec >= 0) a.qjl[rec * mwords + lane] = mine;
      }
    }
    float my_rn = 0.f;
#pragma unroll
    for (int v = 0; v < QV; ++v)
      if (lane == v) my_rn = nrm[v] * sqrtf(rr[v]);
    if (lane < QV && v0 + lane < a.n) {
      const int64_t rec = out_record(a, v0 + lane);
      if (rec >= 0) a.rnorm[rec] = my_rn;
    }
    __syncwarp();
  }
}

// ----------------------------------------------------------------------------
// Quantize, small batches (the per-step cache append): QS vectors per block,
// thread j owns coordinate j (and QJL row j) of each, so the block reads Pi
// and S once for all QS vectors, and a few hundred vectors spread over many
// SMs instead of filling one tile.  Same fp32 arithmetic as above.
// ----------------------------------------------------------------------------
// Block blk of the small-batch quantizer; sh = [QS][dpad] (x, later r) then
// [2][MV_KC][dpad] matrix chunks.  blockDim = dpad.
template <int QS>
__device__ __forceinline__ void quantize_small_body(const QuantArgs& a, int dpad, int64_t blk, float* sh) {
  float* Ms = sh + QS * dpad;
  __shared__ float red[QS][8];
  __shared__ float s_cen[kMaxLevels], s_bnd[kMaxLevels];
  const int j = threadIdx.x, lane = j & 31, warp = j >> 5, nwarp = blockDim.x >> 5;
  const int64_t v0 = blk * QS;
  const int nv = (int)min((int64_t)QS, a.n - v0);
  for (int e = j; e < kMaxLevels; e += blockDim.x) {
    s_cen[e] = (e < (1 << a.bits)) ? a.cen[e] : 0.f;
    s_bnd[e] = (e < a.nbnd) ? a.bnd[e] : INFINITY;
  }
  float nrm[QS];
#pragma unroll
  for (int u = 0; u < QS; ++u) {
    const float xj = (u < nv && j < a.d) ? load_elem(a.x, a.dtype, (v0 + u) * a.ld + j) : 0.f;
    sh[u * dpad + j] = xj;
    nrm[u] = warp_sum(xj * xj);
  }
  if (lane == 0) {
#pragma unroll
    for (int u = 0; u < QS; ++u) red[u][warp] = nrm[u];
  }
  __syncthreads();   // x, tables and the per-warp sums are in shared memory
#pragma unroll
  for (int u = 0; u < QS; ++u) {
    float t = 0.f;
    for (int w = 0; w < nwarp; ++w) t += red[u][w];
    nrm[u] = sqrtf(t);
  }
  float acc[QS];
  mv_rows<QS>(a.PiT, a.d, dpad, sh, Ms, acc);
  float r[QS];
  int ids[QS];
  const int i32 = j >> 5;
#pragma unroll
  for (int u = 0; u < QS; ++u) {
    const float y = (nrm[u] > 0.f && j < a.d) ? acc[u] / nrm[u] : 0.f;
    ids[u] = lm_index(y, s_bnd, a.nbnd);
    r[u] = (j < a.d) ? y - s_cen[ids[u]] : 0.f;
  }
  if (a.nc) {   // uniform; norm correction: store n / |c[idx]| (MSE-only, no QJL stage follows)
    __syncthreads();   // every thread has read the norm sums out of red
#pragma unroll
    for (int u = 0; u < QS; ++u) {
      const float cj = (j < a.d) ? s_cen[ids[u]] : 0.f;
      const float cc = warp_sum(cj * cj);
      if (lane == 0) red[u][warp] = cc;
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < QS; ++u) {
      float t = 0.f;
      for (int w = 0; w < nwarp; ++w) t += red[u][w];
      nrm[u] = nrm[u] / sqrtf(t);
    }
  }
#pragma unroll
  for (int u = 0; u < QS; ++u) {
    const int idx = ids[u];
    if (u >= nv) continue;   // uniform over the block
    const int64_t rec = out_record(a, v0 + u);
    if (rec < 0) continue;   // uniform too (one sequence per vector)
    // b-bit field packing within each warp (b = 3: 2-bit stream, then 1-bit stream)
    const uint32_t iv = (j < a.d) ? (uint32_t)idx : 0u;
    if (a.bits == 3) {
      const int w2 = (a.d + 15) >> 4;
      const uint32_t lo = field_word(iv & 3u, 2, lane);
      const uint32_t hi = field_word(iv >> 2, 1, lane);
      const int wlo = 2 * i32 + (lane >> 4);
      if ((lane & 15) == 0 && wlo < w2) a.codes[rec * a.words + wlo] = lo;
      if (lane == 0) a.codes[rec * a.words + w2 + i32] = hi;
    } else {
      const int per = 32 / a.bits;
      const uint32_t wv = field_word(iv, a.bits, lane);
      const int wi = a.bits * i32 + lane / per;
      if (lane % per == 0 && wi < a.words) a.codes[rec * a.words + wi] = wv;
    }
    if (j == 0) store_norm(a.norm, rec, nrm[u], a.nf16);
  }
  if (a.m == 0) return;
  float rho[QS];
#pragma unroll
  for (int u = 0; u < QS; ++u) {
    sh[u * dpad + j] = r[u];
    rho[u] = warp_sum(r[u] * r[u]);
  }
  if (lane == 0) {
#pragma unroll
    for (int u = 0; u < QS; ++u) red[u][warp] = rho[u];
  }
  __syncthreads();
#pragma unroll
  for (int u = 0; u < QS; ++u) {
    float t = 0.f;
    for (int w = 0; w < nwarp; ++w) t += red[u][w];
    rho[u] = sqrtf(t);
  }
  mv_rows<QS>(a.ST, a.d, dpad, sh, Ms, acc);
#pragma unroll
  for (int u = 0; u < QS; ++u) {
    const uint32_t bits = __ballot_sync(0xffffffffu, acc[u] >= 0.f && j < a.m);
    if (u >= nv) continue;
    const int64_t rec = out_record(a, v0 + u);
    if (rec < 0) continue;
    if (lane == 0 && j < a.m) a.qjl[rec * ((a.m + 31) >> 5) + i32] = bits;
    if (j == 0) a.rnorm[rec] = nrm[u] * rho[u];
  }
}

template <int QS>
__global__ void __launch_bounds__(256) k_quantize_small(QuantArgs a, int dpad) {
  extern __shared__ float sh[];
  quantize_small_body<QS>(a, dpad, blockIdx.x, sh);
}

// ----------------------------------------------------------------------------
// Query pre-rotation: q' = Pi q, s = S q' (PR rows per block).
// ----------------------------------------------------------------------------
// Tile prefix of the segment-partitioned decode: tiles[b] = Hkv * sum over
// b' < b of ceil(len_b' / 16), len = min(max(seq_lens, 0), max_T); one block.
__device__ void tile_plan(const int32_t* seq_lens, int B, int Hkv, int64_t max_T, int64_t* tiles) {
  __shared__ int64_t s_w[32];
  __shared__ int64_t s_carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nt = blockDim.x;
  if (tid == 0) {
    s_carry = 0;
    tiles[0] = 0;
  }
  __syncthreads();
  for (int base = 0; base < B; base += nt) {
    const int b = base + tid;
    int64_t v = 0;
    if (b < B) {
      const int64_t len = min((int64_t)max(seq_lens[b], 0), max_T);
      v = (len + 15) / 16 * Hkv;
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t n = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += n;
    }
    if (lane == 31) s_w[warp] = v;
    __syncthreads();
    int64_t off = s_carry;
    for (int w = 0; w < warp; ++w) off += s_w[w];
    if (b < B) tiles[b + 1] = off + v;
    __syncthreads();
    if (tid == nt - 1) s_carry = off + v;
    __syncthreads();
  }
}

// Query operands of the int8 key product, for the PR rows of a block (thread
// j = coordinate j and QJL row j; d = m = blockDim = 128).
//
// The logit of a 2-bit key is l = n <q', c[idx]> + cq gamma <s, sigma>.  A
// symmetric 2-bit codebook is affine in the index bits, c[i0 + 2 i1] =
// c0 + w0 i0 + w1 i1 (w0 = c1 - c0, w1 = c2 - c0), and <s, sigma> =
// 2 <s, bit> - sum s, so both products are sums of query terms over set code
// bits.  The decode kernel's A operand holds code bit b of a word in byte
// b / 8, at bit position p = b % 8 (value 2^p); this side supplies for that
// position the integer Q = round(2^(S - p) w q'_j) (or 2^(S' - p) s_i),
// with S chosen so |Q| < 2^30, as four balanced base-256 digits (signed
// bytes), one per N-tile column.  The int32 products then sum to
// 2^S <w q', bits> exactly, digit by digit, and
//   scale * log2(e) * l = n (KA acc_key + KB) + gamma (QA acc_qjl + QB)
// with KA = 2^-S sl, KB = c0 sum(q') sl, QA = 2^(1-S') cq sl,
// QB = -sum(s) cq sl (sl = scale * log2(e)).
template <int PR>
__device__ void write_qop(const QopPlan& P, const float (&qv)[PR], const float (&sv)[PR], int64_t row0,
                          int nr) {
  __shared__ float s_red[PR][8][4];
  const int j = threadIdx.x, lane = j & 31, warp = j >> 5, nwarp = blockDim.x >> 5;
#pragma unroll
  for (int r = 0; r < PR; ++r) {
    float mq = fabsf(qv[r]), sq = qv[r], ms = fabsf(sv[r]), ss = sv[r];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mq = fmaxf(mq, __shfl_xor_sync(0xffffffffu, mq, o));
      sq += __shfl_xor_sync(0xffffffffu, sq, o);
      ms = fmaxf(ms, __shfl_xor_sync(0xffffffffu, ms, o));
      ss += __shfl_xor_sync(0xffffffffu, ss, o);
    }
    if (lane == 0) {
      s_red[r][warp][0] = mq;
      s_red[r][warp][1] = sq;
      s_red[r][warp][2] = ms;
      s_red[r][warp][3] = ss;
    }
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < PR; ++r) {
    if (r >= nr) break;   // uniform over the block
    float mq = 0.f, ms = 0.f;
    double sq = 0.0, ss = 0.0;
    for (int w = 0; w < nwarp; ++w) {
      mq = fmaxf(mq, s_red[r][w][0]);
      sq += s_red[r][w][1];
      ms = fmaxf(ms, s_red[r][w][2]);
      ss += s_red[r][w][3];
    }
    const QopExp ex = qop_exponents(P, mq, ms);
    const int64_t row = row0 + r;
    const int64_t b = row / P.Hq;
    const int h = (int)(row % P.Hq), kvh = h / P.G, hg = h % P.G;
    unsigned char* img = P.img + (b * (P.Hq / P.G) + kvh) * (int64_t)kQopBytes;
    qop_put_coord(P, img, hg, j, qv[r], sv[r], ex);
    if (j == 0) qop_put_constants(P, img, hg, ex, sq, ss);
  }
}

// PR query rows per block: thread j owns coordinate j of each row, so Pi and
// S are read once per block.
template <int PR>
__device__ __forceinline__ void prerotate_body(const void* q, int dtype, int64_t rows, int d, int dpad,
                                               int m, const float* PiT, const float* ST, float* qr,
                                               float* qs, int64_t blk, float* sh,
                                               const QopPlan* qop = nullptr) {
  float* sq = sh;                  // [PR][dpad]: q, later q'
  float* Ms = sh + PR * dpad;      // [2][MV_KC][dpad]
  const int j = threadIdx.x;       // blockDim = dpad
  const int64_t row0 = blk * PR;
  const int nr = (int)min((int64_t)PR, rows - row0);
#pragma unroll
  for (int r = 0; r < PR; ++r) sq[r * dpad + j] = (r < nr && j < d) ? load_elem(q, dtype, (row0 + r) * d + j) : 0.f;
  __syncthreads();
  float acc[PR], qv[PR];
  mv_rows<PR>(PiT, d, dpad, sq, Ms, acc);
#pragma unroll
  for (int r = 0; r < PR; ++r) {
    qv[r] = acc[r];
    sq[r * dpad + j] = acc[r];
    if (r < nr) qr[(row0 + r) * dpad + j] = acc[r];
  }
  __syncthreads();
  mv_rows<PR>(ST, d, dpad, sq, Ms, acc);
#pragma unroll
  for (int r = 0; r < PR; ++r) {
    acc[r] = (j < m) ? acc[r] : 0.f;
    if (r < nr) qs[(row0 + r) * dpad + j] = acc[r];
  }
  if (qop && qop->img) write_qop<PR>(*qop, qv, acc, row0, nr);
}

template <int PR>
__global__ void __launch_bounds__(256) k_prerotate(const void* q, int dtype, int64_t rows, int d,
                                                   int dpad, int m, const float* PiT, const float* ST,
                                                   float* qr, float* qs, const int32_t* seq_lens,
                                                   int B, int Hkv, int64_t max_T, int64_t* tiles,
                                                   QopPlan qop) {
  extern __shared__ float sh[];
  prerotate_body<PR>(q, dtype, rows, d, dpad, m, PiT, ST, qr, qs, blockIdx.x, sh, &qop);
  if (tiles && blockIdx.x == 0) tile_plan(seq_lens, B, Hkv, max_T, tiles);
}

// ----------------------------------------------------------------------------
// Decode-step preparation in one launch: blocks [0, n) append the new key
// vectors, [n, 2n) the new value vectors (n = B Hkv, one vector per block),
// the rest pre-rotate the queries (two rows per block); block 2n also writes
// the attention lengths min(pos + 1, max_T) (0 for pos < 0) and, for the
// tensor-core decode, their tile prefix.
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_step_prep(StepPrep s, int d, int dpad, int m, const float* PiT,
                                                   const float* ST) {
  extern __shared__ float sh[];
  int64_t blk = blockIdx.x;
  if (blk < s.nkv) {
    quantize_small_body<1>(s.k, dpad, blk, sh);
    return;
  }
  blk -= s.nkv;
  if (blk < s.nkv) {
    quantize_small_body<1>(s.v, dpad, blk, sh);
    return;
  }
  blk -= s.nkv;
  prerotate_body<2>(s.q, s.qdtype, s.qrows, d, dpad, m, PiT, ST, s.qr, s.qs, blk, sh, &s.qop);
  if (blk == 0) {
    for (int b = threadIdx.x; b < s.B; b += blockDim.x) {
      const int64_t p = s.pos[b];
      s.lens[b] = (int32_t)max((int64_t)0, min(p + 1, s.max_T));
    }
    __syncthreads();
    if (s.tiles) tile_plan(s.lens, s.B, s.Hkv, s.max_T, s.tiles);
  }
}

// ----------------------------------------------------------------------------
// Latency-shaped small kernels for d <= 128 (dpad <= 128): the decode step's
// appends, the query pre-rotation and the merge process a few vectors each,
// so their time is a chain of dependent memory round trips, not bandwidth.
// A CTA of FAST_T = 512 threads splits every matrix product four ways over
// the k range: thread (j, quarter) = (tid % 128, tid / 128) reads its 32
// matrix entries in one unrolled burst of independent L1/L2 loads (no chain
// of streamed chunks), and the four partial sums meet in shared memory as
// (p0 + p1) + (p2 + p3).  Every caller of these helpers uses the same order,
// so an append inside the decode step and a separate append (or the query
// rotation of the decode step and of a separate decode) agree bit for bit.
// ----------------------------------------------------------------------------
constexpr int FAST_T = 512;
constexpr int FAST_KQ = 32;   // k entries per thread: four quarters cover d <= 128

// This thread's entries M[k][j] of its k quarter (M is [d][dpad], k-major;
// zero beyond d or dpad): issued together, one round trip.  The loads are
// volatile asm so that they stay where the caller puts them (ahead of the
// other round trips) instead of being sunk to their first use.
__device__ __forceinline__ void load_quarter(const float* __restrict__ M, int d, int dpad, float (&w)[FAST_KQ]) {
  const int j = threadIdx.x & 127, k0 = (threadIdx.x >> 7) * FAST_KQ;
  const bool jok = j < dpad;
#pragma unroll
  for (int kk = 0; kk < FAST_KQ; ++kk) {
    float v = 0.f;
    if (jok && k0 + kk < d)
      asm volatile("ld.global.nc.f32 %0, [%1];\n" : "=f"(v) : "l"(M + (size_t)(k0 + kk) * dpad + j));
    w[kk] = v;
  }
}
// acc[r] = sum over this thread's k quarter of w[kk] x[r][k0 + kk] (w from
// load_quarter; x rows of 128 floats with zeros beyond d).
template <int R>
__device__ __forceinline__ void dot_w(const float (&w)[FAST_KQ], const float* x, float (&acc)[R]) {
  const int k0 = (threadIdx.x >> 7) * FAST_KQ;
#pragma unroll
  for (int r = 0; r < R; ++r) acc[r] = 0.f;
#pragma unroll
  for (int kk = 0; kk < FAST_KQ; kk += 4) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float4 x4 = *reinterpret_cast<const float4*>(x + r * 128 + k0 + kk);
      acc[r] = fmaf(w[kk], x4.x, acc[r]);
      acc[r] = fmaf(w[kk + 1], x4.y, acc[r]);
      acc[r] = fmaf(w[kk + 2], x4.z, acc[r]);
      acc[r] = fmaf(w[kk + 3], x4.w, acc[r]);
    }
  }
}
// The four quarters' partial sums of output (r, j) (red: [4][R][128]).
__device__ __forceinline__ float sum_quarters(const float* red, int R, int r, int j) {
  return (red[(0 * R + r) * 128 + j] + red[(1 * R + r) * 128 + j]) +
         (red[(2 * R + r) * 128 + j] + red[(3 * R + r) * 128 + j]);
}

// quantize_small_body for QS vectors per 512-thread CTA: the coordinate
// threads tid < dpad (warps 0 .. dpad / 32 - 1) take the roles of the
// small body's threads (Lloyd-Max index, packing, QJL signs); all threads
// take part in the two matrix products.  sh: [QS][128] + [4][QS][128] floats.
template <int QS>
__device__ __forceinline__ void quantize_fast_body(const QuantArgs& a, int dpad, int64_t blk, float* sh) {
  float* xs = sh;                // [QS][128]: x, later r
  float* red = sh + QS * 128;    // [4][QS][128]
  __shared__ float s_nx[QS][4], s_nc[QS][4], s_nr[QS][4];
  __shared__ float s_cen[kMaxLevels], s_bnd[kMaxLevels];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, j = tid & 127;
  const int nwarp = dpad >> 5;
  const bool cw = tid < dpad;    // a coordinate thread (j = tid)
  const int64_t v0 = blk * QS;
  const int nv = (int)min((int64_t)QS, a.n - v0);
  for (int e = tid; e < kMaxLevels; e += blockDim.x) {
    s_cen[e] = (e < (1 << a.bits)) ? a.cen[e] : 0.f;
    s_bnd[e] = (e < a.nbnd) ? a.bnd[e] : INFINITY;
  }
#pragma unroll
  for (int u = 0; u < QS; ++u) {
    float xj = 0.f;
    if (tid < 128) {
      xj = (u < nv && j < a.d) ? load_elem(a.x, a.dtype, (v0 + u) * a.ld + j) : 0.f;
      xs[u * 128 + j] = xj;
    }
    const float t = warp_sum(xj * xj);
    if (lane == 0 && warp < 4) s_nx[u][warp] = t;
  }
  __syncthreads();
  float nrm[QS];
#pragma unroll
  for (int u = 0; u < QS; ++u) {
    float t = 0.f;
    for (int w = 0; w < nwarp; ++w) t += s_nx[u][w];
    nrm[u] = sqrtf(t);
  }
  {
    float acc[QS], wp[FAST_KQ];   // (loaded here: two CTAs per SM fit the registers)
    load_quarter(a.PiT, a.d, dpad, wp);
    dot_w<QS>(wp, xs, acc);
#pragma unroll
    for (int u = 0; u < QS; ++u) red[((tid >> 7) * QS + u) * 128 + j] = acc[u];
  }
  __syncthreads();
  float r[QS];
  int ids[QS];
#pragma unroll
  for (int u = 0; u < QS; ++u) {
    ids[u] = 0;
    r[u] = 0.f;
    if (cw) {
      const float pj = sum_quarters(red, QS, u, j);
      const float y = (nrm[u] > 0.f && j < a.d) ? pj / nrm[u] : 0.f;
      ids[u] = lm_index(y, s_bnd, a.nbnd);
      r[u] = (j < a.d) ? y - s_cen[ids[u]] : 0.f;
    }
  }
  if (a.nc) {   // uniform; norm correction: store n / |c[idx]| (MSE-only, no QJL stage follows)
#pragma unroll
    for (int u = 0; u < QS; ++u) {
      const float cj = (cw && j < a.d) ? s_cen[ids[u]] : 0.f;
      const float cc = warp_sum(cj * cj);
      if (lane == 0 && warp < 4) s_nc[u][warp] = cc;
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < QS; ++u) {
      float t = 0.f;
      for (int w = 0; w < nwarp; ++w) t += s_nc[u][w];
      nrm[u] = nrm[u] / sqrtf(t);
    }
  }
  const int i32 = j >> 5;
  if (warp < nwarp) {   // warp-uniform: the coordinate warps pack and store
#pragma unroll
    for (int u = 0; u < QS; ++u) {
      if (u >= nv) continue;
      const int64_t rec = out_record(a, v0 + u);
      if (rec < 0) continue;   // uniform (one sequence per vector)
      const uint32_t iv = (j < a.d) ? (uint32_t)ids[u] : 0u;
      if (a.bits == 3) {
        const int w2 = (a.d + 15) >> 4;
        const uint32_t lo = field_word(iv & 3u, 2, lane);
        const uint32_t hi = field_word(iv >> 2, 1, lane);
        const int wlo = 2 * i32 + (lane >> 4);
        if ((lane & 15) == 0 && wlo < w2) a.codes[rec * a.words + wlo] = lo;
        if (lane == 0) a.codes[rec * a.words + w2 + i32] = hi;
      } else {
        const int per = 32 / a.bits;
        const uint32_t wv = field_word(iv, a.bits, lane);
        const int wi = a.bits * i32 + lane / per;
        if (lane % per == 0 && wi < a.words) a.codes[rec * a.words + wi] = wv;
      }
      if (j == 0) store_norm(a.norm, rec, nrm[u], a.nf16);
    }
  }
  if (a.m == 0) return;
#pragma unroll
  for (int u = 0; u < QS; ++u) {
    if (tid < 128) xs[u * 128 + j] = r[u];   // r = 0 beyond d
    const float t = warp_sum(r[u] * r[u]);
    if (lane == 0 && warp < 4) s_nr[u][warp] = t;
  }
  __syncthreads();   // also: every read of red above is done
  {
    float acc[QS], ws[FAST_KQ];
    load_quarter(a.ST, a.d, dpad, ws);
    dot_w<QS>(ws, xs, acc);
#pragma unroll
    for (int u = 0; u < QS; ++u) red[((tid >> 7) * QS + u) * 128 + j] = acc[u];
  }
  __syncthreads();
  if (warp < nwarp) {
#pragma unroll
    for (int u = 0; u < QS; ++u) {
      float rho = 0.f;
      for (int w = 0; w < nwarp; ++w) rho += s_nr[u][w];
      rho = sqrtf(rho);
      const float sj = sum_quarters(red, QS, u, j);
      const uint32_t bits = __ballot_sync(0xffffffffu, sj >= 0.f && j < a.m);
      if (u >= nv) continue;
      const int64_t rec = out_record(a, v0 + u);
      if (rec < 0) continue;
      if (lane == 0 && j < a.m) a.qjl[rec * ((a.m + 31) >> 5) + i32] = bits;
      if (j == 0) a.rnorm[rec] = nrm[u] * rho;
    }
  }
}

template <int QS>
__global__ void __launch_bounds__(FAST_T) k_quantize_fast(QuantArgs a, int dpad) {
  __shared__ __align__(16) float sh[5 * QS * 128];
  quantize_fast_body<QS>(a, dpad, blockIdx.x, sh);
}

// Query rows row0 .. row0 + R - 1 (R rows of one CTA): q' = Pi q, s = S q',
// written to qr / qs ([rows][dpad]) and, with qop->img, as int8 operand
// images (tq_qop.cuh).  sh: [R][128] q', [R][128] s, [4][R][128].
template <int R, bool HOIST>
__device__ __forceinline__ void prerotate_fast_body(const void* q, int dtype, int64_t rows, int d, int dpad,
                                                    int m, const float* PiT, const float* ST, float* qr, float* qs,
                                                    int64_t blk, const QopPlan* qop, float* sh) {
  float* xs = sh;               // [R][128]: q, then q'
  float* ys = sh + R * 128;     // [R][128]: s
  float* red = ys + R * 128;    // [4][R][128]
  __shared__ float s_sum[R][2];
  __shared__ int s_ex[R][2];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, j = tid & 127;
  const int64_t row0 = blk * R;
  const int nr = (int)min((int64_t)R, rows - row0);
  float wm[2][FAST_KQ];   // quarters of Pi^T and S^T: up front (HOIST) or before each product
  if (HOIST) {
    load_quarter(PiT, d, dpad, wm[0]);
    load_quarter(ST, d, dpad, wm[1]);
  }
  for (int e = tid; e < R * 128; e += blockDim.x) {
    const int r = e >> 7, jj = e & 127;
    xs[e] = (r < nr && jj < d) ? load_elem(q, dtype, (row0 + r) * d + jj) : 0.f;
  }
  __syncthreads();
#pragma unroll
  for (int pass = 0; pass < 2; ++pass) {
    float acc[R];
    if (!HOIST) load_quarter(pass == 0 ? PiT : ST, d, dpad, wm[pass]);
    dot_w<R>(wm[pass], xs, acc);
#pragma unroll
    for (int r = 0; r < R; ++r) red[((tid >> 7) * R + r) * 128 + j] = acc[r];
    __syncthreads();
    float* y = pass == 0 ? xs : ys;   // q' replaces q: every read of xs is done
    float* g = pass == 0 ? qr : qs;
    for (int e = tid; e < R * 128; e += blockDim.x) {
      const int r = e >> 7, jj = e & 127;
      float v = sum_quarters(red, R, r, jj);
      if (pass == 1 && jj >= m) v = 0.f;
      y[e] = v;
      if (r < nr && jj < dpad) g[(row0 + r) * dpad + jj] = v;
    }
    __syncthreads();
  }
  if (!qop || !qop->img) return;
  if (warp < R) {   // head statistics of row warp: max |q'|, sum q', max |s|, sum s
    float mq = 0.f, sq = 0.f, ms = 0.f, ss = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float qv = xs[warp * 128 + lane + 32 * i], sv = ys[warp * 128 + lane + 32 * i];
      mq = fmaxf(mq, fabsf(qv));
      sq += qv;
      ms = fmaxf(ms, fabsf(sv));
      ss += sv;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mq = fmaxf(mq, __shfl_xor_sync(0xffffffffu, mq, o));
      sq += __shfl_xor_sync(0xffffffffu, sq, o);
      ms = fmaxf(ms, __shfl_xor_sync(0xffffffffu, ms, o));
      ss += __shfl_xor_sync(0xffffffffu, ss, o);
    }
    if (lane == 0) {
      const QopExp ex = qop_exponents(*qop, mq, ms);
      s_ex[warp][0] = ex.S;
      s_ex[warp][1] = ex.S2;
      s_sum[warp][0] = sq;
      s_sum[warp][1] = ss;
    }
  }
  __syncthreads();
  for (int e = tid; e < nr * 128; e += blockDim.x) {
    const int r = e >> 7, jj = e & 127;
    const int64_t row = row0 + r;
    const int64_t b = row / qop->Hq;
    const int h = (int)(row % qop->Hq), kvh = h / qop->G, hg = h % qop->G;
    unsigned char* img = qop->img + (b * (qop->Hq / qop->G) + kvh) * (int64_t)kQopBytes;
    QopExp ex;
    ex.S = s_ex[r][0];
    ex.S2 = s_ex[r][1];
    qop_put_coord(*qop, img, hg, jj, xs[e], ys[e], ex);
    if (jj == 0) qop_put_constants(*qop, img, hg, ex, (double)s_sum[r][0], (double)s_sum[r][1]);
  }
}

constexpr int FAST_R = 4;   // query rows per pre-rotation CTA

__global__ void __launch_bounds__(FAST_T) k_prerotate_fast(const void* q, int dtype, int64_t rows, int d, int dpad,
                                                         int m, const float* PiT, const float* ST, float* qr,
                                                         float* qs, const int32_t* seq_lens, int B, int Hkv,
                                                         int64_t max_T, int64_t* tiles, QopPlan qop) {
  __shared__ __align__(16) float sh[6 * FAST_R * 128];
  prerotate_fast_body<FAST_R, true>(q, dtype, rows, d, dpad, m, PiT, ST, qr, qs, blockIdx.x, &qop, sh);
  if (tiles && blockIdx.x == 0) tile_plan(seq_lens, B, Hkv, max_T, tiles);
}

// The decode step's preparation with the fast bodies: blocks [0, a) append
// the new keys, STEP_QS per block, [a, 2a) the new values (a = ceil(B Hkv /
// STEP_QS)), the rest pre-rotate FAST_R query rows each; the first query
// block writes the lengths and the tile prefix.  Two vectors per append block
// share each thread's matrix loads and keep the grid within one wave of two
// 512-thread CTAs per SM on the Llama-3-8B decode shape.
constexpr int STEP_QS = 2;
__global__ void __launch_bounds__(FAST_T, 2) k_step_prep_fast(StepPrep s, int d, int dpad, int m,
                                                            const float* PiT, const float* ST) {
  __shared__ __align__(16) float sh[6 * FAST_R * 128];
  static_assert(5 * STEP_QS * 128 <= 6 * FAST_R * 128, "append staging fits the shared buffer");
  const int64_t na = (s.nkv + STEP_QS - 1) / STEP_QS;
  int64_t blk = blockIdx.x;
  if (blk < na) {
    quantize_fast_body<STEP_QS>(s.k, dpad, blk, sh);
    return;
  }
  blk -= na;
  if (blk < na) {
    quantize_fast_body<STEP_QS>(s.v, dpad, blk, sh);
    return;
  }
  blk -= na;
  // matrix loads before each product: two CTAs per SM fit the registers
  prerotate_fast_body<FAST_R, false>(s.q, s.qdtype, s.qrows, d, dpad, m, PiT, ST, s.qr, s.qs, blk, &s.qop, sh);
  if (blk == 0) {
    for (int b = threadIdx.x; b < s.B; b += blockDim.x) {
      const int64_t p = s.pos[b];
      s.lens[b] = (int32_t)max((int64_t)0, min(p + 1, s.max_T));
    }
    __syncthreads();
    if (s.tiles) tile_plan(s.lens, s.B, s.Hkv, s.max_T, s.tiles);
  }
}

// ----------------------------------------------------------------------------
// Split-K decode attention, one CTA per (split, kv head, sequence), 128
// threads.  Per tile of 128 tokens: (1) thread t computes the logits of token
// t for the G query heads of the group straight from the packed key codes,
// (2) online-softmax update of the running max / sum per head, (3) thread j
// accumulates o_rot[j] += p_t * |v_t| * cv[vidx_tj] (the rotated-domain value;
// Pi^T is applied once after the merge).
// ----------------------------------------------------------------------------
constexpr int AT = 128;   // tokens per tile = threads per CTA
constexpr int GMAX = 16;

template <int J>
__global__ void __launch_bounds__(AT) k_attn_split(AttnArgs a) {
  constexpr int DP = J * 32;
  constexpr int JJ = (DP + AT - 1) / AT;  // value dims per thread
  extern __shared__ float sh[];
  float* sq = sh;                       // [G][DP]
  float* ssv = sq + a.G * DP;           // [G][DP]
  float* sp = ssv + a.G * DP;           // [AT][G]   p * |v|
  uint32_t* svc = reinterpret_cast<uint32_t*>(sp + AT * a.G);  // [AT][wv]
  __shared__ float s_ck[kMaxLevels], s_cv[kMaxLevels];
  __shared__ float s_wred[AT / 32][GMAX];

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = a.G;
  for (int e = tid; e < kMaxLevels; e += AT) {
    s_ck[e] = (e < (1 << a.bk)) ? a.ck[e] : 0.f;
    s_cv[e] = (e < (1 << a.bv)) ? a.cv[e] : 0.f;
  }
  for (int e = tid; e < G * DP; e += AT) {
    const int h = e / DP, j = e % DP;
    const int64_t row = (int64_t)b * a.Hq + (int64_t)g * G + h;
    sq[e] = a.qr[row * DP + j];
    ssv[e] = a.qs[row * DP + j];
  }
  const int64_t T = min((int64_t)a.seq_lens[b], a.max_T);
  const int64_t t_begin = (int64_t)split * a.chunk;
  const int64_t t_end = min(T, t_begin + a.chunk);
  float m_run[GMAX], l_run[GMAX], o[GMAX][JJ];
#pragma unroll
  for (int h = 0; h < GMAX; ++h) {
    m_run[h] = kNegInf;
    l_run[h] = 0.f;
#pragma unroll
    for (int jj = 0; jj < JJ; ++jj) o[h][jj] = 0.f;
  }
  __syncthreads();
  const int64_t kv_row0 = ((int64_t)b * a.Hkv + g) * a.max_T;
  const int kw = a.wk, vw = a.wv, mw = (a.m + 31) >> 5;

  for (int64_t t0 = t_begin; t0 < t_end; t0 += AT) {
    const int64_t t = t0 + tid;
    const bool valid = t < t_end;
    const int ntile = (int)min((int64_t)AT, t_end - t0);
    float sc[GMAX];
#pragma unroll
    for (int h = 0; h < GMAX; ++h) sc[h] = kNegInf;
    if (valid) {
      const int64_t r = kv_row0 + t;
      uint32_t w[64];   // up to d = 256 at 8 bits
      for (int e = 0; e < kw; ++e) w[e] = a.kcodes[r * kw + e];
      float acc[GMAX], acc2[GMAX];
#pragma unroll
      for (int h = 0; h < GMAX; ++h) acc[h] = acc2[h] = 0.f;
      for (int j = 0; j < a.d; ++j) {
        const float c = s_ck[code_index(w, a.bk, a.d, j)];
#pragma unroll
        for (int h = 0; h < GMAX; ++h)
          if (h < G) acc[h] = fmaf(sq[h * DP + j], c, acc[h]);
      }
      for (int wi = 0; wi < mw; ++wi) {
        const uint32_t bitsw = a.kqjl[r * mw + wi];
        const int lim = min(32, a.m - 32 * wi);
        for (int e = 0; e < lim; ++e) {
          const bool pos = (bitsw >> e) & 1u;
          const int i = 32 * wi + e;
#pragma unroll
          for (int h = 0; h < GMAX; ++h)
            if (h < G) acc2[h] += pos ? ssv[h * DP + i] : -ssv[h * DP + i];
        }
      }
      const float kn = load_norm(a.knorm, r, a.nf16);
      const float kg = a.m > 0 ? a.krnorm[r] * a.cq : 0.f;
#pragma unroll
      for (int h = 0; h < GMAX; ++h)
        if (h < G) sc[h] = (kn * acc[h] + kg * acc2[h]) * a.scale_log2;
    }
    // Tile max per head.
#pragma unroll
    for (int h = 0; h < GMAX; ++h) {
      if (h < G) {
        const float mx = warp_max(sc[h]);
        if (lane == 0) s_wred[warp][h] = mx;
      }
    }
    // Stage this tile's value codes (contiguous words) while the max settles.
    for (int e = tid; e < ntile * vw; e += AT) svc[e] = a.vcodes[(kv_row0 + t0) * vw + e];
    __syncthreads();
    float alpha[GMAX], mnew[GMAX];
#pragma unroll
    for (int h = 0; h < GMAX; ++h) {
      if (h < G) {
        float mx = s_wred[0][h];
        for (int ww = 1; ww < AT / 32; ++ww) mx = fmaxf(mx, s_wred[ww][h]);
        mnew[h] = fmaxf(m_run[h], mx);
        alpha[h] = (mnew[h] == kNegInf) ? 1.f : exp2f(m_run[h] - mnew[h]);
      }
    }
    const float vn = valid ? load_norm(a.vnorm, kv_row0 + t, a.nf16) : 0.f;
    float psum[GMAX];
#pragma unroll
    for (int h = 0; h < GMAX; ++h) {
      if (h < G) {
        const float p = valid ? exp2f(sc[h] - mnew[h]) : 0.f;
        sp[tid * G + h] = p * vn;
        psum[h] = p;
      }
    }
    __syncthreads();  // s_wred reads done before reuse
#pragma unroll
    for (int h = 0; h < GMAX; ++h) {
      if (h < G) {
        const float sm = warp_sum(psum[h]);
        if (lane == 0) s_wred[warp][h] = sm;
      }
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < GMAX; ++h) {
      if (h < G) {
        float sm = 0.f;
        for (int ww = 0; ww < AT / 32; ++ww) sm += s_wred[ww][h];
        l_run[h] = l_run[h] * alpha[h] + sm;
        m_run[h] = mnew[h];
#pragma unroll
        for (int jj = 0; jj < JJ; ++jj) o[h][jj] *= alpha[h];
      }
    }
#pragma unroll
    for (int jj = 0; jj < JJ; ++jj) {
      const int j = tid + AT * jj;
      if (j < a.d) {
        for (int tt = 0; tt < ntile; ++tt) {
          const float c = s_cv[code_index(svc + tt * vw, a.bv, a.d, j)];
#pragma unroll
          for (int h = 0; h < GMAX; ++h)
            if (h < G) o[h][jj] = fmaf(sp[tt * G + h], c, o[h][jj]);
        }
      }
    }
    __syncthreads();
  }
  // Partial state (m, l, o_rot) per query head.
#pragma unroll
  for (int h = 0; h < GMAX; ++h) {
    if (h >= G) break;
    const int64_t row = (int64_t)b * a.Hq + (int64_t)g * G + h;
    float* pp = a.part + (row * a.splits + split) * (DP + 2);
    if (tid == 0) {
      pp[0] = m_run[h];
      pp[1] = l_run[h];
    }
#pragma unroll
    for (int jj = 0; jj < JJ; ++jj) {
      const int j = tid + AT * jj;
      if (j < DP) pp[2 + j] = o[h][jj];
    }
  }
}

// Log-sum-exp merge of the split partials and the final o = Pi^T o_rot.
// The split maxima and sums are staged in shared memory with one load per
// thread; each thread then folds its coordinate over the splits with
// independent loads (eight in flight).
//
// Split path: row r's partials are part[r][0..splits).  Segment path (tiles
// != null): the tiles are split into ranges [w W / N, (w + 1) W / N) over
// N = min(nw, W) owners, each with wpu partial writers; the partials of row
// (b, h) sit in slots wpu (f + i) .. wpu (l + i) + wpu - 1, i = b Hkv + kv
// head, laid out [slot][G][dpad + 2], where f and l are the first and last
// owners whose ranges meet the row's tiles.
__global__ void __launch_bounds__(128) k_attn_merge(const float* part, int splits, int d, int dpad,
                                                    const float* Pi, float* out,
                                                    const int64_t* tiles, int B, int Hq, int Hkv,
                                                    int nw, int wpu) {
  extern __shared__ float sh[];
  float* so = sh;                 // [dpad]
  float* sw = sh + dpad;          // [splits] weights exp2(m_s - M)
  __shared__ float s_red[4];
  __shared__ float s_M, s_L;
  const int64_t row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* pr = part + row * splits * (dpad + 2);
  int64_t sstride = dpad + 2;
  if (tiles) {
    const int b = (int)(row / Hq), h = (int)(row % Hq), G = Hq / Hkv;
    const int kvh = h / G, hg = h % G;
    const int64_t W = tiles[B];
    const int64_t tb = (tiles[b + 1] - tiles[b]) / Hkv;
    splits = 0;
    if (tb > 0) {
      const int64_t N = min((int64_t)nw, W);
      const int64_t S = tiles[b] + kvh * tb, E = S + tb;
      const int64_t f = ((S + 1) * N + W - 1) / W - 1, l = (E * N + W - 1) / W - 1;
      pr = part + (wpu * (f + (int64_t)b * Hkv + kvh) * G + hg) * (dpad + 2);
      sstride = (int64_t)G * (dpad + 2);
      splits = (int)(wpu * (l - f + 1));
    }
  }
  float mloc = -INFINITY;
  for (int sidx = tid; sidx < splits; sidx += blockDim.x) {
    const float ms = pr[(int64_t)sidx * sstride];
    sw[sidx] = ms;
    mloc = fmaxf(mloc, ms);
  }
  mloc = warp_max(mloc);
  if (lane == 0) s_red[warp] = mloc;
  __syncthreads();
  if (tid == 0) s_M = fmaxf(fmaxf(s_red[0], s_red[1]), fmaxf(s_red[2], s_red[3]));
  __syncthreads();
  const float M = s_M;
  float lloc = 0.f;
  for (int sidx = tid; sidx < splits; sidx += blockDim.x) {
    const float ms = sw[sidx];
    const float w = (ms == -INFINITY) ? 0.f : exp2f(ms - M);
    sw[sidx] = w;
    lloc = fmaf(w, pr[(int64_t)sidx * sstride + 1], lloc);
  }
  lloc = warp_sum(lloc);
  __syncthreads();
  if (lane == 0) s_red[warp] = lloc;
  __syncthreads();
  if (tid == 0) s_L = (s_red[0] + s_red[1]) + (s_red[2] + s_red[3]);
  __syncthreads();
  const float L = s_L;
  for (int j = tid; j < dpad; j += blockDim.x) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    int sidx = 0;
    for (; sidx + 8 <= splits; sidx += 8) {
#pragma unroll
      for (int u = 0; u < 8; ++u)
        acc[u] = fmaf(sw[sidx + u], pr[(int64_t)(sidx + u) * sstride + 2 + j], acc[u]);
    }
    for (; sidx < splits; ++sidx) acc[0] = fmaf(sw[sidx], pr[(int64_t)sidx * sstride + 2 + j], acc[0]);
    const float tot = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
    so[j] = (L > 0.f) ? tot / L : 0.f;
  }
  __syncthreads();
  for (int i = tid; i < d; i += blockDim.x) {
    float a4[4] = {0.f, 0.f, 0.f, 0.f};
    int j = 0;
    for (; j + 4 <= d; j += 4) {
#pragma unroll
      for (int u = 0; u < 4; ++u) a4[u] = fmaf(Pi[(size_t)(j + u) * d + i], so[j + u], a4[u]);
    }
    for (; j < d; ++j) a4[0] = fmaf(Pi[(size_t)j * d + i], so[j], a4[0]);
    out[row * d + i] = (a4[0] + a4[1]) + (a4[2] + a4[3]);
  }
}

// ----------------------------------------------------------------------------
// The merge for d <= 128, one 512-thread CTA per KV group (its G <= 16 rows
// share the segment path's slot range): per row, weights w_s / L from the
// partials' (m, l) (one warp per row), o = sum (w_s / L) o_s, then
// out = Pi^T o with the k range of the product split four ways as in
// dot_w (Pi is [d][d] row-major: out_i = sum_j Pi[j][i] o_j), four
// rows at a time.  sh: [Gp][128] o (Gp = G rounded up to 4, zero padding
// rows), [4][4][128] partial sums, [G][slot_cap] weights.
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(FAST_T) k_attn_merge_fast(const float* part, int splits, int d, int dpad,
                                                          const float* Pi, float* out, const int64_t* tiles, int B,
                                                          int Hq, int Hkv, int nw, int wpu, int slot_cap) {
  extern __shared__ __align__(16) float sh[];
  const int G = Hq / Hkv, Gp = (G + 3) & ~3;
  float* so = sh;                       // [Gp][128]
  float* red = so + Gp * 128;           // [4][4][128]
  float* sw = red + 4 * 4 * 128;        // [G][slot_cap]
  const int u = blockIdx.x, b = u / Hkv, kvh = u % Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarp = blockDim.x >> 5;
  const float* pr0;
  int64_t sstride, rstride;
  int nsl;
  if (tiles) {
    const int64_t W = tiles[B];
    const int64_t tb = (tiles[b + 1] - tiles[b]) / Hkv;
    nsl = 0;
    pr0 = part;
    if (tb > 0) {
      const int64_t N = min((int64_t)nw, W);
      const int64_t S = tiles[b] + kvh * tb, E = S + tb;
      const int64_t f = ((S + 1) * N + W - 1) / W - 1, l = (E * N + W - 1) / W - 1;
      pr0 = part + wpu * (f + (int64_t)b * Hkv + kvh) * G * (int64_t)(dpad + 2);
      nsl = (int)(wpu * (l - f + 1));
    }
    sstride = (int64_t)G * (dpad + 2);
    rstride = dpad + 2;
  } else {
    pr0 = part + (int64_t)u * G * splits * (dpad + 2);
    sstride = dpad + 2;
    rstride = (int64_t)splits * (dpad + 2);
    nsl = splits;
  }
  for (int r = warp; r < G; r += nwarp) {
    const float* pr = pr0 + r * rstride;
    // (m, l) of the first 32 slots stay in registers; more slots are re-read
    const float2 ml0 = lane < nsl ? *reinterpret_cast<const float2*>(pr + lane * sstride)
                                  : make_float2(-INFINITY, 0.f);
    float mx = ml0.x;
    for (int sl = lane + 32; sl < nsl; sl += 32) mx = fmaxf(mx, pr[sl * sstride]);
    mx = warp_max(mx);
    float lsum = 0.f;
    for (int sl = lane; sl < nsl; sl += 32) {
      const float2 ml = sl < 32 ? ml0 : *reinterpret_cast<const float2*>(pr + sl * sstride);
      const float w = (ml.x == -INFINITY) ? 0.f : exp2f(ml.x - mx);
      sw[r * slot_cap + sl] = w;
      lsum = fmaf(w, ml.y, lsum);
    }
    lsum = warp_sum(lsum);
    const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
    __syncwarp();
    for (int sl = lane; sl < nsl; sl += 32) sw[r * slot_cap + sl] *= inv;
  }
  __syncthreads();
  for (int e = tid; e < Gp * 128; e += blockDim.x) {
    const int r = e >> 7, j = e & 127;
    float tot = 0.f;
    if (r < G && j < d) {
      const float* pr = pr0 + r * rstride + 2 + j;
      const float* wr = sw + r * slot_cap;
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      int sl = 0;
      for (; sl + 8 <= nsl; sl += 8) {
#pragma unroll
        for (int v = 0; v < 8; ++v) acc[v] = fmaf(wr[sl + v], pr[(int64_t)(sl + v) * sstride], acc[v]);
      }
      for (; sl < nsl; ++sl) acc[0] = fmaf(wr[sl], pr[(int64_t)sl * sstride], acc[0]);
      tot = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
    }
    so[e] = tot;
  }
  __syncthreads();
  // out_i = sum_j Pi[j][i] o_j: dot_w over Pi ([d][d], k = j) with x = o
  float wpi[FAST_KQ];   // this thread's quarter of Pi
  load_quarter(Pi, d, d, wpi);
  for (int r0 = 0; r0 < G; r0 += 4) {
    float acc[4];
    dot_w<4>(wpi, so + r0 * 128, acc);
    const int i = tid & 127, qt = tid >> 7;
#pragma unroll
    for (int r = 0; r < 4; ++r) red[(qt * 4 + r) * 128 + i] = acc[r];
    __syncthreads();
    for (int e = tid; e < 4 * 128; e += blockDim.x) {
      const int r = e >> 7, i2 = e & 127;
      if (r0 + r < G && i2 < d) out[((int64_t)u * G + r0 + r) * d + i2] = sum_quarters(red, 4, r, i2);
    }
    __syncthreads();
  }
}

// ----------------------------------------------------------------------------
// Logits of nq queries against nk packed keys.  Each CTA pre-rotates its QB
// queries into shared memory, then thread t scores key t of its slice.
// ----------------------------------------------------------------------------
constexpr int LQB = 8;

template <int J>
__global__ void __launch_bounds__(128) k_logits(const void* q, int dtype, int64_t nq, int d,
                                                int bk, int kw, int m, const float* PiT,
                                                const float* ST, const float* ck, float cq,
                                                const uint32_t* kcodes, const uint32_t* kqjl,
                                                const float* knorm, const float* krnorm,
                                                int64_t nk, int nf16, float* out) {
  constexpr int DP = J * 32;
  __shared__ float sx[LQB][DP], sq[LQB][DP], ss[LQB][DP];
  __shared__ float s_ck[kMaxLevels];
  const int tid = threadIdx.x;
  const int64_t q0 = (int64_t)blockIdx.y * LQB;
  for (int e = tid; e < kMaxLevels; e += blockDim.x) s_ck[e] = (e < (1 << bk)) ? ck[e] : 0.f;
  for (int e = tid; e < LQB * DP; e += blockDim.x) {
    const int qq = e / DP, k = e % DP;
    sx[qq][k] = (k < d && q0 + qq < nq) ? load_elem(q, dtype, (q0 + qq) * d + k) : 0.f;
  }
  __syncthreads();
  for (int e = tid; e < LQB * DP; e += blockDim.x) {
    const int qq = e / DP, j = e % DP;
    float acc = 0.f;
    for (int k = 0; k < d; ++k) acc = fmaf(PiT[(size_t)k * DP + j], sx[qq][k], acc);
    sq[qq][j] = acc;
  }
  __syncthreads();
  for (int e = tid; e < LQB * DP; e += blockDim.x) {
    const int qq = e / DP, i = e % DP;
    float acc = 0.f;
    if (i < m)
      for (int k = 0; k < d; ++k) acc = fmaf(ST[(size_t)k * DP + i], sq[qq][k], acc);
    ss[qq][i] = acc;
  }
  __syncthreads();
  const int64_t key = (int64_t)blockIdx.x * blockDim.x + tid;
  if (key >= nk) return;
  const int mw = (m + 31) >> 5;
  uint32_t w[64];   // up to d = 256 at 8 bits
  for (int e = 0; e < kw; ++e) w[e] = kcodes[key * kw + e];
  float acc[LQB], acc2[LQB];
#pragma unroll
  for (int qq = 0; qq < LQB; ++qq) acc[qq] = acc2[qq] = 0.f;
  for (int j = 0; j < d; ++j) {
    const float c = s_ck[code_index(w, bk, d, j)];
#pragma unroll
    for (int qq = 0; qq < LQB; ++qq) acc[qq] = fmaf(sq[qq][j], c, acc[qq]);
  }
  for (int wi = 0; wi < mw; ++wi) {
    const uint32_t bitsw = kqjl[key * mw + wi];
    const int lim = min(32, m - 32 * wi);
    for (int e = 0; e < lim; ++e) {
      const bool pos = (bitsw >> e) & 1u;
#pragma unroll
      for (int qq = 0; qq < LQB; ++qq) acc2[qq] += pos ? ss[qq][32 * wi + e] : -ss[qq][32 * wi + e];
    }
  }
  const float kn = load_norm(knorm, key, nf16);
  const float kg = m > 0 ? krnorm[key] * cq : 0.f;
#pragma unroll
  for (int qq = 0; qq < LQB; ++qq)
    if (q0 + qq < nq) out[(q0 + qq) * nk + key] = kn * acc[qq] + kg * acc2[qq];
}

// ----------------------------------------------------------------------------
// Dequantize one vector per CTA: rot_j = |x| c[idx_j] (+ C gamma (S^T sigma)_j),
// then x_hat = Pi^T rot.
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(128) k_dequant(int d, int dpad, int bits, int words, int m,
                                                 const float* Pi, const float* S,
                                                 const float* cen, float cq,
                                                 const uint32_t* codes, const uint32_t* qjl,
                                                 const float* norm, const float* rnorm,
                                                 int nf16, float* out) {
  extern __shared__ float sh[];
  float* srot = sh;  // [dpad]
  const int64_t v = blockIdx.x;
  const int mw = (m + 31) >> 5;
  const uint32_t* w = codes + v * words;
  const float n = load_norm(norm, v, nf16);
  const float kg = m > 0 ? rnorm[v] * cq : 0.f;
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    float r = n * cen[code_index(w, bits, d, j)];
    if (m > 0) {
      float acc = 0.f;
      for (int i = 0; i < m; ++i) {
        const bool pos = (qjl[v * mw + (i >> 5)] >> (i & 31)) & 1u;
        acc += pos ? S[(size_t)i * d + j] : -S[(size_t)i * d + j];
      }
      r = fmaf(kg, acc, r);
    }
    srot[j] = r;
  }
  __syncthreads();
  for (int k = threadIdx.x; k < d; k += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j < d; ++j) acc = fmaf(Pi[(size_t)j * d + k], srot[j], acc);
    out[v * d + k] = acc;
  }
}

// ----------------------------------------------------------------------------
// Top-k, final phase: one warp per query selects the k best of all candidate
// lists written by the tensor-core scoring kernel (tq_topk_mma.cu).
// Order: score descending, then index ascending.
// ----------------------------------------------------------------------------
__device__ __forceinline__ bool better(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

__global__ void __launch_bounds__(32) k_topk_final(const float* cand_v, const int* cand_i,
                                                   int nchunks, int K, int32_t* idx, float* score) {
  const int64_t q = blockIdx.x;
  const int lane = threadIdx.x;
  const int total = nchunks * K;
  const float* cv = cand_v + q * total;
  const int* ci = cand_i + q * total;
  float taken_v = INFINITY;
  int taken_i = -1;
  // K rounds; in each, the best candidate strictly after the previous pick.
  for (int r = 0; r < K; ++r) {
    float bv = kNegInf;
    int bi = INT_MAX;
    for (int e = lane; e < total; e += 32) {
      const float v = cv[e];
      const int i = ci[e];
      const bool after = better(taken_v, taken_i, v, i);
      if (after && better(v, i, bv, bi)) { bv = v; bi = i; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
    }
    if (lane == 0) {
      idx[q * K + r] = (bi == INT_MAX) ? -1 : bi;
      score[q * K + r] = bv;
    }
    taken_v = bv;
    taken_i = bi;
  }
}

template <int J>
cudaError_t quantize_J(const QuantArgs& a, cudaStream_t s) {
  constexpr int QV = quant_qv<J>();
  const size_t shm = (size_t)QWARPS * J * 32 * QV * sizeof(float);
  const int64_t groups = (a.n + QV - 1) / QV;
  int64_t blocks = (groups + QWARPS - 1) / QWARPS;
  blocks = blocks < 148 * 16 ? blocks : 148 * 16;
  k_quantize<J><<<(unsigned)blocks, QWARPS * 32, shm, s>>>(a);
  return cudaGetLastError();
}

template <int J>
cudaError_t attn_J(const tq_ctx* c, const AttnArgs& a, float* out, cudaStream_t s) {
  const size_t shm = (size_t)(2 * a.G * J * 32 + AT * a.G) * sizeof(float) +
                     (size_t)AT * a.wv * sizeof(uint32_t);
  dim3 grid(a.splits, a.Hkv, a.B);
  k_attn_split<J><<<grid, AT, shm, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_attn_merge(c, a, out, s);
}

}  // namespace

#define TQ_DISPATCH_J(J, ...)                      \
  switch (J) {                                     \
    case 1: { constexpr int JV = 1; __VA_ARGS__; } \
    case 2: { constexpr int JV = 2; __VA_ARGS__; } \
    case 3: { constexpr int JV = 3; __VA_ARGS__; } \
    case 4: { constexpr int JV = 4; __VA_ARGS__; } \
    case 5: { constexpr int JV = 5; __VA_ARGS__; } \
    case 6: { constexpr int JV = 6; __VA_ARGS__; } \
    case 7: { constexpr int JV = 7; __VA_ARGS__; } \
    case 8: { constexpr int JV = 8; __VA_ARGS__; } \
    default: return cudaErrorInvalidValue;         \
  }

cudaError_t launch_quantize(const tq_ctx* c, const QuantArgs& a, cudaStream_t s) {
  TQ_DISPATCH_J(c->J, return quantize_J<JV>(a, s));
}

cudaError_t launch_quantize_small(const tq_ctx* c, const QuantArgs& a, cudaStream_t s) {
  if (a.n == 0) return cudaSuccess;
  // One vector per block while that still fills the GPU; eight per block
  // (one read of Pi and S for all eight) beyond.  d <= 128: the fast bodies
  // (the same per-vector arithmetic for both batchings).
  if (c->dpad <= 128) {
    if (a.n <= 1024)
      k_quantize_fast<1><<<(unsigned)a.n, FAST_T, 0, s>>>(a, c->dpad);
    else
      k_quantize_fast<8><<<(unsigned)((a.n + 7) / 8), FAST_T, 0, s>>>(a, c->dpad);
    return cudaGetLastError();
  }
  if (a.n <= 1024) {
    k_quantize_small<1><<<(unsigned)a.n, c->dpad, (1 + 2 * MV_KC) * c->dpad * sizeof(float), s>>>(a, c->dpad);
  } else {
    k_quantize_small<8><<<(unsigned)((a.n + 7) / 8), c->dpad, (8 + 2 * MV_KC) * c->dpad * sizeof(float), s>>>(
        a, c->dpad);
  }
  return cudaGetLastError();
}

cudaError_t launch_step_prep(const tq_ctx* c, const StepPrep& sp, cudaStream_t s) {
  if (c->dpad <= 128) {
    const int64_t blocks = 2 * ((sp.nkv + STEP_QS - 1) / STEP_QS) + (sp.qrows + FAST_R - 1) / FAST_R;
    if (blocks == 0) return cudaSuccess;
    k_step_prep_fast<<<(unsigned)blocks, FAST_T, 0, s>>>(sp, c->d, c->dpad, c->qjl_m, c->PiT, c->ST);
    return cudaGetLastError();
  }
  const int64_t blocks = 2 * sp.nkv + (sp.qrows + 1) / 2;
  if (blocks == 0) return cudaSuccess;
  k_step_prep<<<(unsigned)blocks, c->dpad, (2 + 2 * MV_KC) * c->dpad * sizeof(float), s>>>(
      sp, c->d, c->dpad, c->qjl_m, c->PiT, c->ST);
  return cudaGetLastError();
}

cudaError_t launch_prerotate(const tq_ctx* c, const void* q, int dtype, int64_t rows, const AttnArgs* plan,
                             float* qr, float* qs, cudaStream_t s, const QopPlan* qop) {
  if (rows == 0) return cudaSuccess;
  const int32_t* sl = plan ? plan->seq_lens : nullptr;
  const int pB = plan ? plan->B : 0, pH = plan ? plan->Hkv : 1;
  const int64_t pT = plan ? plan->max_T : 0;
  int64_t* tl = plan ? plan->tiles : nullptr;
  QopPlan qp{};
  if (qop) qp = *qop;
  if (c->dpad <= 128) {
    k_prerotate_fast<<<(unsigned)((rows + FAST_R - 1) / FAST_R), FAST_T, 0, s>>>(
        q, dtype, rows, c->d, c->dpad, c->qjl_m, c->PiT, c->ST, qr, qs, sl, pB, pH, pT, tl, qp);
  } else if (rows <= 1024) {
    k_prerotate<2><<<(unsigned)((rows + 1) / 2), c->dpad, (2 + 2 * MV_KC) * c->dpad * sizeof(float), s>>>(
        q, dtype, rows, c->d, c->dpad, c->qjl_m, c->PiT, c->ST, qr, qs, sl, pB, pH, pT, tl, qp);
  } else {
    k_prerotate<8><<<(unsigned)((rows + 7) / 8), c->dpad, (8 + 2 * MV_KC) * c->dpad * sizeof(float), s>>>(
        q, dtype, rows, c->d, c->dpad, c->qjl_m, c->PiT, c->ST, qr, qs, sl, pB, pH, pT, tl, qp);
  }
  return cudaGetLastError();
}

int attn_splits(const tq_ctx* c, int B, int Hkv, int64_t max_T, int* chunk) {
  (void)c;
  // Aim for about 8 CTAs per SM over the 148 SMs, tiles of whole 128 tokens.
  const int64_t pairs = (int64_t)B * Hkv;
  const int64_t target = 148 * 8;
  int64_t splits = (target + pairs - 1) / pairs;
  int64_t ch = (max_T + splits - 1) / splits;
  ch = ((ch + AT - 1) / AT) * AT;
  if (ch < AT) ch = AT;
  splits = (max_T + ch - 1) / ch;
  if (splits < 1) splits = 1;
  *chunk = (int)ch;
  return (int)splits;
}

// Shared memory limit of the fast merge.
constexpr size_t kMergeFastSmem = 200 * 1024;

cudaError_t launch_attn_merge(const tq_ctx* c, const AttnArgs& a, float* out, cudaStream_t s) {
  const int slots = a.tiles ? a.nw * a.wpu : a.splits;
  const int G = a.Hq / a.Hkv, Gp = (G + 3) & ~3;
  const size_t fsm = ((size_t)Gp * 128 + 4 * 4 * 128 + (size_t)G * slots) * sizeof(float);
  if (c->dpad <= 128 && fsm <= kMergeFastSmem) {
    k_attn_merge_fast<<<(unsigned)((int64_t)a.B * a.Hkv), FAST_T, fsm, s>>>(
        a.part, a.splits, c->d, c->dpad, c->Pi_f, out, a.tiles, a.B, a.Hq, a.Hkv, a.nw, a.wpu, slots);
    return cudaGetLastError();
  }
  k_attn_merge<<<(unsigned)(a.B * a.Hq), 128, (c->dpad + slots) * sizeof(float), s>>>(
      a.part, a.splits, c->d, c->dpad, c->Pi_f, out, a.tiles, a.B, a.Hq, a.Hkv, a.nw, a.wpu);
  return cudaGetLastError();
}

cudaError_t launch_attn(const tq_ctx* c, const AttnArgs& a, float* out, cudaStream_t s) {
  TQ_DISPATCH_J(c->J, return attn_J<JV>(c, a, out, s));
}

cudaError_t launch_logits(const tq_ctx* c, const void* q, int dtype, int64_t nq,
                          const uint32_t* kcodes, const uint32_t* kqjl, const float* knorm,
                          const float* krnorm, int64_t nk, float* out, cudaStream_t s) {
  if (nq == 0 || nk == 0) return cudaSuccess;
  dim3 grid((unsigned)((nk + 127) / 128), (unsigned)((nq + LQB - 1) / LQB));
  const float cq = c->qjl_m > 0 ? (float)(std::sqrt(M_PI / 2.0) / c->qjl_m) : 0.f;
  TQ_DISPATCH_J(c->J, k_logits<JV><<<grid, 128, 0, s>>>(q, dtype, nq, c->d, c->bk_lm, c->wk, c->qjl_m,
                                                        c->PiT, c->ST, c->ck_f, cq, kcodes, kqjl,
                                                        knorm, krnorm, nk, c->norm_f16 ? 1 : 0, out);
                return cudaGetLastError());
}

cudaError_t launch_dequant(const tq_ctx* c, int which, const uint32_t* codes,
                           const uint32_t* qjl, const float* norm, const float* rnorm,
                           int64_t n, float* out, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const bool key = which == TQ_KEY;
  const int m = key ? c->qjl_m : 0;
  const float cq = m > 0 ? (float)(std::sqrt(M_PI / 2.0) / m) : 0.f;
  k_dequant<<<(unsigned)n, 128, c->dpad * sizeof(float), s>>>(
      c->d, c->dpad, key ? c->bk_lm : c->bits_v, key ? c->wk : c->wv, m, c->Pi_f, c->S_f,
      key ? c->ck_f : c->cv_f, cq,
      codes, qjl, norm, rnorm, c->norm_f16 ? 1 : 0, out);
  return cudaGetLastError();
}

// Two passes when the database is large: the k-th best of the first
// kTopkSample vectors sets every list's starting bar, so the full pass
// inserts almost nothing.
constexpr int64_t kTopkSample = 32768;

static size_t up256(size_t b) { return (b + 255) & ~(size_t)255; }

// The plans of both passes: the tcgen05 scorer when it fits, else mma.sync.
static void topk_plans(const tq_ctx* c, int64_t nq, int64_t n, int k, TopkPlan& p, TopkPlan& ps) {
  p = topk_tc_plan(c, nq, n > 0 ? n : 1, k, 0);
  if (p.use_tc) {
    ps = topk_tc_plan(c, nq, n > 0 ? n : 1, k, kTopkSample);
  } else {
    p = topk_mma_plan(c, nq, n > 0 ? n : 1, k);
    ps = topk_mma_sample_plan(p, kTopkSample, c->sms);
  }
}

size_t topk_workspace(const tq_ctx* c, int64_t nq, int64_t n, int k) {
  TopkPlan p, ps;
  topk_plans(c, nq, n, k, p, ps);
  size_t b = 2 * up256((size_t)nq * c->dpad * sizeof(float));                 // q', s
  b += up256(p.qh_bytes) + up256(p.qsc_bytes) + up256(p.rows_bytes);
  b += 2 * up256((size_t)nq * p.nlists * k * sizeof(float));                  // candidates
  b += 2 * up256((size_t)nq * ps.nlists * k * sizeof(float));                 // sample candidates
  b += 2 * up256((size_t)nq * k * sizeof(float));                             // bars
  return b + 1024;
}

cudaError_t launch_topk(const tq_ctx* c, const void* q, int dtype, int64_t nq,
                        const uint32_t* codes, const uint32_t* qjl, const float* norm,
                        const float* rnorm, int64_t n, int k, int32_t* idx, float* score,
                        void* ws, cudaStream_t s) {
  if (nq == 0) return cudaSuccess;
  TopkPlan pl, ps;
  topk_plans(c, nq, n, k, pl, ps);
  auto score_pass = pl.use_tc ? launch_topk_tc : launch_topk_mma;
  char* p = static_cast<char*>(ws);
  auto take = [&](size_t bytes) {
    char* r = p;
    p += up256(bytes);
    return r;
  };
  float* qr = reinterpret_cast<float*>(take((size_t)nq * c->dpad * sizeof(float)));
  float* qs = reinterpret_cast<float*>(take((size_t)nq * c->dpad * sizeof(float)));
  void* qh = take(pl.qh_bytes);
  float* qsc = reinterpret_cast<float*>(take(pl.qsc_bytes));
  void* rows = take(pl.rows_bytes);
  float* cv = reinterpret_cast<float*>(take((size_t)nq * pl.nlists * k * sizeof(float)));
  int* ci = reinterpret_cast<int*>(take((size_t)nq * pl.nlists * k * sizeof(int)));
  float* scv = reinterpret_cast<float*>(take((size_t)nq * ps.nlists * k * sizeof(float)));
  int* sci = reinterpret_cast<int*>(take((size_t)nq * ps.nlists * k * sizeof(int)));
  float* barv = reinterpret_cast<float*>(take((size_t)nq * k * sizeof(float)));
  int32_t* bari = reinterpret_cast<int32_t*>(take((size_t)nq * k * sizeof(int32_t)));
  if (n == 0) {   // nothing to score: every slot is (-1, -inf)
    k_topk_final<<<(unsigned)nq, 32, 0, s>>>(cv, ci, 0, k, idx, score);
    return cudaGetLastError();
  }
  cudaError_t e = launch_prerotate(c, q, dtype, nq, nullptr, qr, qs, s);
  if (e != cudaSuccess) return e;
  if ((e = launch_topk_qprep(c, pl, qr, qs, nq, qh, qsc, s)) != cudaSuccess) return e;
  if ((e = launch_topk_dequant(c, pl, codes, qjl, n, rows, s)) != cudaSuccess) return e;
  const bool two_pass = n >= 4 * kTopkSample;
  if (two_pass) {
    e = score_pass(c, ps, qh, qsc, nq, rows, norm, rnorm, kTopkSample, k, nullptr, nullptr, scv, sci, s);
    if (e != cudaSuccess) return e;
    k_topk_final<<<(unsigned)nq, 32, 0, s>>>(scv, sci, ps.nlists, k, bari, barv);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  e = score_pass(c, pl, qh, qsc, nq, rows, norm, rnorm, n, k, two_pass ? barv : nullptr,
                      two_pass ? bari : nullptr, cv, ci, s);
  if (e != cudaSuccess) return e;
  k_topk_final<<<(unsigned)nq, 32, 0, s>>>(cv, ci, pl.nlists, k, idx, score);
  return cudaGetLastError();
}

// Raise the dynamic shared-memory limit of every kernel that needs more
// than the default 48 KB, on the current device (called by tq_init).
template <int J>
static cudaError_t configure_J() {
  cudaError_t e = cudaFuncSetAttribute(k_quantize<J>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)(QWARPS * J * 32 * quant_qv<J>() * sizeof(float)));
  if (e != cudaSuccess) return e;
  const int attn_max = (2 * GMAX * J * 32 + AT * GMAX) * (int)sizeof(float) + AT * 64 * (int)sizeof(uint32_t);
  e = cudaFuncSetAttribute(k_attn_split<J>, cudaFuncAttributeMaxDynamicSharedMemorySize, attn_max);
  return e;
}

cudaError_t configure_kernels() {
  cudaError_t e;
  if ((e = configure_J<1>()) != cudaSuccess) return e;
  if ((e = configure_J<2>()) != cudaSuccess) return e;
  if ((e = configure_J<3>()) != cudaSuccess) return e;
  if ((e = configure_J<4>()) != cudaSuccess) return e;
  if ((e = configure_J<5>()) != cudaSuccess) return e;
  if ((e = configure_J<6>()) != cudaSuccess) return e;
  if ((e = configure_J<7>()) != cudaSuccess) return e;
  if ((e = configure_J<8>()) != cudaSuccess) return e;
  // Row-batched small kernels: up to (8 + 2 * MV_KC) rows of dpad = 256 floats.
  const int small_smem = (8 + 2 * MV_KC) * 256 * (int)sizeof(float);
  const cudaFuncAttribute ms = cudaFuncAttributeMaxDynamicSharedMemorySize;
  if ((e = cudaFuncSetAttribute(k_quantize_small<1>, ms, small_smem))) return e;
  if ((e = cudaFuncSetAttribute(k_quantize_small<8>, ms, small_smem))) return e;
  if ((e = cudaFuncSetAttribute(k_prerotate<2>, ms, small_smem))) return e;
  if ((e = cudaFuncSetAttribute(k_prerotate<8>, ms, small_smem))) return e;
  if ((e = cudaFuncSetAttribute(k_step_prep, ms, small_smem))) return e;
  if ((e = cudaFuncSetAttribute(k_attn_merge_fast, ms, (int)kMergeFastSmem))) return e;
  if ((e = configure_quant_tc()) != cudaSuccess) return e;
  if ((e = configure_attn_lut()) != cudaSuccess) return e;
  if ((e = configure_attn_i8()) != cudaSuccess) return e;
  if ((e = configure_topk_mma()) != cudaSuccess) return e;
  if ((e = configure_topk_tc()) != cudaSuccess) return e;
  return configure_attn_mma();
}

}  // namespace tqk
