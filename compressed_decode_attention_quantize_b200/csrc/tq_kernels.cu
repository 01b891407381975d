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
// Quantize: one warp quantizes QV vectors at a time.  Lane l owns the output
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

constexpr int QV = 8;
constexpr int QWARPS = 8;

template <int J>
__global__ void __launch_bounds__(QWARPS * 32) k_quantize(QuantArgs a) {
  constexpr int DP = J * 32;
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
      const float4 x0 = *reinterpret_cast<const float4*>(sx + k * QV);
      const float4 x1 = *reinterpret_cast<const float4*>(sx + k * QV + 4);
      const float xv[QV] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
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
      const float4 x0 = *reinterpret_cast<const float4*>(sx + k * QV);
      const float4 x1 = *reinterpret_cast<const float4*>(sx + k * QV + 4);
      const float xv[QV] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
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
  __shared__ int64_t s_w[8];
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
  const double c0 = P.c0, w0 = (double)P.c1 - c0, w1 = (double)P.c2 - c0;
  const double wmax = fmax(fabs(w0), fabs(w1));
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
    // 2^e <= max |w q'| < 2^(e+1), S = 29 - e: |Q| < 2^30 at p = 0.
    const double mk = wmax * mq;
    const int S = mk > 0.0 ? 29 - ilogb(mk) : 0;
    const int S2 = ms > 0.f ? 29 - ilogb((double)ms) : 0;
    const int64_t row = row0 + r;
    const int64_t b = row / P.Hq;
    const int h = (int)(row % P.Hq), kvh = h / P.G, hg = h % P.G;
    unsigned char* img = P.img + (b * (P.Hq / P.G) + kvh) * (int64_t)kQopBytes;
    auto put = [&](int reg, int tt, int e, int64_t Q) {
      // four balanced digits, digit l to column 2 hg + l % 2 of N tile l / 2
#pragma unroll
      for (int l = 0; l < 4; ++l) {
        const int dg = (int)(signed char)(Q & 0xFF);
        Q = (Q - dg) >> 8;
        const int rr = reg + 2 * (l >> 1);
        const int ln = 4 * (2 * hg + (l & 1)) + tt;
        img[(((rr >> 2) * 32 + ln) * 4 + (rr & 3)) * 4 + e] = (unsigned char)(dg & 0xFF);
      }
    };
    {
      const double q = qv[r];
#pragma unroll
      for (int pl = 0; pl < 2; ++pl) {
        const int bit = 2 * (j & 15) + pl, w = j >> 4, p = bit & 7;
        const int64_t Q = llrint(ldexp((pl ? w1 : w0) * q, S - p));
        put(4 * p + (w >> 2), w & 3, bit >> 3, Q);
      }
      const int bit = j & 31, p = bit & 7;
      const int64_t Q = llrint(ldexp((double)sv[r], S2 - p));
      put(32 + 4 * (p >> 1) + (p & 1), j >> 5, bit >> 3, Q);
    }
    if (j == 0) {
      const double sl = P.scale_log2;
      float4 cst;
      cst.x = (float)ldexp(sl, -S);
      cst.y = (float)(c0 * sq * sl);
      cst.z = (float)ldexp(2.0 * (double)P.cq * sl, -S2);
      cst.w = (float)(-ss * (double)P.cq * sl);
      reinterpret_cast<float4*>(img + kQopRegs * 32 * 4)[hg] = cst;
    }
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
  // (one read of Pi and S for all eight) beyond.
  if (a.n <= 1024) {
    k_quantize_small<1><<<(unsigned)a.n, c->dpad, (1 + 2 * MV_KC) * c->dpad * sizeof(float), s>>>(a, c->dpad);
  } else {
    k_quantize_small<8><<<(unsigned)((a.n + 7) / 8), c->dpad, (8 + 2 * MV_KC) * c->dpad * sizeof(float), s>>>(
        a, c->dpad);
  }
  return cudaGetLastError();
}

cudaError_t launch_step_prep(const tq_ctx* c, const StepPrep& sp, cudaStream_t s) {
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
  if (rows <= 1024) {
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

cudaError_t launch_attn_merge(const tq_ctx* c, const AttnArgs& a, float* out, cudaStream_t s) {
  const int slots = a.tiles ? a.nw * a.wpu : a.splits;
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
                                       (int)(QWARPS * J * 32 * QV * sizeof(float)));
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
  if ((e = configure_quant_tc()) != cudaSuccess) return e;
  if ((e = configure_attn_lut()) != cudaSuccess) return e;
  if ((e = configure_attn_i8()) != cudaSuccess) return e;
  if ((e = configure_topk_mma()) != cudaSuccess) return e;
  if ((e = configure_topk_tc()) != cudaSuccess) return e;
  return configure_attn_mma();
}

}  // namespace tqk
