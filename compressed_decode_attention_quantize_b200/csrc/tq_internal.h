// Internal declarations shared by the host table builder, the kernels and the
// C ABI of libtq.
#pragma once

#include <cstdint>
#include <string>
#include <vector>

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "tq.h"

struct tq_ctx {
  int d = 0;        // vector dimension
  int J = 0;        // words per bit-plane, ceil(d/32)
  int dpad = 0;     // 32*J
  int bits_k = 0;   // key bits including the QJL bit
  int bk_lm = 0;    // key Lloyd-Max bits
  int bits_v = 0;   // value Lloyd-Max bits
  int qjl_m = 0;    // QJL rows (0 = none)
  int wk = 0;       // code words per key vector
  int wv = 0;       // code words per value vector
  int device = 0;
  uint64_t seed = 0;
  // fp64 host tables
  std::vector<double> Pi, S, ck, bk, cv, bv;
  // device tables (one allocation owned by the context)
  void* dev_block = nullptr;
  const float* PiT = nullptr;   // [d][dpad]  PiT[k*dpad+j] = Pi[j][k]; zero for j >= d
  const float* Pi_f = nullptr;  // [d][d]     row-major Pi
  const float* ST = nullptr;    // [d][dpad]  ST[k*dpad+i] = S[i][k]; zero for i >= m
  const float* S_f = nullptr;   // [dpad][d]  row-major S; zero rows for i >= m
  const float* ck_f = nullptr;  // [256] key centroids (padded)
  const float* bk_f = nullptr;  // [256] key boundaries (padded with +inf)
  const float* cv_f = nullptr;  // [256]
  const float* bv_f = nullptr;  // [256]
  // Tensor-core quantize (d = 128): swizzled fp16 operand images and QJL row norms.
  bool tc_ok = false;
  void* tc_block = nullptr;
  int sms = 148;
  bool nc_k = false;   // norm correction of keys (MSE-only keys)
  bool nc_v = false;   // norm correction of values
  bool norm_f16 = false;   // norms stored as binary16 (MSE-only keys)
  const void* tc_pih = nullptr;   // 2^8 Pi, fp16 head
  const void* tc_pil = nullptr;   // 2^8 Pi - head, fp16
  const void* tc_s = nullptr;     // S, fp16 (exact)
  const float* tc_snorm = nullptr;  // |S_i|
  const void* tc_pib = nullptr;   // 2^8 Pi as three bf16 terms (head, middle, tail), 3 x 32 KB
  // Polls before a tensor-core kernel's main bounded wait gives up (0 = the
  // kernels' full limit); set only by tq_set_wait_limit, for testing the
  // fault path.
  int wait_limit = 0;
};

namespace tqh {
double round_to_half(double x);
void rotation(int d, uint64_t seed, std::vector<double>& Pi);
void qjl_matrix(int m, int d, uint64_t seed, std::vector<double>& S);
void lloyd_max(int d, int bits, std::vector<double>& cen, std::vector<double>& bnd);
}  // namespace tqh

// Code words per vector for d coordinates of b-bit indices (field layout).
inline int tq_code_words(int d, int b) {
  if (b == 3) return (d + 15) / 16 + (d + 31) / 32;
  const int per = 32 / b;
  return (d + per - 1) / per;
}

namespace tqk {

// Codebook sizes up to 2^8 levels (Lloyd-Max bits 1..4 and 8).
constexpr int kMaxLevels = 256;

// Per-vector norms are fp32, or binary16 when the context stores them so.
__device__ __forceinline__ float load_norm(const float* p, int64_t i, int f16) {
  return f16 ? __half2float(reinterpret_cast<const __half*>(p)[i]) : p[i];
}
__device__ __forceinline__ void store_norm(float* p, int64_t i, float v, int f16) {
  if (f16)
    reinterpret_cast<__half*>(p)[i] = __float2half_rn(v);
  else
    p[i] = v;
}

struct QuantArgs {
  const void* x;
  int dtype;
  int64_t n, ld;
  int d, bits, nbnd, m, words;
  const float* PiT;
  const float* ST;
  const float* cen;
  const float* bnd;
  uint32_t* codes;
  uint32_t* qjl;
  float* norm;
  float* rnorm;
  // Optional cache placement: when pos != nullptr, input row v = b*H + g is
  // written to cache record (b*H + g)*max_T + pos[b]; otherwise to record v.
  // With block_table != nullptr the cache is paged: record
  // (block_table[b][pos / block_size] * H + g) * block_size + pos % block_size,
  // max_T = max_blocks * block_size; an invalid pos or block id writes nothing.
  const int32_t* pos;
  int H;
  int64_t max_T;
  const int32_t* block_table;
  int max_blocks, block_size;
  int64_t num_blocks;
  // Norm correction (MSE-only vectors): store n / |c[idx]| instead of n.
  int nc;
  // Norms stored as binary16 (the norm pointer then addresses __half values).
  int nf16;
};

// Query operands of the int8 key product (decode with 2-bit keys + QJL,
// d = m = 128, groups of at most four query heads).  Per (sequence, kv head)
// one image of kQopBytes: 48 registers per lane in lane order
// ([12][32 lanes][4] uint32), each four signed bytes, then four float4 of
// per-head logit constants.  Register r = (k-step s, N tile j, half hb):
// keys r = 4 s + 2 j + hb (s < 8), QJL r = 32 + 4 s + 2 j + hb (s < 4).
// Column n of an N tile is head n / 2, limb 2 j + n % 2 of that head's
// balanced base-256 digits.
constexpr int kQopRegs = 48;
constexpr int kQopBytes = kQopRegs * 32 * 4 + 4 * 16;
struct QopPlan {
  unsigned char* img;  // [B * Hkv][kQopBytes]; null = no image
  int Hq, G;           // query heads, heads per kv group (<= 4)
  float scale_log2;    // softmax scale * log2(e)
  float cq;            // sqrt(pi/2) / m
  float c0, c1, c2;    // 2-bit key centroids 0..2
};

struct AttnArgs {
  const float* qr;   // [B*Hq][dpad] pre-rotated queries
  const float* qs;   // [B*Hq][dpad] S q'
  int B, Hq, Hkv, G, d, bk, bv, m, wk, wv;
  const uint32_t* kcodes;
  const uint32_t* kqjl;
  const float* knorm;
  const float* krnorm;
  const uint32_t* vcodes;
  const float* vnorm;
  int64_t max_T;
  const int32_t* seq_lens;
  float scale_log2;  // softmax scale * log2(e)
  float cq;          // sqrt(pi/2)/m
  const float* ck;
  const float* cv;
  int splits;
  int chunk;         // tokens per split
  float* part;       // [B*Hq][splits][dpad+2], or [slots][G][dpad+2] on the segment path
  // Segment path (tensor-core decode, group <= 4): 16-token tile prefix over
  // sequences, tiles[b] = Hkv * sum_{b' < b} ceil(len_b' / 16), written by the
  // pre-rotation kernel; null on the split path.  nw = owners of tile ranges
  // (warps, or CTAs for group 8), wpu = partial writers per owner.
  int64_t* tiles;
  int nw;
  int wpu;
  // Paged caches (tensor-core paths): block_table [B][max_blocks] of block ids
  // in [0, num_blocks); arrays are [num_blocks][Hkv][block_size][...] and
  // block_size is a multiple of 16.  Null for the contiguous [B][Hkv][max_T].
  const int32_t* block_table;
  int max_blocks, block_size;
  int64_t num_blocks;
  // Norms stored as binary16 (knorm / vnorm then address __half values).
  int nf16;
  // Query-operand images of the int8 key product (see QopPlan).
  const unsigned char* qimg;
};

struct QuantTcArgs {
  const void* x;
  int dtype;
  int64_t n, ld;
  int bits, m;
  const void* pi_hi;
  const void* pi_lo;
  const void* pi_b;    // three bf16 terms of 2^8 Pi (bf16 inputs)
  const void* s_img;
  const float* snorm;
  const float* s_f32;
  uint32_t* codes;
  uint32_t* qjl;
  float* norm;      // binary16 [n] when nf16
  float* rnorm;
  const int32_t* pos;
  int H;
  int64_t max_T;
  float cen[16];
  float bnd[16];
  const float* bnd_dev;   // device fp32 thresholds [2^bits - 1] (8-bit codes)
  int wait_limit;   // polls of the main MMA waits (the full limit when 0)
  int nc;           // norm correction: store n / |c[idx]| (MSE-only formats)
  int nf16;         // binary16 norms (MSE-only formats)
};

cudaError_t launch_quantize(const tq_ctx* c, const QuantArgs& a, cudaStream_t s);
// One block per vector, for small batches (n <= kSmallQuantize).
constexpr int64_t kSmallQuantize = 4096;
cudaError_t launch_quantize_small(const tq_ctx* c, const QuantArgs& a, cudaStream_t s);
// Tensor-core quantize for d = 128 (16-bit inputs).  Norm-corrected and
// binary16-norm formats run on the warp-specialised kernel only
// (quant_ws_eligible); launch_quant_tc returns cudaErrorNotSupported for them
// when the input cannot take that form.
bool quant_ws_eligible(const QuantTcArgs& a);
cudaError_t launch_quant_tc(const QuantTcArgs& a, int sms, cudaStream_t s);
cudaError_t configure_quant_tc();
cudaError_t read_and_clear_fault(int* value);
// One launch before a fused decode step: append the new K and V vectors (one
// per (sequence, kv head)), pre-rotate the queries, write the attention
// lengths (and the tile prefix when tiles != null).
struct StepPrep {
  QuantArgs k, v;
  const void* q;
  int qdtype;
  int64_t qrows;
  float* qr;
  float* qs;
  const int32_t* pos;
  int32_t* lens;
  int B, Hkv;
  int64_t max_T;
  int64_t* tiles;
  int64_t nkv;
  QopPlan qop;
};
cudaError_t launch_step_prep(const tq_ctx* c, const StepPrep& sp, cudaStream_t s);
// With plan != null the kernel also writes plan->tiles (the segment path's
// tile prefix) from plan->seq_lens, B, Hkv and max_T; with qop != null and
// qop->img != null it writes the int8 query-operand images.
cudaError_t launch_prerotate(const tq_ctx* c, const void* q, int dtype, int64_t rows, const AttnArgs* plan,
                             float* qr, float* qs, cudaStream_t s, const QopPlan* qop = nullptr);
// The int8 key-product decode (2-bit keys + QJL, m = 128, 4-bit values,
// d = 128, group 1, 2 or 4): whether it applies, and the plan of its
// query-operand images.
bool attn_i8_supported(const tq_ctx* c, const AttnArgs& a);
QopPlan attn_i8_qop(const tq_ctx* c, const AttnArgs& a, unsigned char* img);
// Needs AttnArgs::tiles (the tile prefix) and AttnArgs::qimg (the images).
cudaError_t launch_attn_i8(const tq_ctx* c, const AttnArgs& a, float* out, cudaStream_t s);
cudaError_t configure_attn_i8();
cudaError_t launch_attn(const tq_ctx* c, const AttnArgs& a, float* out, cudaStream_t s);
cudaError_t launch_attn_merge(const tq_ctx* c, const AttnArgs& a, float* out, cudaStream_t s);
// Tensor-core decode path with fp16 bit operands (d = 128, k3 with m = 128,
// v4, group 8); it needs AttnArgs::tiles (the tile prefix) set.
bool attn_mma_supported(const tq_ctx* c, const AttnArgs& a);
// Upper bound on the warps of a segment-path launch (sizes the partials).
int64_t attn_seg_max_warps(const tq_ctx* c);
cudaError_t launch_attn_mma(const tq_ctx* c, const AttnArgs& a, float* out, cudaStream_t s);
// Tensor-core decode path with table-dequantized keys (d = 128, values 4
// bits, group 4 or 8): 3-bit Lloyd-Max keys + QJL with m = 128 (k4v4), or
// MSE-only 3- or 4-bit keys (the norm-corrected formats); needs AttnArgs::tiles.
bool attn_lut_supported(const tq_ctx* c, const AttnArgs& a);
cudaError_t launch_attn_lut(const tq_ctx* c, const AttnArgs& a, float* out, cudaStream_t s);
cudaError_t configure_attn_lut();
// Top-k on the tensor cores: query blocks of 64 or 128 x database chunks.
struct TopkPlan {
  int KL, KQ;            // padded centroid and sign widths
  int qb;                // queries per CTA (64 or 128)
  int64_t chunks, chunk; // database chunks, vectors per chunk
  int64_t qblocks;       // query blocks; work items = qblocks x chunks
  int nlists;            // candidate lists per query (chunks x 2 row groups)
  size_t qh_bytes, qsc_bytes, cand_bytes, rows_bytes, smem;
  int nkb = 0, stages = 0;   // tensor-core scorer: K blocks of 64, shared-memory stages
  bool use_tc = false;       // the tcgen05 scorer fits (else the mma.sync one)
};
TopkPlan topk_mma_plan(const tq_ctx* c, int64_t nq, int64_t n, int k);
// The same queries over the first n_sample database vectors (the bar pass).
TopkPlan topk_mma_sample_plan(const TopkPlan& full, int64_t n_sample, int sms);
cudaError_t launch_topk_qprep(const tq_ctx* c, const TopkPlan& p, const float* qr, const float* qs,
                              int64_t nq, void* qh, float* qsc, cudaStream_t s);
// Dequantized database rows [n][KL + KQ] in fp16 (centroids | signs).
cudaError_t launch_topk_dequant(const tq_ctx* c, const TopkPlan& p, const uint32_t* codes, const uint32_t* qjl,
                                int64_t n, void* rows, cudaStream_t s);
cudaError_t launch_topk_mma(const tq_ctx* c, const TopkPlan& p, const void* qh, const float* qsc, int64_t nq,
                            const void* rows, const float* norm, const float* rnorm, int64_t n, int k,
                            const float* bar_v, const int* bar_i, float* cand_v, int* cand_i, cudaStream_t s);
cudaError_t configure_topk_mma();
// The tcgen05 scorer (128 queries per item, TMA-fed, TMEM accumulators).
// n_sample > 0 plans the bar pass over the first n_sample vectors.
TopkPlan topk_tc_plan(const tq_ctx* c, int64_t nq, int64_t n, int k, int64_t n_sample);
cudaError_t launch_topk_tc(const tq_ctx* c, const TopkPlan& p, const void* qh, const float* qsc, int64_t nq,
                           const void* rows, const float* norm, const float* rnorm, int64_t n, int k,
                           const float* bar_v, const int* bar_i, float* cand_v, int* cand_i, cudaStream_t s);
cudaError_t configure_topk_tc();
cudaError_t read_and_clear_topk_fault(int* value);
cudaError_t launch_logits(const tq_ctx* c, const void* q, int dtype, int64_t nq,
                          const uint32_t* kcodes, const uint32_t* kqjl, const float* knorm,
                          const float* krnorm, int64_t nk, float* out, cudaStream_t s);
cudaError_t launch_dequant(const tq_ctx* c, int which, const uint32_t* codes,
                           const uint32_t* qjl, const float* norm, const float* rnorm,
                           int64_t n, float* out, cudaStream_t s);
size_t topk_workspace(const tq_ctx* c, int64_t nq, int64_t n, int k);
cudaError_t launch_topk(const tq_ctx* c, const void* q, int dtype, int64_t nq,
                        const uint32_t* codes, const uint32_t* qjl, const float* norm,
                        const float* rnorm, int64_t n, int k, int32_t* idx, float* score,
                        void* ws, cudaStream_t s);
int attn_splits(const tq_ctx* c, int B, int Hkv, int64_t max_T, int* chunk);
// Shared-memory limits of all kernels on the current device (tq_init).
cudaError_t configure_kernels();
cudaError_t configure_attn_mma();

}  // namespace tqk
