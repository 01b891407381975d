/*
 * tq.h - C ABI of libtq: TurboQuant-style online K/V quantization and decode
 * attention computed from the packed codes, for one NVIDIA B200 (sm_100a).
 *
 * Method sources (web pages, by title and section):
 *   [WHAT] a2a-mcp.org, "什么是TurboQuant？谷歌突破性AI压缩技术实现6倍KV缓存缩减和8倍推理加速"
 *          ("What is TurboQuant?"), section "TurboQuant 工作原理：技术深度解析"
 *          ("How TurboQuant works") stage 1 (random orthogonal rotation from
 *          the QR of a Gaussian matrix; Beta((d-1)/2,(d-1)/2) law of rotated
 *          coordinates; normalisation; Lloyd-Max quantizer for that law),
 *          stage 2 (1-bit QJL sign sketch of the residual), closing paragraph
 *          (attention logits straight from compressed indices); section
 *          "如何实现 TurboQuant：分步指南" ("How to implement") part 1 (codebook per
 *          dimension and bit width; the fused kernel pre-rotates the query once
 *          and takes dot products from the indices); section "基准测试与实际性能表现"
 *          ("Benchmarks") (inner-product top-k on d=200 vectors).
 *   [VLLM] papercache.org, "A First Comprehensive Study of TurboQuant: Accuracy
 *          and Performance", sections A2-A3 (values are dequantized for the
 *          attention; variant naming k3v4 = 3-bit keys, 4-bit values).
 *
 * Conventions shared by every call
 * --------------------------------
 * - Pointers marked "device" are CUDA device pointers on the context's device,
 *   allocated and owned by the caller; the library never frees or keeps them.
 *   `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 * - Compute calls (quantize, dequantize, logits, attention, decode step,
 *   top-k) launch on the current device, which must be the context's device
 *   (the one current at tq_init); otherwise they return TQ_ERR_ARG before any
 *   launch.
 * - Norm arrays are 4-byte aligned fp32, or 2-byte aligned binary16 under
 *   TQ_NORM_F16; code and QJL arrays are 4-byte aligned.
 * - Compute calls only enqueue kernels on `stream`: they neither allocate,
 *   synchronise, nor fall back to the CPU.  Scratch memory comes from the
 *   caller's `workspace` (device, at least the size the *_workspace_bytes
 *   query returns, 256-byte aligned).
 * - Every call but tq_init/tq_init_ex/tq_destroy/tq_last_error returns a status:
 *   TQ_OK, TQ_ERR_ARG (bad pointer, size, alignment or enum),
 *   TQ_ERR_UNSUPPORTED (valid but not implemented: dimension, bit width),
 *   TQ_ERR_CUDA (a CUDA launch or runtime error), TQ_ERR_WORKSPACE (workspace
 *   missing or too small).  tq_last_error() then returns a message (per
 *   thread; valid until the next call on that thread).
 * - Sizes: 8 <= d <= 256 with d % 8 == 0; Lloyd-Max bits 1..4 or 8 (8-bit
 *   codes serve the k8v4 format; tq_topk takes 1..4);
 *   0 <= qjl_m <= 32*ceil(d/32), qjl_m % 8 == 0.
 *
 * Packed layout of one vector
 * ---------------------------
 *   codes  uint32[W]   Lloyd-Max indices as b-bit fields, LSB first, 32/b
 *                      fields per word, for b in {1, 2, 4, 8}: coordinate j sits
 *                      in word j/(32/b) at bit b*(j%(32/b)); W = ceil(d*b/32).
 *                      For b = 3 the low two bits of every index form a 2-bit
 *                      field stream (ceil(d/16) words) followed by a 1-bit
 *                      stream of the top bits (ceil(d/32) words).  Padding
 *                      bits are 0.
 *   qjl    uint32[ceil(m/32)]  keys only: bit i%32 of word i/32 is 1 when
 *                      (S r)_i >= 0.
 *   norm   float       |x| (fp32); |x| / |c[idx]| under norm correction
 *                      (see tq_init_ex); binary16 under TQ_NORM_F16 (the
 *                      norm pointers of the calls are void* for this).
 *   rnorm  float       keys with QJL only: gamma = |x| * |r|, r the residual
 *                      of the rotated unit vector.
 * Arrays of vectors are these records laid out as separate dense arrays
 * (codes [N][W], qjl [N][ceil(m/32)], norm [N], rnorm [N]).  A KV cache is
 * [B][Hkv][max_T] records in each array.  tq_layout reports W.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum tq_status {
  TQ_OK = 0,
  TQ_ERR_ARG = 1,
  TQ_ERR_UNSUPPORTED = 2,
  TQ_ERR_CUDA = 3,
  TQ_ERR_WORKSPACE = 4
};

enum tq_which { TQ_KEY = 0, TQ_VALUE = 1 };
enum tq_dtype { TQ_F32 = 0, TQ_BF16 = 1, TQ_F16 = 2 };

typedef struct tq_ctx tq_ctx;

typedef struct tq_layout_t {
  int32_t d;              /* head / vector dimension                        */
  int32_t bits;           /* Lloyd-Max bits per coordinate                    */
  int32_t words;          /* W, code words per vector                         */
  int32_t qjl_m;          /* QJL rows (0 for values or when disabled)        */
  int32_t qjl_words;      /* ceil(qjl_m/32)                                  */
  int32_t has_rnorm;      /* 1 when an rnorm (gamma) array is produced       */
  int64_t bytes_per_vector; /* codes + qjl + norm (+ rnorm) bytes            */
  int32_t norm_bytes;     /* 4 (fp32 norms) or 2 (fp16, TQ_NORM_F16)         */
} tq_layout_t;

/* Message for the last failed call on this thread ("" if none). */
const char* tq_last_error(void);

/* Library version string. */
const char* tq_version(void);

/*
 * tq_device_fault - synchronising diagnostic: reads and clears the device
 * fault code that kernels set when a bounded wait on the tensor cores gives
 * up: 0 = none, bit 0 = quantize, bit 1 = top-k scorer.  The kernel that set
 * it has released its resources and returned; its outputs for the affected
 * tiles are undefined.
 */
int tq_device_fault(int* code);

/*
 * tq_set_wait_limit - diagnostic for testing the fault path: the tensor-core
 * quantize and top-k kernels launched with context c after this call give up
 * a bounded wait on an MMA or copy after `polls` polls instead of their full
 * limit (polls = 0 restores the full limit).  A kernel that gives up first
 * waits, with the full limit, for the MMAs and copies it has issued, then
 * sets its tq_device_fault bit, releases its tensor memory and returns; its
 * outputs are undefined.  Not for production use: a short limit makes
 * ordinary launches fail.  Errors: TQ_ERR_ARG for a null context or
 * polls < 0.  Host-only; no device work.
 */
int tq_set_wait_limit(tq_ctx* c, int polls);

/*
 * tq_init - build the per-context tables on the host in fp64 and upload them
 * to the current CUDA device ([WHAT] stage 1 steps 1-2, stage 2).
 *   d       vector dimension.
 *   bits_k  bits per key coordinate, counting the QJL bit when qjl_m > 0
 *           (k3 = 2 Lloyd-Max bits + 1 QJL bit).
 *   bits_v  Lloyd-Max bits per value coordinate (values get no QJL stage).
 *   qjl_m   rows of the QJL matrix S (0 disables the key QJL stage).
 *   seed    seeds the Gaussian matrix G (rotation) and S (SplitMix64 streams
 *           0 and 1, Box-Muller normals, row-major fill).
 * Tables: Pi = Q diag(sgn diag R) from G = QR (y = Pi x); S (m x d) rounded to
 * fp16; Lloyd-Max centroids and boundaries for the law
 * f(t) ~ (1-t^2)^((d-3)/2) at each bit width.  Allocates device memory owned
 * by the context (the only allocating call).  Returns NULL on error (see
 * tq_last_error).
 */
tq_ctx* tq_init(int d, int bits_k, int bits_v, int qjl_m, uint64_t seed);

/* Flags of tq_init_ex. */
enum tq_flags { TQ_NC_KEYS = 1, TQ_NC_VALUES = 2, TQ_NORM_F16 = 4 };

/*
 * tq_init_ex - tq_init with options.  The norm-corrected variants named in
 * "A First Comprehensive Study of TurboQuant: Accuracy and Performance",
 * section A3 (k3v4_nc, 3bit_nc, 4bit_nc) leave "norm correction" undefined;
 * this library reads it as storing n / |c[idx]| in place of n, where c[idx]
 * is the vector of the Lloyd-Max centroids a vector's indices select in the
 * rotated domain, so the dequantized vector n Pi^T c[idx] / |c[idx]| keeps
 * the input's norm exactly.  The packed layout is unchanged; only the value
 * stored in `norm` differs, so dequantize, logits, attention and top-k read
 * it as before.
 *   flags  TQ_NC_KEYS: norm correction of keys, which must then be MSE-only
 *          (qjl_m = 0, else NULL with TQ_ERR_UNSUPPORTED);
 *          TQ_NC_VALUES: norm correction of values;
 *          TQ_NORM_F16: the per-vector norms of keys and values are stored as
 *          IEEE binary16 (2 bytes, rounded to nearest even from the fp32
 *          value) instead of fp32, as the serving formats of that study do;
 *          keys must then be MSE-only (qjl_m = 0: gamma stays fp32-only).
 *          The `norm` arrays of every call are then uint16 arrays.
 *          Other bits: NULL with TQ_ERR_ARG.
 * Otherwise as tq_init.
 */
tq_ctx* tq_init_ex(int d, int bits_k, int bits_v, int qjl_m, uint64_t seed, int flags);

/* Frees the context's device tables.  NULL is ignored. */
void tq_destroy(tq_ctx* ctx);

/* Packed layout of keys (which = TQ_KEY) or values (TQ_VALUE). */
int tq_layout(const tq_ctx* ctx, int which, tq_layout_t* out);

/*
 * tq_host_tables - the same tables tq_init builds, computed on the host only
 * (no CUDA call; usable without a GPU).  Any output pointer may be NULL.
 *   pi  [d*d] row-major Pi;  S [qjl_m*d] row-major (fp16-rounded values);
 *   ck  [2^(bits_k_lm)] key centroids, bk [2^(bits_k_lm)-1] key boundaries;
 *   cv  [2^bits_v] value centroids, bv [2^bits_v - 1] value boundaries
 *   (bits_k_lm = bits_k - 1 when qjl_m > 0, else bits_k).
 */
int tq_host_tables(int d, int bits_k, int bits_v, int qjl_m, uint64_t seed,
                   double* pi, double* S, double* ck, double* bk,
                   double* cv, double* bv);

/* Copies the context's fp64 host tables (layouts as tq_host_tables). */
int tq_export_tables(const tq_ctx* ctx, double* pi, double* S, double* ck,
                     double* bk, double* cv, double* bv);

/*
 * tq_quantize - online quantization of n vectors ([WHAT] stage 1: normalise,
 * rotate, Lloyd-Max index per coordinate; stage 2 for keys: residual
 * r = Pi x/|x| - c[idx], QJL bits sign(S r), gamma = |x| |r|).
 *   which   TQ_KEY or TQ_VALUE.
 *   x       device, [n][ld] elements of `dtype` (TQ_F32/TQ_BF16/TQ_F16),
 *           ld >= d; rows 16-byte aligned when dtype is 16-bit and ld%8==0.
 *   codes   device, uint32 [n][W].
 *   qjl     device, uint32 [n][ceil(m/32)] (keys with QJL; else ignored, may be NULL).
 *   norm    device, float [n] (binary16 under TQ_NORM_F16).
 *   rnorm   device, float [n] (keys with QJL; else ignored, may be NULL).
 * n = 0 is a no-op.  A zero vector gets norm 0, every index 2^bits/2, rnorm 0.
 * Inputs must be finite with |x|^2 representable in fp32.
 */
int tq_quantize(tq_ctx* ctx, int which, const void* x, int dtype, int64_t n,
                int64_t ld, uint32_t* codes, uint32_t* qjl, void* norm,
                float* rnorm, void* stream);

/*
 * tq_quantize_append - quantize the newest token of each sequence straight
 * into a packed KV cache (the per-step cache update of decoding; "What is
 * TurboQuant?", "How to implement" part 1: the cache quantizes on every
 * update).  Same arithmetic as tq_quantize.
 *   x       device, [B][H][d] rows of `dtype` (row b*H+g is head g of sequence
 *           b; row stride ld >= d elements).
 *   max_T   cache capacity per (sequence, head).
 *   pos     device, int32 [B]: the slot to write for sequence b.  A sequence
 *           whose pos is outside [0, max_T) is skipped (nothing written).
 *   codes/qjl/norm/rnorm  device cache arrays [B][H][max_T][...] as in
 *           tq_quantize; only the B*H addressed records are written.
 */
int tq_quantize_append(tq_ctx* ctx, int which, const void* x, int dtype, int B,
                       int H, int64_t ld, int64_t max_T, const int32_t* pos,
                       uint32_t* codes, uint32_t* qjl, void* norm, float* rnorm,
                       void* stream);

/*
 * tq_quantize_append_paged - tq_quantize_append into a paged cache (blocks of
 * block_size tokens allocated from a pool, as serving engines lay out their
 * KV caches; "A First Comprehensive Study of TurboQuant", section A3).
 *   codes/qjl/norm/rnorm  device cache arrays [num_blocks][H][block_size][...].
 *   block_table  device, int32 [B][max_blocks]: block ids in [0, num_blocks).
 *   pos          device, int32 [B]: token position of sequence b; it goes to
 *                slot pos % block_size of block block_table[b][pos / block_size].
 * A sequence whose pos is outside [0, max_blocks * block_size), or whose
 * block id is outside [0, num_blocks), is skipped (nothing written).
 */
int tq_quantize_append_paged(tq_ctx* ctx, int which, const void* x, int dtype, int B,
                             int H, int64_t ld, const int32_t* block_table,
                             int max_blocks, int block_size, int64_t num_blocks,
                             const int32_t* pos, uint32_t* codes, uint32_t* qjl,
                             void* norm, float* rnorm, void* stream);

/*
 * tq_dequantize - x_hat = |x| Pi^T c[idx], plus for keys with QJL the
 * back-projection sqrt(pi/2)/m * gamma * Pi^T S^T sigma (sigma = +-1 from the
 * QJL bits), so that <q, x_hat> equals tq_logits.
 *   codes/qjl/norm/rnorm  device arrays as produced by tq_quantize.
 *   out     device, float [n][d].
 */
int tq_dequantize(tq_ctx* ctx, int which, const uint32_t* codes,
                  const uint32_t* qjl, const void* norm, const float* rnorm,
                  int64_t n, float* out, void* stream);

/*
 * tq_logits - unscaled logits <q, k> evaluated from the packed keys without
 * dequantizing them ([WHAT] "How TurboQuant works" closing paragraph; "How to
 * implement" part 1): q' = Pi q once, s = S q', then
 *   l = norm * <q', c[idx]> + sqrt(pi/2)/m * rnorm * <s, sigma>.
 *   q       device, [nq][d] of `dtype`.
 *   kcodes/kqjl/knorm/krnorm  device key arrays for nk keys.
 *   out     device, float [nq][nk].
 */
int tq_logits(tq_ctx* ctx, const void* q, int dtype, int64_t nq,
              const uint32_t* kcodes, const uint32_t* kqjl, const void* knorm,
              const float* krnorm, int64_t nk, float* out, void* stream);

/* Bytes of workspace tq_attn_decode needs for these sizes. */
size_t tq_attn_workspace_bytes(const tq_ctx* ctx, int B, int Hq, int64_t max_T);

/*
 * tq_attn_decode - one decode step of attention over a packed KV cache
 * ([WHAT] "How TurboQuant works" closing paragraph; [VLLM] A2): for query
 * head h of sequence b, kv head g = h*Hkv/Hq (GQA grouping),
 *   s_i = scale * l_i (i < seq_lens[b]),  p = softmax(s),
 *   out = sum_i p_i * vnorm_i * Pi^T cv[vidx_i].
 * The context is split over CTAs; partial softmax states are merged by
 * log-sum-exp and the Pi^T is applied once per head after the merge.
 *   q        device, [B][Hq][d] of `dtype`.
 *   kcodes   device, uint32 [B][Hkv][max_T][Wk]; kqjl [B][Hkv][max_T][ceil(m/32)];
 *   knorm, krnorm  device, float [B][Hkv][max_T] (knorm binary16 under
 *            TQ_NORM_F16).
 *   vcodes   device, uint32 [B][Hkv][max_T][Wv]; vnorm float [B][Hkv][max_T]
 *            (binary16 under TQ_NORM_F16).
 *   seq_lens device, int32 [B], each in [0, max_T]; a length of 0 gives out = 0.
 *   scale    softmax scale (callers usually pass 1/sqrt(d)).
 *   out      device, float [B][Hq][d].
 *   workspace/ws_bytes  device scratch of tq_attn_workspace_bytes() bytes.
 * Requires Hq % Hkv == 0 and Hq/Hkv <= 16.
 */
int tq_attn_decode(tq_ctx* ctx, const void* q, int dtype, int B, int Hq,
                   int Hkv, const uint32_t* kcodes, const uint32_t* kqjl,
                   const void* knorm, const float* krnorm,
                   const uint32_t* vcodes, const void* vnorm, int64_t max_T,
                   const int32_t* seq_lens, float scale, float* out,
                   void* workspace, size_t ws_bytes, void* stream);

/*
 * tq_attn_decode_static - tq_attn_decode for callers that cannot allocate
 * device memory on the call path (for example a plugin whose host framework
 * owns every device allocation, or a serving loop that forbids allocation
 * after start-up) and cannot pass a workspace.  The method's sources have no
 * counterpart: this is an interface convenience.
 * The scratch is a file-scope device array of tq_attn_static_scratch_bytes()
 * bytes (32 MiB) that every GPU loading the library holds until exit; sizes
 * whose tq_attn_workspace_bytes() exceed it are rejected with
 * TQ_ERR_WORKSPACE.  The first call on a device looks up the array's device
 * address (once per device, with that device current); make that first call
 * before any stream capture.  The call allocates nothing.  All calls share
 * the one array and it keeps the last call's contents (nothing in it needs to
 * start at zero), so calls that overlap on the GPU - on different streams,
 * or from different threads - race and must be serialised by the caller.
 * Arguments and results are those of tq_attn_decode.
 */
int tq_attn_decode_static(tq_ctx* ctx, const void* q, int dtype, int B, int Hq,
                          int Hkv, const uint32_t* kcodes, const uint32_t* kqjl,
                          const void* knorm, const float* krnorm,
                          const uint32_t* vcodes, const void* vnorm,
                          int64_t max_T, const int32_t* seq_lens, float scale,
                          float* out, void* stream);

/* Size in bytes of the static scratch used by tq_attn_decode_static. */
size_t tq_attn_static_scratch_bytes(void);

/*
 * tq_attn_decode_paged - tq_attn_decode over a paged cache: token t of
 * sequence b is record (block_table[b][t / block_size] * Hkv + g) *
 * block_size + t % block_size of the arrays [num_blocks][Hkv][block_size][...]
 * (g = kv head).  block_size must be a multiple of 16; seq_lens[b] is clamped
 * to max_blocks * block_size.  The tokens of a block whose id is outside
 * [0, num_blocks) are masked: like tokens past seq_lens[b] they get no
 * weight (a sequence with every token masked gets out = 0).  Only the
 * tensor-core decode takes paged caches: d = 128, GQA group 1, 2, 4 or 8, and
 * keys of 2 or 3 Lloyd-Max bits + 128 QJL rows with 4-bit values, or MSE-only
 * keys of 3, 4 or 8 bits with 4-bit values (3-bit keys also with 3-bit
 * values); other formats return TQ_ERR_UNSUPPORTED.  Workspace:
 * tq_attn_workspace_bytes(ctx, B, Hq, max_blocks * block_size).
 */
int tq_attn_decode_paged(tq_ctx* ctx, const void* q, int dtype, int B, int Hq, int Hkv,
                         const uint32_t* kcodes, const uint32_t* kqjl, const void* knorm,
                         const float* krnorm, const uint32_t* vcodes, const void* vnorm,
                         const int32_t* block_table, int max_blocks, int block_size,
                         int64_t num_blocks, const int32_t* seq_lens, float scale, float* out,
                         void* workspace, size_t ws_bytes, void* stream);

/*
 * tq_decode_step - one whole decode step: append the newest key and value of
 * every (sequence, kv head) to the packed cache, then attend over the cache
 * including them ([WHAT] "How to implement" part 1: the cache quantizes on
 * every update and the fused kernel attends straight from the codes).  Same
 * results as tq_quantize_append (keys, then values) followed by
 * tq_attn_decode with seq_lens[b] = min(pos[b] + 1, max_T), in three launches
 * instead of five: append + query pre-rotation in one, attention, merge.
 *   q        device, [B][Hq][d] of q_dtype.
 *   k_new, v_new  device, [B][Hkv][d] contiguous rows of kv_dtype.
 *   kcodes .. vnorm  the cache arrays of tq_attn_decode (written at pos).
 *   pos      device, int32 [B]: the slot of the new token; sequence b then
 *            attends over tokens [0, pos[b]].  pos outside [0, max_T) writes
 *            nothing (pos < 0 attends over nothing, out = 0; pos >= max_T
 *            attends over the full cache).
 *   scale, out, workspace/ws_bytes  as in tq_attn_decode
 *            (tq_attn_workspace_bytes() bytes).
 */
int tq_decode_step(tq_ctx* ctx, const void* q, int q_dtype, const void* k_new,
                   const void* v_new, int kv_dtype, int B, int Hq, int Hkv,
                   uint32_t* kcodes, uint32_t* kqjl, void* knorm, float* krnorm,
                   uint32_t* vcodes, void* vnorm, int64_t max_T, const int32_t* pos,
                   float scale, float* out, void* workspace, size_t ws_bytes,
                   void* stream);

/*
 * tq_decode_step_paged - tq_decode_step over a paged cache (block table and
 * layout as in tq_attn_decode_paged; the new token of sequence b goes to
 * position pos[b] as in tq_quantize_append_paged).
 */
int tq_decode_step_paged(tq_ctx* ctx, const void* q, int q_dtype, const void* k_new,
                         const void* v_new, int kv_dtype, int B, int Hq, int Hkv,
                         uint32_t* kcodes, uint32_t* kqjl, void* knorm, float* krnorm,
                         uint32_t* vcodes, void* vnorm, const int32_t* block_table,
                         int max_blocks, int block_size, int64_t num_blocks,
                         const int32_t* pos, float scale, float* out, void* workspace,
                         size_t ws_bytes, void* stream);

/*
 * Bytes of workspace tq_topk needs: the database dequantized once into fp16
 * rows (n * (d + m, each rounded up to 16) * 2 bytes; 832 MB for 1e6
 * vectors at d = m = 200), the queries' operands, and the candidate lists.
 */
size_t tq_topk_workspace_bytes(const tq_ctx* ctx, int64_t nq, int64_t n, int k);

/*
 * tq_topk - exact top-k of the compressed inner-product scores of nq queries
 * against n packed database keys ([WHAT] "Benchmarks": vector search by
 * inner product), ordered by (score desc, index asc).  Scores are tq_logits
 * up to the fp16 rounding of the scorer's operands (~1e-5 |q| |k|): the
 * database rows and the queries are rounded to fp16 for the tensor cores,
 * the norms and the accumulation stay fp32.
 *   q        device, [nq][d] of `dtype`.
 *   codes/qjl/norm/rnorm  device key arrays for the n database vectors.
 *   k        1..32.
 *   idx      device, int32 [nq][k];  score  device, float [nq][k].
 * If n < k the missing slots get index -1 and score -inf.  Keys of 8
 * Lloyd-Max bits: TQ_ERR_UNSUPPORTED.
 */
int tq_topk(tq_ctx* ctx, const void* q, int dtype, int64_t nq,
            const uint32_t* codes, const uint32_t* qjl, const void* norm,
            const float* rnorm, int64_t n, int k, int32_t* idx, float* score,
            void* workspace, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
