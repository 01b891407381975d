// C ABI of libtq: argument checks, context set-up and kernel launches.
// The operations and their sources are documented in include/tq.h.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <string>

#include "tq_internal.h"

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* where) {
  return fail(TQ_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool valid_dims(int d, int bits_k, int bits_v, int qjl_m, int* code) {
  if (d < 8 || d > 256 || d % 8 != 0) {
    *code = fail(TQ_ERR_UNSUPPORTED, "d=%d unsupported (need 8 <= d <= 256, d %% 8 == 0)", d);
    return false;
  }
  const int J = (d + 31) / 32;
  if (qjl_m < 0 || qjl_m % 8 != 0 || qjl_m > 32 * J) {
    *code = fail(TQ_ERR_UNSUPPORTED, "qjl_m=%d unsupported (need 0 <= m <= %d, m %% 8 == 0)", qjl_m, 32 * J);
    return false;
  }
  const int bk_lm = qjl_m > 0 ? bits_k - 1 : bits_k;
  if (!((bk_lm >= 1 && bk_lm <= 4) || bk_lm == 8)) {
    *code = fail(TQ_ERR_UNSUPPORTED, "bits_k=%d with qjl_m=%d gives %d Lloyd-Max bits (need 1..4 or 8)",
                 bits_k, qjl_m, bk_lm);
    return false;
  }
  if (!((bits_v >= 1 && bits_v <= 4) || bits_v == 8)) {
    *code = fail(TQ_ERR_UNSUPPORTED, "bits_v=%d unsupported (need 1..4 or 8)", bits_v);
    return false;
  }
  return true;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_ctx(const tq_ctx* c) {
  if (!c) return fail(TQ_ERR_ARG, "null context");
  return TQ_OK;
}

// Compute calls launch on the current device, and the context's tables live
// on the device it was created on: a mismatch is refused before any launch.
int check_ctx_dev(const tq_ctx* c, const char* name) {
  if (!c) return fail(TQ_ERR_ARG, "%s: null context", name);
  int cur = -1;
  const cudaError_t e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return cuda_fail(e, name);
  if (cur != c->device)
    return fail(TQ_ERR_ARG, "%s: the context belongs to device %d but device %d is current", name,
                c->device, cur);
  return TQ_OK;
}

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

}  // namespace

extern "C" {

const char* tq_last_error(void) { return g_err.c_str(); }

const char* tq_version(void) { return "libtq 0.1 (sm_100a)"; }

int tq_set_wait_limit(tq_ctx* c, int polls) {
  if (!c || polls < 0) return fail(TQ_ERR_ARG, "tq_set_wait_limit: null context or negative polls");
  c->wait_limit = polls;
  return TQ_OK;
}

int tq_device_fault(int* code) {
  if (!code) return fail(TQ_ERR_ARG, "tq_device_fault: null output");
  int q = 0, t = 0;
  cudaError_t e = tqk::read_and_clear_fault(&q);
  if (e == cudaSuccess) e = tqk::read_and_clear_topk_fault(&t);
  if (e != cudaSuccess) return cuda_fail(e, "tq_device_fault");
  *code = q | (t << 1);
  return TQ_OK;
}

int tq_host_tables(int d, int bits_k, int bits_v, int qjl_m, uint64_t seed, double* pi,
                   double* S, double* ck, double* bk, double* cv, double* bv) {
  int code = TQ_OK;
  if (!valid_dims(d, bits_k, bits_v, qjl_m, &code)) return code;
  const int bk_lm = qjl_m > 0 ? bits_k - 1 : bits_k;
  try {
    if (pi) {
      std::vector<double> P;
      tqh::rotation(d, seed, P);
      std::memcpy(pi, P.data(), P.size() * sizeof(double));
    }
    if (S && qjl_m > 0) {
      std::vector<double> Sm;
      tqh::qjl_matrix(qjl_m, d, seed, Sm);
      std::memcpy(S, Sm.data(), Sm.size() * sizeof(double));
    }
    std::vector<double> c, b;
    if (ck || bk) {
      tqh::lloyd_max(d, bk_lm, c, b);
      if (ck) std::memcpy(ck, c.data(), c.size() * sizeof(double));
      if (bk) std::memcpy(bk, b.data(), b.size() * sizeof(double));
    }
    if (cv || bv) {
      tqh::lloyd_max(d, bits_v, c, b);
      if (cv) std::memcpy(cv, c.data(), c.size() * sizeof(double));
      if (bv) std::memcpy(bv, b.data(), b.size() * sizeof(double));
    }
  } catch (const std::bad_alloc&) {
    return fail(TQ_ERR_ARG, "host allocation failed");
  }
  return TQ_OK;
}

tq_ctx* tq_init(int d, int bits_k, int bits_v, int qjl_m, uint64_t seed) {
  return tq_init_ex(d, bits_k, bits_v, qjl_m, seed, 0);
}

tq_ctx* tq_init_ex(int d, int bits_k, int bits_v, int qjl_m, uint64_t seed, int flags) {
  int code = TQ_OK;
  if (!valid_dims(d, bits_k, bits_v, qjl_m, &code)) return nullptr;
  if (flags & ~(TQ_NC_KEYS | TQ_NC_VALUES | TQ_NORM_F16)) {
    fail(TQ_ERR_ARG, "tq_init_ex: unknown flag bits 0x%x", flags);
    return nullptr;
  }
  if ((flags & TQ_NC_KEYS) && qjl_m > 0) {
    fail(TQ_ERR_UNSUPPORTED, "tq_init_ex: key norm correction needs MSE-only keys (qjl_m = 0)");
    return nullptr;
  }
  if ((flags & TQ_NORM_F16) && qjl_m > 0) {
    fail(TQ_ERR_UNSUPPORTED, "tq_init_ex: fp16 norms need MSE-only keys (qjl_m = 0)");
    return nullptr;
  }
  tq_ctx* c = new (std::nothrow) tq_ctx();
  if (!c) {
    fail(TQ_ERR_ARG, "host allocation failed");
    return nullptr;
  }
  c->nc_k = (flags & TQ_NC_KEYS) != 0;
  c->nc_v = (flags & TQ_NC_VALUES) != 0;
  c->norm_f16 = (flags & TQ_NORM_F16) != 0;
  c->d = d;
  c->J = (d + 31) / 32;
  c->dpad = 32 * c->J;
  c->bits_k = bits_k;
  c->bk_lm = qjl_m > 0 ? bits_k - 1 : bits_k;
  c->bits_v = bits_v;
  c->qjl_m = qjl_m;
  c->seed = seed;
  c->wk = tq_code_words(d, c->bk_lm);
  c->wv = tq_code_words(d, bits_v);
  tqh::rotation(d, seed, c->Pi);
  tqh::qjl_matrix(qjl_m, d, seed, c->S);
  tqh::lloyd_max(d, c->bk_lm, c->ck, c->bk);
  tqh::lloyd_max(d, bits_v, c->cv, c->bv);

  cudaError_t e = cudaGetDevice(&c->device);
  if (e != cudaSuccess) {
    cuda_fail(e, "tq_init: cudaGetDevice");
    delete c;
    return nullptr;
  }
  const int dp = c->dpad;
  // Every table starts on a 16-byte boundary (kernels copy them with 16-byte
  // asynchronous copies): Pi's d * d entries are padded to a multiple of 4.
  const size_t nPiT = (size_t)d * dp, nPi = ((size_t)d * d + 3) & ~(size_t)3, nST = (size_t)d * dp,
               nS = (size_t)dp * d;
  const size_t total = (nPiT + nPi + nST + nS + 4 * tqk::kMaxLevels) * sizeof(float);
  std::vector<float> h(total / sizeof(float), 0.f);
  float* hPiT = h.data();
  float* hPi = hPiT + nPiT;
  float* hST = hPi + nPi;
  float* hS = hST + nST;
  float* hck = hS + nS;
  float* hbk = hck + tqk::kMaxLevels;
  float* hcv = hbk + tqk::kMaxLevels;
  float* hbv = hcv + tqk::kMaxLevels;
  for (int j = 0; j < d; ++j)
    for (int k = 0; k < d; ++k) {
      hPiT[(size_t)k * dp + j] = (float)c->Pi[(size_t)j * d + k];
      hPi[(size_t)j * d + k] = (float)c->Pi[(size_t)j * d + k];
    }
  for (int i = 0; i < qjl_m; ++i)
    for (int k = 0; k < d; ++k) {
      hST[(size_t)k * dp + i] = (float)c->S[(size_t)i * d + k];
      hS[(size_t)i * d + k] = (float)c->S[(size_t)i * d + k];
    }
  for (int i = 0; i < tqk::kMaxLevels; ++i) {
    hbk[i] = INFINITY;
    hbv[i] = INFINITY;
  }
  for (size_t i = 0; i < c->ck.size(); ++i) hck[i] = (float)c->ck[i];
  for (size_t i = 0; i < c->bk.size(); ++i) hbk[i] = (float)c->bk[i];
  for (size_t i = 0; i < c->cv.size(); ++i) hcv[i] = (float)c->cv[i];
  for (size_t i = 0; i < c->bv.size(); ++i) hbv[i] = (float)c->bv[i];

  e = tqk::configure_kernels();
  if (e != cudaSuccess) {
    cuda_fail(e, "tq_init: kernel attributes");
    delete c;
    return nullptr;
  }
  e = cudaMalloc(&c->dev_block, total);
  if (e != cudaSuccess) {
    cuda_fail(e, "tq_init: cudaMalloc");
    delete c;
    return nullptr;
  }
  e = cudaMemcpy(c->dev_block, h.data(), total, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    cuda_fail(e, "tq_init: cudaMemcpy");
    cudaFree(c->dev_block);
    delete c;
    return nullptr;
  }
  // Operand images of the tensor-core quantizer (d = 128): 128 x 128 fp16,
  // K-major, two 64-wide K blocks, 16-byte chunks swizzled with the row.
  if (cudaDeviceGetAttribute(&c->sms, cudaDevAttrMultiProcessorCount, c->device) != cudaSuccess) c->sms = 148;
  if (d == 128) {
    // images: 0 fp16 head, 1 fp16 tail, 2 S, then (after the row norms) the
    // three bf16 terms of 2^8 Pi
    std::vector<uint16_t> img(3 * 128 * 128, 0), imgb(3 * 128 * 128, 0);
    std::vector<float> snorm(128, 0.f);
    auto put = [&](int which, int r, int k, double v) {
      const int kb = k >> 6, kk = k & 63, ch = kk >> 3, w = kk & 7;
      const size_t off = (size_t)kb * 16384 + (size_t)(r >> 3) * 1024 + (size_t)(r & 7) * 128 +
                         (size_t)((ch ^ (r & 7)) << 4) + (size_t)w * 2;
      const __half h = __float2half_rn((float)v);
      img[(size_t)which * 16384 + off / 2] = *reinterpret_cast<const uint16_t*>(&h);
    };
    auto bf16_rn = [](double v) {   // nearest bf16 (ties to even) of the fp32 rounding of v
      const float f = (float)v;
      uint32_t u;
      std::memcpy(&u, &f, 4);
      u += 0x7FFFu + ((u >> 16) & 1u);
      const uint16_t h = (uint16_t)(u >> 16);
      uint32_t back = (uint32_t)h << 16;
      float g;
      std::memcpy(&g, &back, 4);
      return std::make_pair(h, (double)g);
    };
    for (int j = 0; j < 128; ++j)
      for (int k = 0; k < 128; ++k) {
        const double v = 256.0 * c->Pi[(size_t)j * d + k];
        const double hi = tqh::round_to_half(v);
        put(0, j, k, hi);
        put(1, j, k, tqh::round_to_half(v - hi));
        // bf16 terms: v = b0 + b1 + b2 to ~24 bits
        double rem = v;
        const int kb = k >> 6, kk = k & 63, ch = kk >> 3, w = kk & 7;
        const size_t off = (size_t)kb * 16384 + (size_t)(j >> 3) * 1024 + (size_t)(j & 7) * 128 +
                           (size_t)((ch ^ (j & 7)) << 4) + (size_t)w * 2;
        for (int t = 0; t < 3; ++t) {
          const auto b = bf16_rn(rem);
          imgb[(size_t)t * 16384 + off / 2] = b.first;
          rem -= b.second;
        }
      }
    for (int i = 0; i < qjl_m; ++i) {
      double nn = 0.0;
      for (int k = 0; k < 128; ++k) {
        put(2, i, k, c->S[(size_t)i * d + k]);
        nn += c->S[(size_t)i * d + k] * c->S[(size_t)i * d + k];
      }
      snorm[i] = (float)std::sqrt(nn);
    }
    void* tc = nullptr;
    const size_t boff = 98304 + 1024;   // bf16 images after the row norms, 1 KB aligned
    e = cudaMalloc(&tc, boff + imgb.size() * 2);
    if (e == cudaSuccess) {
      e = cudaMemcpy(tc, img.data(), img.size() * 2, cudaMemcpyHostToDevice);
      if (e == cudaSuccess)
        e = cudaMemcpy(static_cast<char*>(tc) + img.size() * 2, snorm.data(), snorm.size() * 4,
                       cudaMemcpyHostToDevice);
      if (e == cudaSuccess)
        e = cudaMemcpy(static_cast<char*>(tc) + boff, imgb.data(), imgb.size() * 2, cudaMemcpyHostToDevice);
    }
    if (e != cudaSuccess) {
      cuda_fail(e, "tq_init: tensor-core tables");
      if (tc) cudaFree(tc);
      cudaFree(c->dev_block);
      delete c;
      return nullptr;
    }
    c->tc_block = tc;
    c->tc_pih = tc;
    c->tc_pil = static_cast<char*>(tc) + 32768;
    c->tc_s = static_cast<char*>(tc) + 65536;
    c->tc_snorm = reinterpret_cast<const float*>(static_cast<char*>(tc) + 98304);
    c->tc_pib = static_cast<char*>(tc) + boff;
    c->tc_ok = true;
  }
  const float* base = static_cast<const float*>(c->dev_block);
  c->PiT = base;
  c->Pi_f = base + (hPi - hPiT);
  c->ST = base + (hST - hPiT);
  c->S_f = base + (hS - hPiT);
  c->ck_f = base + (hck - hPiT);
  c->bk_f = base + (hbk - hPiT);
  c->cv_f = base + (hcv - hPiT);
  c->bv_f = base + (hbv - hPiT);
  return c;
}

void tq_destroy(tq_ctx* c) {
  if (!c) return;
  if (c->dev_block) {
    int cur = 0;
    cudaGetDevice(&cur);
    if (cur != c->device) cudaSetDevice(c->device);
    cudaFree(c->dev_block);
    if (c->tc_block) cudaFree(c->tc_block);
    if (cur != c->device) cudaSetDevice(cur);
  }
  delete c;
}

int tq_layout(const tq_ctx* c, int which, tq_layout_t* out) {
  if (int r = check_ctx(c)) return r;
  if (!out) return fail(TQ_ERR_ARG, "tq_layout: null output");
  if (which != TQ_KEY && which != TQ_VALUE) return fail(TQ_ERR_ARG, "tq_layout: bad which=%d", which);
  const bool key = which == TQ_KEY;
  out->d = c->d;
  out->bits = key ? c->bk_lm : c->bits_v;
  out->words = key ? c->wk : c->wv;
  out->qjl_m = key ? c->qjl_m : 0;
  out->qjl_words = (out->qjl_m + 31) / 32;
  out->has_rnorm = (key && c->qjl_m > 0) ? 1 : 0;
  out->norm_bytes = c->norm_f16 ? 2 : 4;
  out->bytes_per_vector = (int64_t)out->words * 4 + (int64_t)out->qjl_words * 4 + out->norm_bytes +
                          (out->has_rnorm ? 4 : 0);
  return TQ_OK;
}

int tq_export_tables(const tq_ctx* c, double* pi, double* S, double* ck, double* bk, double* cv,
                     double* bv) {
  if (int r = check_ctx(c)) return r;
  if (pi) std::memcpy(pi, c->Pi.data(), c->Pi.size() * sizeof(double));
  if (S && c->qjl_m > 0) std::memcpy(S, c->S.data(), c->S.size() * sizeof(double));
  if (ck) std::memcpy(ck, c->ck.data(), c->ck.size() * sizeof(double));
  if (bk) std::memcpy(bk, c->bk.data(), c->bk.size() * sizeof(double));
  if (cv) std::memcpy(cv, c->cv.data(), c->cv.size() * sizeof(double));
  if (bv) std::memcpy(bv, c->bv.data(), c->bv.size() * sizeof(double));
  return TQ_OK;
}

// Block table of a paged cache: arrays [num_blocks][H][block_size][...],
// table [B][max_blocks]; null table = contiguous [B][H][max_T][...].
struct Paging {
  const int32_t* table = nullptr;
  int max_blocks = 0, block_size = 0;
  int64_t num_blocks = 0;
};

static int quantize_common(tq_ctx* c, int which, const void* x, int dtype, int64_t n, int64_t ld,
                           uint32_t* codes, uint32_t* qjl, void* norm, float* rnorm,
                           const int32_t* pos, int H, int64_t max_T, void* stream,
                           const char* name, const Paging& pg = Paging()) {
  if (int r = check_ctx_dev(c, name)) return r;
  if (which != TQ_KEY && which != TQ_VALUE) return fail(TQ_ERR_ARG, "%s: bad which=%d", name, which);
  if (dtype != TQ_F32 && dtype != TQ_BF16 && dtype != TQ_F16)
    return fail(TQ_ERR_ARG, "%s: bad dtype=%d", name, dtype);
  if (n < 0 || ld < c->d)
    return fail(TQ_ERR_ARG, "%s: n=%lld ld=%lld (need n >= 0, ld >= d)", name, (long long)n, (long long)ld);
  if (n == 0) return TQ_OK;
  const bool key = which == TQ_KEY;
  const int m = key ? c->qjl_m : 0;
  if (!x || !codes || !norm) return fail(TQ_ERR_ARG, "%s: null pointer", name);
  if (m > 0 && (!qjl || !rnorm)) return fail(TQ_ERR_ARG, "%s: keys with QJL need qjl and rnorm", name);
  if (!aligned(codes, 4) || !aligned(norm, c->norm_f16 ? 2 : 4))
    return fail(TQ_ERR_ARG, "%s: misaligned output", name);
  tqk::QuantArgs a{};
  a.x = x;
  a.dtype = dtype;
  a.n = n;
  a.ld = ld;
  a.d = c->d;
  a.bits = key ? c->bk_lm : c->bits_v;
  a.nbnd = (1 << a.bits) - 1;
  a.m = m;
  a.words = key ? c->wk : c->wv;
  a.PiT = c->PiT;
  a.ST = c->ST;
  a.cen = key ? c->ck_f : c->cv_f;
  a.bnd = key ? c->bk_f : c->bv_f;
  a.codes = codes;
  a.qjl = qjl;
  a.norm = static_cast<float*>(norm);
  a.rnorm = rnorm;
  a.pos = pos;
  a.H = H;
  a.max_T = max_T;
  a.block_table = pg.table;
  a.max_blocks = pg.max_blocks;
  a.block_size = pg.block_size;
  a.num_blocks = pg.num_blocks;
  a.nc = (key ? c->nc_k : c->nc_v) ? 1 : 0;
  a.nf16 = c->norm_f16 ? 1 : 0;
  if (n <= tqk::kSmallQuantize) {
    cudaError_t e = tqk::launch_quantize_small(c, a, as_stream(stream));
    if (e != cudaSuccess) return cuda_fail(e, name);
    return TQ_OK;
  }
  const bool tc = !pg.table && (a.bits <= 4 || a.bits == 8) && c->tc_ok && c->d == 128 && (dtype == TQ_BF16 || dtype == TQ_F16) && ld % 8 == 0 &&
                  aligned(x, 16) && aligned(codes, 16) && (m == 0 || (m == 128 && aligned(qjl, 16)));
  if (tc) {
    tqk::QuantTcArgs t{};
    t.x = x;
    t.dtype = dtype;
    t.n = n;
    t.ld = ld;
    t.bits = a.bits;
    t.m = m;
    t.pi_hi = c->tc_pih;
    t.pi_lo = c->tc_pil;
    t.pi_b = c->tc_pib;
    t.s_img = c->tc_s;
    t.snorm = c->tc_snorm;
    t.s_f32 = c->S_f;
    t.codes = codes;
    t.qjl = qjl;
    t.norm = static_cast<float*>(norm);
    t.rnorm = rnorm;
    t.pos = pos;
    t.H = H;
    t.max_T = max_T;
    const std::vector<double>& cen = key ? c->ck : c->cv;
    const std::vector<double>& bnd = key ? c->bk : c->bv;
    for (int i = 0; i < 16; ++i) {
      t.cen[i] = i < (int)cen.size() ? (float)cen[i] : 0.f;
      t.bnd[i] = i < (int)bnd.size() ? (float)bnd[i] : INFINITY;
    }
    t.wait_limit = c->wait_limit;
    t.nc = a.nc ? 1 : 0;
    t.nf16 = a.nf16 ? 1 : 0;
    t.bnd_dev = a.bnd;
    cudaError_t e = tqk::launch_quant_tc(t, c->sms, as_stream(stream));
    if (e != cudaErrorNotSupported) {   // unsupported: nothing was launched, the fp32 kernels take it
      if (e != cudaSuccess) return cuda_fail(e, name);
      return TQ_OK;
    }
  }
  cudaError_t e = tqk::launch_quantize(c, a, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, name);
  return TQ_OK;
}

int tq_quantize(tq_ctx* c, int which, const void* x, int dtype, int64_t n, int64_t ld,
                uint32_t* codes, uint32_t* qjl, void* norm, float* rnorm, void* stream) {
  return quantize_common(c, which, x, dtype, n, ld, codes, qjl, norm, rnorm, nullptr, 0, 0, stream,
                         "tq_quantize");
}

int tq_quantize_append(tq_ctx* c, int which, const void* x, int dtype, int B, int H, int64_t ld,
                       int64_t max_T, const int32_t* pos, uint32_t* codes, uint32_t* qjl,
                       void* norm, float* rnorm, void* stream) {
  if (B < 0 || H <= 0 || max_T <= 0) return fail(TQ_ERR_ARG, "tq_quantize_append: bad sizes");
  if (B > 0 && !pos) return fail(TQ_ERR_ARG, "tq_quantize_append: null pos");
  return quantize_common(c, which, x, dtype, (int64_t)B * H, ld, codes, qjl, norm, rnorm, pos, H,
                         max_T, stream, "tq_quantize_append");
}

int tq_quantize_append_paged(tq_ctx* c, int which, const void* x, int dtype, int B, int H,
                             int64_t ld, const int32_t* block_table, int max_blocks, int block_size,
                             int64_t num_blocks, const int32_t* pos, uint32_t* codes, uint32_t* qjl,
                             void* norm, float* rnorm, void* stream) {
  if (B < 0 || H <= 0 || max_blocks <= 0 || block_size <= 0 || num_blocks <= 0)
    return fail(TQ_ERR_ARG, "tq_quantize_append_paged: bad sizes");
  if (B > 0 && (!pos || !block_table)) return fail(TQ_ERR_ARG, "tq_quantize_append_paged: null pos or block_table");
  Paging pg;
  pg.table = block_table;
  pg.max_blocks = max_blocks;
  pg.block_size = block_size;
  pg.num_blocks = num_blocks;
  return quantize_common(c, which, x, dtype, (int64_t)B * H, ld, codes, qjl, norm, rnorm, pos, H,
                         (int64_t)max_blocks * block_size, stream, "tq_quantize_append_paged", pg);
}

int tq_dequantize(tq_ctx* c, int which, const uint32_t* codes, const uint32_t* qjl,
                  const void* norm, const float* rnorm, int64_t n, float* out, void* stream) {
  if (int r = check_ctx_dev(c, "tq_dequantize")) return r;
  if (which != TQ_KEY && which != TQ_VALUE) return fail(TQ_ERR_ARG, "tq_dequantize: bad which=%d", which);
  if (n < 0) return fail(TQ_ERR_ARG, "tq_dequantize: n < 0");
  if (n == 0) return TQ_OK;
  if (!codes || !norm || !out) return fail(TQ_ERR_ARG, "tq_dequantize: null pointer");
  if (which == TQ_KEY && c->qjl_m > 0 && (!qjl || !rnorm))
    return fail(TQ_ERR_ARG, "tq_dequantize: keys with QJL need qjl and rnorm");
  cudaError_t e = tqk::launch_dequant(c, which, codes, qjl, static_cast<const float*>(norm), rnorm, n, out, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "tq_dequantize");
  return TQ_OK;
}

int tq_logits(tq_ctx* c, const void* q, int dtype, int64_t nq, const uint32_t* kcodes,
              const uint32_t* kqjl, const void* knorm, const float* krnorm, int64_t nk, float* out,
              void* stream) {
  if (int r = check_ctx_dev(c, "tq_logits")) return r;
  if (dtype != TQ_F32 && dtype != TQ_BF16 && dtype != TQ_F16)
    return fail(TQ_ERR_ARG, "tq_logits: bad dtype=%d", dtype);
  if (nq < 0 || nk < 0) return fail(TQ_ERR_ARG, "tq_logits: negative size");
  if (nq == 0 || nk == 0) return TQ_OK;
  if (!q || !kcodes || !knorm || !out) return fail(TQ_ERR_ARG, "tq_logits: null pointer");
  if (c->qjl_m > 0 && (!kqjl || !krnorm)) return fail(TQ_ERR_ARG, "tq_logits: keys with QJL need kqjl and krnorm");
  if (nq > 65535LL * 8) return fail(TQ_ERR_UNSUPPORTED, "tq_logits: nq too large");
  cudaError_t e = tqk::launch_logits(c, q, dtype, nq, kcodes, kqjl, static_cast<const float*>(knorm), krnorm, nk, out,
                                     as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "tq_logits");
  return TQ_OK;
}

// Workspace: [q' and S q' rows][tile prefix][step lengths][int8 query-operand
// images, one per (sequence, kv head), sized for B Hq][partials].  The partials are
// sized for the larger of the split layout ([B Hq][splits][dpad + 2]) and
// the segment layouts: [warps + B Hkv][G][dpad + 2] for groups up to 4, and
// [4 (CTAs + B Hkv)][8][dpad + 2] for group 8; both are at most
// [8 warps + 4 B Hq][dpad + 2].
namespace {
struct AttnWs {
  size_t q_bytes, tiles_off, lens_off, qimg_off, part_off, total;
};
AttnWs attn_ws_layout(const tq_ctx* c, int B, int Hq, int64_t max_T) {
  int chunk = 0;
  // Split count depends on Hkv; size for the largest (Hkv = 1 gives the most).
  const int splits = tqk::attn_splits(c, B, 1, max_T > 0 ? max_T : 1, &chunk);
  const size_t rows = (size_t)B * Hq;
  const size_t row_bytes = (size_t)(c->dpad + 2) * sizeof(float);
  const size_t split_part = rows * (size_t)splits * row_bytes;
  const size_t seg_part = ((size_t)tqk::attn_seg_max_warps(c) * 8 + 4 * rows) * row_bytes;
  AttnWs w;
  w.q_bytes = 2 * rows * c->dpad * sizeof(float);
  w.tiles_off = (w.q_bytes + 255) & ~(size_t)255;
  w.lens_off = (w.tiles_off + ((size_t)B + 1) * sizeof(int64_t) + 255) & ~(size_t)255;
  w.qimg_off = (w.lens_off + (size_t)B * sizeof(int32_t) + 255) & ~(size_t)255;
  w.part_off = (w.qimg_off + rows * (size_t)tqk::kQopBytes + 255) & ~(size_t)255;
  w.total = w.part_off + (split_part > seg_part ? split_part : seg_part) + 256;
  return w;
}
}  // namespace

size_t tq_attn_workspace_bytes(const tq_ctx* c, int B, int Hq, int64_t max_T) {
  if (!c || B <= 0 || Hq <= 0 || max_T < 0) return 0;
  return attn_ws_layout(c, B, Hq, max_T).total;
}

static int attn_decode_impl(tq_ctx* c, const void* q, int dtype, int B, int Hq, int Hkv,
                            const uint32_t* kcodes, const uint32_t* kqjl, const void* knorm,
                            const float* krnorm, const uint32_t* vcodes, const void* vnorm,
                            int64_t max_T, const int32_t* seq_lens, float scale, float* out,
                            void* workspace, size_t ws_bytes, void* stream, const Paging& pg,
                            const char* name) {
  if (int r = check_ctx_dev(c, name)) return r;
  if (dtype != TQ_F32 && dtype != TQ_BF16 && dtype != TQ_F16)
    return fail(TQ_ERR_ARG, "%s: bad dtype=%d", name, dtype);
  if (B < 0 || Hq <= 0 || Hkv <= 0 || max_T < 0) return fail(TQ_ERR_ARG, "%s: bad sizes", name);
  if (Hq % Hkv != 0 || Hq / Hkv > 16)
    return fail(TQ_ERR_UNSUPPORTED, "%s: Hq=%d Hkv=%d (need Hq %% Hkv == 0, group <= 16)", name, Hq, Hkv);
  if (B == 0) return TQ_OK;
  if (!q || !kcodes || !knorm || !vcodes || !vnorm || !seq_lens || !out)
    return fail(TQ_ERR_ARG, "%s: null pointer", name);
  if (c->qjl_m > 0 && (!kqjl || !krnorm)) return fail(TQ_ERR_ARG, "%s: keys with QJL need kqjl and krnorm", name);
  if (B > 65535 || Hkv > 65535) return fail(TQ_ERR_UNSUPPORTED, "%s: B or Hkv too large", name);
  const size_t need = tq_attn_workspace_bytes(c, B, Hq, max_T);
  if (!workspace || ws_bytes < need)
    return fail(TQ_ERR_WORKSPACE, "%s: workspace %zu bytes < %zu", name, ws_bytes, need);
  if (!aligned(workspace, 256)) return fail(TQ_ERR_ARG, "%s: workspace not 256-byte aligned", name);
  cudaStream_t s = as_stream(stream);
  const size_t rows = (size_t)B * Hq;
  const AttnWs lay = attn_ws_layout(c, B, Hq, max_T);
  char* p = static_cast<char*>(workspace);
  float* qr = reinterpret_cast<float*>(p);
  float* qs = qr + rows * c->dpad;
  float* part = reinterpret_cast<float*>(p + lay.part_off);
  tqk::AttnArgs a{};
  a.qr = qr;
  a.qs = qs;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = Hq / Hkv;
  a.d = c->d;
  a.bk = c->bk_lm;
  a.bv = c->bits_v;
  a.m = c->qjl_m;
  a.wk = c->wk;
  a.wv = c->wv;
  a.kcodes = kcodes;
  a.kqjl = kqjl;
  a.knorm = static_cast<const float*>(knorm);
  a.krnorm = krnorm;
  a.vcodes = vcodes;
  a.vnorm = static_cast<const float*>(vnorm);
  a.nf16 = c->norm_f16 ? 1 : 0;
  a.max_T = max_T;
  a.seq_lens = seq_lens;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.cq = c->qjl_m > 0 ? (float)(std::sqrt(M_PI / 2.0) / c->qjl_m) : 0.f;
  a.ck = c->ck_f;
  a.cv = c->cv_f;
  a.splits = tqk::attn_splits(c, B, Hkv, max_T > 0 ? max_T : 1, &a.chunk);
  a.part = part;
  a.tiles = nullptr;
  a.block_table = pg.table;
  a.max_blocks = pg.max_blocks;
  a.block_size = pg.block_size;
  a.num_blocks = pg.num_blocks;
  const bool i8 = tqk::attn_i8_supported(c, a) && max_T > 0;
  const bool mma = !i8 && tqk::attn_mma_supported(c, a) && max_T > 0;
  const bool lut = !i8 && !mma && tqk::attn_lut_supported(c, a) && max_T > 0;
  if (pg.table && !(i8 || mma || lut))
    return fail(TQ_ERR_UNSUPPORTED, "%s: paged caches need the tensor-core decode (d = 128, 4-bit values; "
                "2- or 3-bit keys + QJL with m = 128, or MSE-only 3/4/8-bit keys)", name);
  tqk::QopPlan qop{};
  if (i8 || mma || lut) {
    a.tiles = reinterpret_cast<int64_t*>(p + lay.tiles_off);
  } else if (a.splits > 4096) {
    return fail(TQ_ERR_UNSUPPORTED, "%s: too many splits", name);
  }
  if (i8) {
    unsigned char* img = reinterpret_cast<unsigned char*>(p + lay.qimg_off);
    a.qimg = img;
    qop = tqk::attn_i8_qop(c, a, img);
  }
  cudaError_t e = tqk::launch_prerotate(c, q, dtype, (int64_t)rows, a.tiles ? &a : nullptr, qr, qs, s,
                                        i8 ? &qop : nullptr);
  if (e != cudaSuccess) return cuda_fail(e, name);
  e = i8 ? tqk::launch_attn_i8(c, a, out, s)
         : (mma ? tqk::launch_attn_mma(c, a, out, s)
                : (lut ? tqk::launch_attn_lut(c, a, out, s) : tqk::launch_attn(c, a, out, s)));
  if (e != cudaSuccess) return cuda_fail(e, name);
  return TQ_OK;
}

static bool paging_ok(const Paging& pg) {
  return pg.table && pg.max_blocks > 0 && pg.block_size > 0 && pg.block_size % 16 == 0 && pg.num_blocks > 0 &&
         (int64_t)pg.max_blocks * pg.block_size <= (int64_t)1 << 30;
}

int tq_attn_decode(tq_ctx* c, const void* q, int dtype, int B, int Hq, int Hkv,
                   const uint32_t* kcodes, const uint32_t* kqjl, const void* knorm,
                   const float* krnorm, const uint32_t* vcodes, const void* vnorm, int64_t max_T,
                   const int32_t* seq_lens, float scale, float* out, void* workspace,
                   size_t ws_bytes, void* stream) {
  return attn_decode_impl(c, q, dtype, B, Hq, Hkv, kcodes, kqjl, knorm, krnorm, vcodes, vnorm, max_T,
                          seq_lens, scale, out, workspace, ws_bytes, stream, Paging(), "tq_attn_decode");
}

int tq_attn_decode_paged(tq_ctx* c, const void* q, int dtype, int B, int Hq, int Hkv,
                         const uint32_t* kcodes, const uint32_t* kqjl, const void* knorm,
                         const float* krnorm, const uint32_t* vcodes, const void* vnorm,
                         const int32_t* block_table, int max_blocks, int block_size,
                         int64_t num_blocks, const int32_t* seq_lens, float scale, float* out,
                         void* workspace, size_t ws_bytes, void* stream) {
  Paging pg;
  pg.table = block_table;
  pg.max_blocks = max_blocks;
  pg.block_size = block_size;
  pg.num_blocks = num_blocks;
  if (B > 0 && !paging_ok(pg))
    return fail(TQ_ERR_ARG, "tq_attn_decode_paged: bad block table (need block_size %% 16 == 0, "
                "max_blocks, num_blocks > 0)");
  return attn_decode_impl(c, q, dtype, B, Hq, Hkv, kcodes, kqjl, knorm, krnorm, vcodes, vnorm,
                          (int64_t)max_blocks * block_size, seq_lens, scale, out, workspace, ws_bytes,
                          stream, pg, "tq_attn_decode_paged");
}

static int decode_step_impl(tq_ctx* c, const void* q, int q_dtype, const void* k_new,
                            const void* v_new, int kv_dtype, int B, int Hq, int Hkv, uint32_t* kcodes,
                            uint32_t* kqjl, void* knorm, float* krnorm, uint32_t* vcodes,
                            void* vnorm, int64_t max_T, const int32_t* pos, float scale, float* out,
                            void* workspace, size_t ws_bytes, void* stream, const Paging& pg,
                            const char* name) {
  if (int r = check_ctx_dev(c, name)) return r;
  for (int dt : {q_dtype, kv_dtype})
    if (dt != TQ_F32 && dt != TQ_BF16 && dt != TQ_F16) return fail(TQ_ERR_ARG, "%s: bad dtype=%d", name, dt);
  if (B < 0 || Hq <= 0 || Hkv <= 0 || max_T <= 0) return fail(TQ_ERR_ARG, "%s: bad sizes", name);
  if (Hq % Hkv != 0 || Hq / Hkv > 16)
    return fail(TQ_ERR_UNSUPPORTED, "%s: Hq=%d Hkv=%d (need Hq %% Hkv == 0, group <= 16)", name, Hq, Hkv);
  if (B == 0) return TQ_OK;
  if (!q || !k_new || !v_new || !kcodes || !knorm || !vcodes || !vnorm || !pos || !out)
    return fail(TQ_ERR_ARG, "%s: null pointer", name);
  if (c->qjl_m > 0 && (!kqjl || !krnorm)) return fail(TQ_ERR_ARG, "%s: keys with QJL need kqjl and krnorm", name);
  if (B > 65535 || Hkv > 65535) return fail(TQ_ERR_UNSUPPORTED, "%s: B or Hkv too large", name);
  if (!aligned(kcodes, 4) || !aligned(knorm, c->norm_f16 ? 2 : 4) || !aligned(vcodes, 4) ||
      !aligned(vnorm, c->norm_f16 ? 2 : 4))
    return fail(TQ_ERR_ARG, "%s: misaligned cache", name);
  const size_t need = tq_attn_workspace_bytes(c, B, Hq, max_T);
  if (!workspace || ws_bytes < need)
    return fail(TQ_ERR_WORKSPACE, "%s: workspace %zu bytes < %zu", name, ws_bytes, need);
  if (!aligned(workspace, 256)) return fail(TQ_ERR_ARG, "%s: workspace not 256-byte aligned", name);
  cudaStream_t s = as_stream(stream);
  const size_t rows = (size_t)B * Hq;
  const AttnWs lay = attn_ws_layout(c, B, Hq, max_T);
  char* p = static_cast<char*>(workspace);
  float* qr = reinterpret_cast<float*>(p);
  float* qs = qr + rows * c->dpad;
  int32_t* lens = reinterpret_cast<int32_t*>(p + lay.lens_off);

  auto qargs = [&](bool key) {
    tqk::QuantArgs a{};
    a.x = key ? k_new : v_new;
    a.dtype = kv_dtype;
    a.n = (int64_t)B * Hkv;
    a.ld = c->d;
    a.d = c->d;
    a.bits = key ? c->bk_lm : c->bits_v;
    a.nbnd = (1 << a.bits) - 1;
    a.m = key ? c->qjl_m : 0;
    a.nc = (key ? c->nc_k : c->nc_v) ? 1 : 0;
    a.nf16 = c->norm_f16 ? 1 : 0;
    a.words = key ? c->wk : c->wv;
    a.PiT = c->PiT;
    a.ST = c->ST;
    a.cen = key ? c->ck_f : c->cv_f;
    a.bnd = key ? c->bk_f : c->bv_f;
    a.codes = key ? kcodes : vcodes;
    a.qjl = key ? kqjl : nullptr;
    a.norm = static_cast<float*>(key ? knorm : vnorm);
    a.rnorm = key ? krnorm : nullptr;
    a.pos = pos;
    a.H = Hkv;
    a.max_T = max_T;
    a.block_table = pg.table;
    a.max_blocks = pg.max_blocks;
    a.block_size = pg.block_size;
    a.num_blocks = pg.num_blocks;
    return a;
  };
  tqk::AttnArgs a{};
  a.qr = qr;
  a.qs = qs;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = Hq / Hkv;
  a.d = c->d;
  a.bk = c->bk_lm;
  a.bv = c->bits_v;
  a.m = c->qjl_m;
  a.wk = c->wk;
  a.wv = c->wv;
  a.kcodes = kcodes;
  a.kqjl = kqjl;
  a.knorm = static_cast<const float*>(knorm);
  a.krnorm = krnorm;
  a.vcodes = vcodes;
  a.vnorm = static_cast<const float*>(vnorm);
  a.nf16 = c->norm_f16 ? 1 : 0;
  a.max_T = max_T;
  a.seq_lens = lens;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.cq = c->qjl_m > 0 ? (float)(std::sqrt(M_PI / 2.0) / c->qjl_m) : 0.f;
  a.ck = c->ck_f;
  a.cv = c->cv_f;
  a.splits = tqk::attn_splits(c, B, Hkv, max_T, &a.chunk);
  a.part = reinterpret_cast<float*>(p + lay.part_off);
  a.tiles = nullptr;
  a.block_table = pg.table;
  a.max_blocks = pg.max_blocks;
  a.block_size = pg.block_size;
  a.num_blocks = pg.num_blocks;
  const bool i8 = tqk::attn_i8_supported(c, a);
  const bool mma = !i8 && tqk::attn_mma_supported(c, a);
  const bool lut = !i8 && !mma && tqk::attn_lut_supported(c, a);
  if (pg.table && !(i8 || mma || lut))
    return fail(TQ_ERR_UNSUPPORTED, "%s: paged caches need the tensor-core decode", name);
  if (i8 || mma || lut) {
    a.tiles = reinterpret_cast<int64_t*>(p + lay.tiles_off);
  } else if (a.splits > 4096) {
    return fail(TQ_ERR_UNSUPPORTED, "%s: too many splits", name);
  }
  if (i8) a.qimg = reinterpret_cast<unsigned char*>(p + lay.qimg_off);
  tqk::StepPrep sp{};
  sp.k = qargs(true);
  sp.v = qargs(false);
  sp.q = q;
  sp.qdtype = q_dtype;
  sp.qrows = (int64_t)rows;
  sp.qr = qr;
  sp.qs = qs;
  sp.pos = pos;
  sp.lens = lens;
  sp.B = B;
  sp.Hkv = Hkv;
  sp.max_T = max_T;
  sp.tiles = a.tiles;
  sp.nkv = (int64_t)B * Hkv;
  sp.qop = i8 ? tqk::attn_i8_qop(c, a, const_cast<unsigned char*>(a.qimg)) : tqk::QopPlan{};
  cudaError_t e = tqk::launch_step_prep(c, sp, s);
  if (e != cudaSuccess) return cuda_fail(e, name);
  e = i8 ? tqk::launch_attn_i8(c, a, out, s)
         : (mma ? tqk::launch_attn_mma(c, a, out, s)
                : (lut ? tqk::launch_attn_lut(c, a, out, s) : tqk::launch_attn(c, a, out, s)));
  if (e != cudaSuccess) return cuda_fail(e, name);
  return TQ_OK;
}

int tq_decode_step(tq_ctx* c, const void* q, int q_dtype, const void* k_new, const void* v_new,
                   int kv_dtype, int B, int Hq, int Hkv, uint32_t* kcodes, uint32_t* kqjl,
                   void* knorm, float* krnorm, uint32_t* vcodes, void* vnorm, int64_t max_T,
                   const int32_t* pos, float scale, float* out, void* workspace, size_t ws_bytes,
                   void* stream) {
  return decode_step_impl(c, q, q_dtype, k_new, v_new, kv_dtype, B, Hq, Hkv, kcodes, kqjl, knorm, krnorm,
                          vcodes, vnorm, max_T, pos, scale, out, workspace, ws_bytes, stream, Paging(),
                          "tq_decode_step");
}

int tq_decode_step_paged(tq_ctx* c, const void* q, int q_dtype, const void* k_new, const void* v_new,
                         int kv_dtype, int B, int Hq, int Hkv, uint32_t* kcodes, uint32_t* kqjl,
                         void* knorm, float* krnorm, uint32_t* vcodes, void* vnorm,
                         const int32_t* block_table, int max_blocks, int block_size,
                         int64_t num_blocks, const int32_t* pos, float scale, float* out,
                         void* workspace, size_t ws_bytes, void* stream) {
  Paging pg;
  pg.table = block_table;
  pg.max_blocks = max_blocks;
  pg.block_size = block_size;
  pg.num_blocks = num_blocks;
  if (B > 0 && !paging_ok(pg))
    return fail(TQ_ERR_ARG, "tq_decode_step_paged: bad block table (need block_size %% 16 == 0, "
                "max_blocks, num_blocks > 0)");
  return decode_step_impl(c, q, q_dtype, k_new, v_new, kv_dtype, B, Hq, Hkv, kcodes, kqjl, knorm, krnorm,
                          vcodes, vnorm, (int64_t)max_blocks * block_size, pos, scale, out, workspace,
                          ws_bytes, stream, pg, "tq_decode_step_paged");
}

size_t tq_topk_workspace_bytes(const tq_ctx* c, int64_t nq, int64_t n, int k) {
  if (!c || nq < 0 || n < 0 || k < 1 || k > 32) return 0;
  return tqk::topk_workspace(c, nq, n, k);
}

int tq_topk(tq_ctx* c, const void* q, int dtype, int64_t nq, const uint32_t* codes,
            const uint32_t* qjl, const void* norm, const float* rnorm, int64_t n, int k,
            int32_t* idx, float* score, void* workspace, size_t ws_bytes, void* stream) {
  if (int r = check_ctx_dev(c, "tq_topk")) return r;
  if (dtype != TQ_F32 && dtype != TQ_BF16 && dtype != TQ_F16)
    return fail(TQ_ERR_ARG, "tq_topk: bad dtype=%d", dtype);
  if (nq < 0 || n < 0 || k < 1 || k > 32) return fail(TQ_ERR_ARG, "tq_topk: bad sizes (k must be 1..32)");
  if (c->bk_lm > 4) return fail(TQ_ERR_UNSUPPORTED, "tq_topk: keys of %d Lloyd-Max bits (need 1..4)", c->bk_lm);
  if (nq == 0) return TQ_OK;
  if (n > 0x7ffffff0LL) return fail(TQ_ERR_UNSUPPORTED, "tq_topk: n too large");
  if (nq > 65535LL * 16) return fail(TQ_ERR_UNSUPPORTED, "tq_topk: nq too large");
  if (!q || !idx || !score || (n > 0 && (!codes || !norm)))
    return fail(TQ_ERR_ARG, "tq_topk: null pointer");
  if (n > 0 && c->qjl_m > 0 && (!qjl || !rnorm)) return fail(TQ_ERR_ARG, "tq_topk: keys with QJL need qjl and rnorm");
  const size_t need = tq_topk_workspace_bytes(c, nq, n, k);
  if (!workspace || ws_bytes < need)
    return fail(TQ_ERR_WORKSPACE, "tq_topk: workspace %zu bytes < %zu", ws_bytes, need);
  if (!aligned(workspace, 256)) return fail(TQ_ERR_ARG, "tq_topk: workspace not 256-byte aligned");
  cudaError_t e = tqk::launch_topk(c, q, dtype, nq, codes, qjl, static_cast<const float*>(norm), rnorm, n, k, idx, score,
                                   workspace, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "tq_topk");
  return TQ_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode attention without caller-provided scratch.
//
// Some callers cannot allocate device memory on the call path: a plugin whose
// host framework owns every device allocation, or a serving loop that has
// banned allocation after start-up to keep latency flat.  They also may not be
// able to carry a workspace buffer through their interface.  For them the
// scratch of tq_attn_decode lives in this file-scope device array; every GPU
// that loads the library holds it until the process exits.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kStaticScratchBytes = (size_t)32 << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
void* g_static_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  The array's
// name in host code is only a stand-in for the symbol, so the address is
// looked up (once per device, with that device current) and cached.
int static_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "tq_attn_decode_static: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(TQ_ERR_UNSUPPORTED, "tq_attn_decode_static: device %d", dev);
  std::lock_guard<std::mutex> lk(g_static_mu);
  if (!g_static_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "tq_attn_decode_static: cudaGetSymbolAddress");
    g_static_ptr[dev] = p;
  }
  *out = g_static_ptr[dev];
  return TQ_OK;
}

}  // namespace

extern "C" size_t tq_attn_static_scratch_bytes(void) { return kStaticScratchBytes; }

extern "C" int tq_attn_decode_static(tq_ctx* c, const void* q, int dtype, int B, int Hq, int Hkv,
                                     const uint32_t* kcodes, const uint32_t* kqjl,
                                     const void* knorm, const float* krnorm,
                                     const uint32_t* vcodes, const void* vnorm, int64_t max_T,
                                     const int32_t* seq_lens, float scale, float* out,
                                     void* stream) {
  // The scratch address below is the current device's: refuse a context of
  // another device first.
  if (int r = check_ctx_dev(c, "tq_attn_decode_static")) return r;
  const size_t need = tq_attn_workspace_bytes(c, B, Hq, max_T);
  if (need > kStaticScratchBytes)
    return fail(TQ_ERR_WORKSPACE,
                "tq_attn_decode_static: these sizes need %zu bytes of scratch, above the %zu-byte "
                "static limit; use tq_attn_decode with a workspace",
                need, kStaticScratchBytes);
  void* ws = nullptr;
  if (int r = static_scratch(&ws)) return r;
  return tq_attn_decode(c, q, dtype, B, Hq, Hkv, kcodes, kqjl, knorm, krnorm, vcodes, vnorm, max_T,
                        seq_lens, scale, out, ws, kStaticScratchBytes, stream);
}
