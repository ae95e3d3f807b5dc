// C-ABI entry points of liborbitquant (declared in include/orbitquant.h):
// argument checks, the layer object (permutation, codebooks, device tables)
// and dispatch to the kernels.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <new>
#include <string>

#include "oq_internal.h"

namespace oq {

static thread_local std::string g_last_error;

void set_error(const std::string& msg) { g_last_error = msg; }

static oq_status fail(oq_status st, const std::string& msg) {
  set_error(msg);
  return st;
}

static bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

static oq_status cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return OQ_OK;
  return fail(e == cudaErrorMemoryAllocation ? OQ_ERR_NOMEM : OQ_ERR_CUDA,
              std::string(what) + ": " + cudaGetErrorString(e));
}


}  // namespace oq

using namespace oq;

extern "C" {

const char* oq_last_error(void) { return g_last_error.c_str(); }

const char* oq_status_string(oq_status st) {
  switch (st) {
    case OQ_OK: return "ok";
    case OQ_ERR_INVALID_ARG: return "invalid argument";
    case OQ_ERR_UNSUPPORTED: return "unsupported shape or bit width";
    case OQ_ERR_CUDA: return "CUDA error";
    case OQ_ERR_TIMEOUT: return "device wait timed out";
    case OQ_ERR_NOMEM: return "out of memory";
    case OQ_ERR_DEVICE: return "device-side check failed";
  }
  return "unknown status";
}

oq_status oq_codebook_build(int32_t d, int32_t bits, int32_t flags, oq_codebook* out) {
  if (!out) return fail(OQ_ERR_INVALID_ARG, "oq_codebook_build: out is null");
  if (d < 3) return fail(OQ_ERR_INVALID_ARG, "oq_codebook_build: d must be >= 3");
  if (bits < 1 || bits > 8) return fail(OQ_ERR_UNSUPPORTED, "oq_codebook_build: bits must be 1..8");
  return get_codebook(d, bits, flags, out);
}

oq_status oq_rotation_build(int32_t d, uint64_t seed, int32_t flags, uint32_t* perm, int8_t* signs) {
  if (d < 1 || !perm) return fail(OQ_ERR_INVALID_ARG, "oq_rotation_build: d < 1 or perm is null");
  std::vector<uint32_t> p;
  std::vector<int8_t> sg;
  const bool want_signs = (flags & OQ_FLAG_SIGNS) && signs;
  make_permutation(d, seed, p, want_signs ? &sg : nullptr);
  std::memcpy(perm, p.data(), (size_t)d * sizeof(uint32_t));
  if (want_signs) std::memcpy(signs, sg.data(), (size_t)d);
  return OQ_OK;
}

// The fused kernel's producer warps run the block transform of h = 1024 on the
// CUDA cores (oq_rqcc_dev.cuh): beside the tcgen05 contraction, warp MMAs
// would wait behind it.  (The stand-alone kernels keep the warp-MMA transform,
// which is faster on its own.)
constexpr bool kCudaCoreBlockTransform = true;

static oq_status check_shape(int32_t d_in, int32_t d_out, int32_t a_bits, int32_t w_bits) {
  if (d_in <= 0 || d_out <= 0) return fail(OQ_ERR_INVALID_ARG, "dimensions must be positive");
  if (d_in % 32) return fail(OQ_ERR_UNSUPPORTED, "d_in must be a multiple of 32");
  if (d_in > 65535) return fail(OQ_ERR_UNSUPPORTED, "d_in must be < 65536");
  const int h = d_in & -d_in;
  if (h < 32 || h > 4096) return fail(OQ_ERR_UNSUPPORTED, "block size h must be in [32, 4096]");
  if (d_out % 16) return fail(OQ_ERR_UNSUPPORTED, "d_out must be a multiple of 16");
  if (!(a_bits == 2 || a_bits == 3 || a_bits == 4 || a_bits == 8))
    return fail(OQ_ERR_UNSUPPORTED, "a_bits must be 2, 3, 4 or 8");
  if (!(w_bits == 2 || w_bits == 3 || w_bits == 4)) return fail(OQ_ERR_UNSUPPORTED, "w_bits must be 2, 3 or 4");
  return OQ_OK;
}

void oq_layer_destroy(oq_layer* L) {
  if (!L) return;
  io_release(L);
  cudaFree(L->d_gather_a);
  cudaFree(L->d_gather_tc);
  cudaFree(L->d_gather_cc);
  cudaFree(L->d_signmask);
  cudaFree(L->d_levels_a);
  cudaFree(L->d_levels_w);
  cudaFree(L->bins_a.d_codes);
  cudaFree(L->bins_a.d_levels);
  cudaFree(L->bins_w.d_codes);
  cudaFree(L->bins_w.d_levels);
  cudaFree(L->bins_a_full.d_levels);
  cudaFree(L->bins_a_full.d_codes);
  cudaFree(L->d_counters);
  cudaFree(L->d_error);
  delete L;
}

// The AdaLN exception layer (gecl notes Method 5): INT4 weight-only RTN, no
// rotation, no codebooks; bf16 decode tables of the integer levels -7..7.
static oq_status create_int4_layer(int32_t d_in, int32_t d_out, uint64_t seed, int32_t a_bits, int32_t w_bits,
                                   int32_t flags, oq_layer** out) {
  if (flags != OQ_FLAG_WEIGHT_ONLY_INT4)
    return fail(OQ_ERR_INVALID_ARG, "OQ_FLAG_WEIGHT_ONLY_INT4 takes no other flag");
  if (a_bits != 16 || w_bits != 4)
    return fail(OQ_ERR_UNSUPPORTED, "the INT4 weight-only layer takes a_bits = 16, w_bits = 4");
  if (d_in <= 0 || d_out <= 0) return fail(OQ_ERR_INVALID_ARG, "dimensions must be positive");
  if (d_in % 32 || d_out % 128)
    return fail(OQ_ERR_UNSUPPORTED, "the INT4 weight-only layer needs d_in % 32 == 0 and d_out % 128 == 0");
  oq_layer* L = new (std::nothrow) oq_layer();
  if (!L) return fail(OQ_ERR_NOMEM, "host allocation failed");
  L->int4_only = true;
  L->d_in = d_in;
  L->d_out = d_out;
  L->h = d_in & -d_in;
  L->k = d_in / L->h;
  L->a_bits = a_bits;
  L->w_bits = w_bits;
  L->flags = flags;
  L->seed = seed;
  L->a_scale = L->w_scale = 1.0;
  cudaGetDevice(&L->device);
  // bf16 bits of the level of each code (c >= 8: c - 8; c < 8: c - 7)
  for (int c = 0; c < 16; ++c) {
    const float v = (float)(c >= 8 ? c - 8 : c - 7);
    uint32_t u;
    std::memcpy(&u, &v, 4);
    L->lv_w[c] = (uint16_t)(u >> 16);   // exact: small integers
  }
  const size_t cb = (size_t)(d_out / 32) * sizeof(int);
  oq_status st = cuda_check(cudaMalloc(&L->d_counters, cb), "cudaMalloc(split counters)");
  if (st == OQ_OK) st = cuda_check(cudaMemset(L->d_counters, 0, cb), "clear split counters");
  if (st == OQ_OK) st = cuda_check(cudaMalloc(&L->d_error, sizeof(int)), "cudaMalloc(error word)");
  if (st == OQ_OK) st = cuda_check(cudaMemset(L->d_error, 0, sizeof(int)), "clear error word");
  if (st != OQ_OK) {
    oq_layer_destroy(L);
    return st;
  }
  *out = L;
  return OQ_OK;
}

static oq_status not_for_int4(const oq_layer* L, const char* who) {
  return fail(OQ_ERR_UNSUPPORTED, std::string(who) + ": not available on an INT4 weight-only layer");
}

oq_status oq_layer_create(int32_t d_in, int32_t d_out, uint64_t seed, int32_t a_bits, int32_t w_bits,
                          int32_t flags, oq_layer** out) {
  if (!out) return fail(OQ_ERR_INVALID_ARG, "oq_layer_create: out is null");
  *out = nullptr;
  if (flags & OQ_FLAG_WEIGHT_ONLY_INT4) return create_int4_layer(d_in, d_out, seed, a_bits, w_bits, flags, out);
  oq_status st = check_shape(d_in, d_out, a_bits, w_bits);
  if (st != OQ_OK) return st;
  if (flags & ~(OQ_FLAG_SIGNS | OQ_FLAG_GAUSSIAN_MARGINAL | OQ_FLAG_FP8_CONTRACTION))
    return fail(OQ_ERR_INVALID_ARG, "unknown flag bits");
  if ((flags & OQ_FLAG_FP8_CONTRACTION) && (a_bits != 4 || w_bits != 4 || d_out % 256))
    return fail(OQ_ERR_UNSUPPORTED, "the FP8 contraction mode needs a_bits = w_bits = 4 and d_out % 256 == 0");

  oq_layer* L = new (std::nothrow) oq_layer();
  if (!L) return fail(OQ_ERR_NOMEM, "host allocation failed");
  L->d_in = d_in;
  L->d_out = d_out;
  L->h = d_in & -d_in;
  L->k = d_in / L->h;
  L->log_h = 0;
  while ((1 << L->log_h) < L->h) ++L->log_h;
  L->a_bits = a_bits;
  L->w_bits = w_bits;
  L->flags = flags;
  L->seed = seed;
  cudaGetDevice(&L->device);

  if ((st = get_codebook(d_in, a_bits, flags, &L->cb_a)) != OQ_OK ||
      (st = get_codebook(d_in, w_bits, flags, &L->cb_w)) != OQ_OK) {
    delete L;
    return st;
  }
  const bool signed_rot = (flags & OQ_FLAG_SIGNS) != 0;
  make_permutation(d_in, seed, L->perm_host, signed_rot ? &L->signs_host : nullptr);
  std::vector<uint16_t> gather;
  std::vector<uint32_t> signmask;
  rq_build_gather(d_in, L->h, L->perm_host, signed_rot ? &L->signs_host : nullptr, gather, signmask);

  L->a_scale = choose_fp16_scale(L->cb_a);
  L->w_scale = choose_fp16_scale(L->cb_w);
  uint16_t lv_a[256] = {0}, lv_w[256] = {0};
  for (int i = 0; i < (1 << a_bits); ++i) lv_a[i] = f64_to_f16_bits(L->a_scale * L->cb_a.levels[i]);
  for (int i = 0; i < (1 << w_bits); ++i) lv_w[i] = f64_to_f16_bits(L->w_scale * L->cb_w.levels[i]);
  std::memcpy(L->lv_a, lv_a, sizeof(lv_a));
  std::memcpy(L->lv_w, lv_w, sizeof(lv_w));
  if (flags & OQ_FLAG_FP8_CONTRACTION) {
    L->fp8 = true;
    L->a8_scale = choose_fp8_scale(L->cb_a, &L->a8_err);
    L->w8_scale = choose_fp8_scale(L->cb_w, &L->w8_err);
    for (int i = 0; i < 16; ++i) {
      L->lv8_a[i] = f64_to_e4m3_bits(L->a8_scale * L->cb_a.levels[i]);
      L->lv8_w[i] = f64_to_e4m3_bits(L->w8_scale * L->cb_w.levels[i]);
    }
  }
  std::vector<uint32_t> ta_codes, ta_levels, tw_codes, tw_levels;
  if ((st = build_bin_table(L->cb_a, d_in, L->h, lv_a, &L->bins_a.kscale, &L->bins_a.b0, &L->bins_a.nb, ta_codes,
                            ta_levels)) != OQ_OK ||
      (st = build_bin_table(L->cb_w, d_in, L->h, lv_w, &L->bins_w.kscale, &L->bins_w.b0, &L->bins_w.nb, tw_codes,
                            tw_levels)) != OQ_OK) {
    delete L;
    return st;
  }

  // full-range activation table for the tensor-core rotate-quantize kernel
  // (kept in shared memory: at most 2048 bins)
  std::vector<uint32_t> taf_codes, taf_levels;
  bool full_table = false;
  const bool tc_rq = ((L->h == 1024 && d_in / L->h <= 8) || (L->h == 512 && d_in / L->h <= 32)) && !signed_rot;
  if (tc_rq) {
    float kf = 0.f;
    int b0f = 0, nbf = 0;
    const std::string saved = g_last_error;   // a table too large for this use is not an error
    if (build_bin_table(L->cb_a, d_in, L->h, lv_a, &kf, &b0f, &nbf, taf_codes, taf_levels, true) == OQ_OK &&
        nbf <= 2048 && kf == L->bins_a.kscale) {
      full_table = true;
      L->bins_a_full.kscale = kf;
      L->bins_a_full.b0 = b0f;
      L->bins_a_full.nb = nbf;
    }
    g_last_error = saved;
  }

  st = cuda_check(cudaMalloc(&L->d_gather_a, gather.size() * sizeof(uint16_t)), "cudaMalloc(gather)");
  if (st == OQ_OK) st = cuda_check(cudaMemcpy(L->d_gather_a, gather.data(), gather.size() * sizeof(uint16_t),
                                              cudaMemcpyHostToDevice), "upload gather");
  if (st == OQ_OK && tc_rq) {
    std::vector<uint16_t> gather_tc;
    rqtc_build_gather(d_in, L->h, L->perm_host, gather_tc);
    st = cuda_check(cudaMalloc(&L->d_gather_tc, gather_tc.size() * sizeof(uint16_t)), "cudaMalloc(gather)");
    if (st == OQ_OK)
      st = cuda_check(cudaMemcpy(L->d_gather_tc, gather_tc.data(), gather_tc.size() * sizeof(uint16_t),
                                 cudaMemcpyHostToDevice), "upload gather");
    if (st == OQ_OK && L->h == 1024 && kCudaCoreBlockTransform) {
      std::vector<uint16_t> gather_cc;
      rqcc_build_gather(d_in, L->perm_host, gather_cc);
      st = cuda_check(cudaMalloc(&L->d_gather_cc, gather_cc.size() * sizeof(uint16_t)), "cudaMalloc(gather)");
      if (st == OQ_OK)
        st = cuda_check(cudaMemcpy(L->d_gather_cc, gather_cc.data(), gather_cc.size() * sizeof(uint16_t),
                                   cudaMemcpyHostToDevice), "upload gather");
    }
  }
  if (st == OQ_OK && signed_rot) {
    st = cuda_check(cudaMalloc(&L->d_signmask, signmask.size() * sizeof(uint32_t)), "cudaMalloc(signs)");
    if (st == OQ_OK) st = cuda_check(cudaMemcpy(L->d_signmask, signmask.data(), signmask.size() * sizeof(uint32_t),
                                                cudaMemcpyHostToDevice), "upload signs");
  }
  if (st == OQ_OK) st = cuda_check(cudaMalloc(&L->d_levels_a, sizeof(lv_a)), "cudaMalloc(levels)");
  if (st == OQ_OK) st = cuda_check(cudaMemcpy(L->d_levels_a, lv_a, sizeof(lv_a), cudaMemcpyHostToDevice), "upload levels");
  if (st == OQ_OK) st = cuda_check(cudaMalloc(&L->d_levels_w, sizeof(lv_w)), "cudaMalloc(levels)");
  if (st == OQ_OK) st = cuda_check(cudaMemcpy(L->d_levels_w, lv_w, sizeof(lv_w), cudaMemcpyHostToDevice), "upload levels");
  auto upload = [&](uint32_t** dst, const std::vector<uint32_t>& v) {
    if (st == OQ_OK) st = cuda_check(cudaMalloc(dst, v.size() * 4), "cudaMalloc(threshold table)");
    if (st == OQ_OK)
      st = cuda_check(cudaMemcpy(*dst, v.data(), v.size() * 4, cudaMemcpyHostToDevice), "upload threshold table");
  };
  upload(&L->bins_a.d_codes, ta_codes);
  upload(&L->bins_a.d_levels, ta_levels);
  upload(&L->bins_w.d_codes, tw_codes);
  upload(&L->bins_w.d_levels, tw_levels);
  if (full_table) {
    upload(&L->bins_a_full.d_levels, taf_levels);
    upload(&L->bins_a_full.d_codes, taf_codes);
  }
  if (st == OQ_OK && d_out % 128 == 0) {
    const size_t cb = (size_t)(d_out / 32) * sizeof(int);
    st = cuda_check(cudaMalloc(&L->d_counters, cb), "cudaMalloc(split counters)");
    if (st == OQ_OK) st = cuda_check(cudaMemset(L->d_counters, 0, cb), "clear split counters");
  }
  if (st == OQ_OK) st = cuda_check(cudaMalloc(&L->d_error, sizeof(int)), "cudaMalloc(error word)");
  if (st == OQ_OK) st = cuda_check(cudaMemset(L->d_error, 0, sizeof(int)), "clear error word");
  if (st != OQ_OK) {
    oq_layer_destroy(L);
    return st;
  }
  *out = L;
  return OQ_OK;
}

oq_status oq_layer_get_info(const oq_layer* L, oq_layer_info* out) {
  if (!L || !out) return fail(OQ_ERR_INVALID_ARG, "oq_layer_get_info: null argument");
  std::memset(out, 0, sizeof(*out));
  out->d_in = L->d_in;
  out->d_out = L->d_out;
  out->h = L->h;
  out->k = L->k;
  out->a_bits = L->a_bits;
  out->w_bits = L->w_bits;
  out->flags = L->flags;
  out->seed = L->seed;
  out->a_words_per_row = (int64_t)L->d_in * L->a_bits / 32;
  out->w_words_per_row = (int64_t)L->d_in * L->w_bits / 32;
  out->a_scale = L->a_scale;
  out->w_scale = L->w_scale;
  return OQ_OK;
}

oq_status oq_layer_get_perm(const oq_layer* L, uint32_t* perm) {
  if (!L || !perm) return fail(OQ_ERR_INVALID_ARG, "oq_layer_get_perm: null argument");
  if (L->int4_only) return not_for_int4(L, "oq_layer_get_perm");
  std::memcpy(perm, L->perm_host.data(), L->perm_host.size() * sizeof(uint32_t));
  return OQ_OK;
}

static oq_status check_rows_input(const void* x, int32_t dtype, const char* who) {
  if (!x) return fail(OQ_ERR_INVALID_ARG, std::string(who) + ": input is null");
  if (dtype != OQ_DTYPE_BF16 && dtype != OQ_DTYPE_F32)
    return fail(OQ_ERR_INVALID_ARG, std::string(who) + ": dtype must be OQ_DTYPE_BF16 or OQ_DTYPE_F32");
  if (!aligned(x, 16)) return fail(OQ_ERR_INVALID_ARG, std::string(who) + ": input must be 16-byte aligned");
  return OQ_OK;
}

static oq_status rq(const oq_layer* L, const void* x, int32_t dtype, int64_t rows, int bits,
                    const oq_bin_table& bins, uint32_t* codes, float* norms, void* stream) {
  RQArgs a{};
  a.src = x;
  a.src_dtype = dtype;
  a.rows = rows;
  a.d = L->d_in;
  a.h = L->h;
  a.log_h = L->log_h;
  a.bits = bits;
  a.gather = L->d_gather_a;
  a.signmask = L->d_signmask;
  a.bins = bins.d_codes;
  a.nb = bins.nb;
  a.b0 = bins.b0;
  a.kscale = bins.kscale;
  a.codes = codes;
  a.norms = norms;
  a.err = L->d_error;
  // activation rows in bf16 at a block size of 1024 or 512: the tensor-core
  // block transform, writing the packed codes
  if (&bins == &L->bins_a && L->d_gather_tc) {
    a.gather_tc = L->d_gather_tc;
    a.bins_full = L->bins_a_full.d_codes;
    a.nb_full = L->bins_a_full.nb;
    a.b0_full = L->bins_a_full.b0;
    if (rqtc_supported(a)) {
      const oq_status st = rqtc_launch(a, stream);
      if (st != OQ_ERR_UNSUPPORTED) return st;
    }
  }
  return rq_launch(a, stream);
}

oq_status oq_rotate_quantize(const oq_layer* L, const void* x, int32_t x_dtype, int64_t T, uint32_t* codes,
                             float* s, void* stream) {
  if (!L) return fail(OQ_ERR_INVALID_ARG, "oq_rotate_quantize: layer is null");
  if (L->int4_only) return not_for_int4(L, "oq_rotate_quantize");
  if (T < 0) return fail(OQ_ERR_INVALID_ARG, "oq_rotate_quantize: T < 0");
  if (T == 0) return OQ_OK;
  oq_status st = check_rows_input(x, x_dtype, "oq_rotate_quantize");
  if (st != OQ_OK) return st;
  if (!codes || !s || !aligned(codes, 16) || !aligned(s, 4))
    return fail(OQ_ERR_INVALID_ARG, "oq_rotate_quantize: codes (16-byte) / s (4-byte) pointers invalid");
  return rq(L, x, x_dtype, T, L->a_bits, L->bins_a, codes, s, stream);
}

oq_status oq_weight_prepare(const oq_layer* L, const void* W, int32_t W_dtype, uint32_t* Wcodes, float* r,
                            void* stream) {
  if (!L) return fail(OQ_ERR_INVALID_ARG, "oq_weight_prepare: layer is null");
  oq_status st = check_rows_input(W, W_dtype, "oq_weight_prepare");
  if (st != OQ_OK) return st;
  if (!Wcodes || !r || !aligned(Wcodes, 16) || !aligned(r, 4))
    return fail(OQ_ERR_INVALID_ARG, "oq_weight_prepare: Wcodes (16-byte) / r (4-byte) pointers invalid");
  if (L->int4_only) return rtn4_prepare_launch(W, W_dtype, L->d_out, L->d_in, Wcodes, r, stream);
  return rq(L, W, W_dtype, L->d_out, L->w_bits, L->bins_w, Wcodes, r, stream);
}

// The contraction kernels address token rows with 32-bit TMA coordinates.
constexpr int64_t MAX_TOKENS = ((int64_t)1 << 31) - 1024;

static oq_status linear_impl(const oq_layer* L, const uint32_t* codes, const float* s, int64_t T,
                             const uint32_t* Wcodes, const float* r, void* y, bool y_bf16, void* stream,
                             const uint16_t* a_f16 = nullptr) {
  if (T > MAX_TOKENS) return fail(OQ_ERR_UNSUPPORTED, "batch too large: at most 2^31 - 1024 tokens per call");
  GemmArgs g{};
  g.a_codes = codes;
  g.a_f16 = a_f16;
  g.b_codes = Wcodes;
  g.a_scale = s;
  g.b_scale = r;
  g.a_levels = L->d_levels_a;
  g.b_levels = L->d_levels_w;
  g.a_levels_host = L->lv_a;
  g.b_levels_host = L->lv_w;
  g.out_scale = (float)(1.0 / (L->a_scale * L->w_scale));
  if (L->fp8) {
    g.fp8 = true;
    g.a_levels8 = L->lv8_a;
    g.b_levels8 = L->lv8_w;
    g.out_scale = (float)(1.0 / (L->a8_scale * L->w8_scale));
  }
  g.y = y;
  g.y_bf16 = y_bf16;
  g.M = T;
  g.N = L->d_out;
  g.K = L->d_in;
  g.a_bits = L->a_bits;
  g.b_bits = L->w_bits;
  g.err = L->d_error;
  // up to GEMV_MAX_T tokens: the GEMV kernel (weights streamed once, warp
  // MMAs); a few hundred tokens or fewer: the small-batch kernel (weight rows
  // as the MMA's M, split K, its splits added in fp32 in y itself, so fp32 y
  // only); larger batches and bf16 y: the CTA-pair kernel
  if (a_f16 && T <= GEMV_MAX_T && !L->fp8) {
    const oq_status st = gemv_launch(g, stream);
    if (st != OQ_ERR_UNSUPPORTED) return st;
  }
  if (a_f16 && T <= SKINNY_MAX_T && L->d_counters && !y_bf16) {
    const oq_status st = gemm_skinny_launch(g, L->d_counters, stream);
    if (st != OQ_ERR_UNSUPPORTED) return st;
  }
  return gemm_launch(g, stream);
}

// fp32 or bf16 y
static oq_status check_y_dtype(int32_t y_dtype, const char* who) {
  if (y_dtype == OQ_DTYPE_F32 || y_dtype == OQ_DTYPE_BF16) return OQ_OK;
  return fail(OQ_ERR_INVALID_ARG, std::string(who) + ": y_dtype must be OQ_DTYPE_F32 or OQ_DTYPE_BF16");
}

oq_status oq_linear(const oq_layer* L, const uint32_t* codes, const float* s, int64_t T, const uint32_t* Wcodes,
                    const float* r, void* y, int32_t y_dtype, void* stream) {
  if (!L) return fail(OQ_ERR_INVALID_ARG, "oq_linear: layer is null");
  if (L->int4_only) return not_for_int4(L, "oq_linear");
  if (check_y_dtype(y_dtype, "oq_linear") != OQ_OK) return OQ_ERR_INVALID_ARG;
  if (T < 0) return fail(OQ_ERR_INVALID_ARG, "oq_linear: T < 0");
  if (T == 0) return OQ_OK;
  if (!codes || !s || !Wcodes || !r || !y) return fail(OQ_ERR_INVALID_ARG, "oq_linear: null pointer");
  if (!aligned(codes, 16) || !aligned(Wcodes, 16) || !aligned(y, 16) || !aligned(s, 4) || !aligned(r, 16))
    return fail(OQ_ERR_INVALID_ARG, "oq_linear: misaligned pointer");
  return linear_impl(L, codes, s, T, Wcodes, r, y, y_dtype == OQ_DTYPE_BF16, stream);
}

// The fused call has two routes.  With bf16 activations and d_out % 256 == 0
// the rotate-quantize kernel writes the fp16 levels of the codes (the
// contraction's A operand) and the CTA-pair kernel reads them with TMA, so
// only the weight codes are decoded during the contraction.  Otherwise the
// packed codes go through the workspace to the code-decoding contraction.
static bool fused_f16_route(const oq_layer* L, int32_t x_dtype) {
  return x_dtype == OQ_DTYPE_BF16 && L->d_out % 256 == 0 && !L->fp8;
}

static size_t fused_codes_bytes(const oq_layer* L, int64_t T) {
  return (size_t)T * ((size_t)L->d_in * L->a_bits / 32) * 4;
}

static size_t fused_f16_bytes(const oq_layer* L, int64_t T) { return (size_t)T * (size_t)L->d_in * 2; }

static size_t round256(size_t b) { return (b + 255) & ~(size_t)255; }

// Large batches on the fp16-level route decode the weight codes once per call
// into fp16 levels held in the workspace, and both contraction operands come
// by TMA (oq_gemm_w16.cu); this needs 2 d_out d_in more bytes.
static bool fused_w16_route(const oq_layer* L, int32_t x_dtype, int64_t T) {
  return fused_f16_route(L, x_dtype) && T >= W16_MIN_T;
}

static size_t fused_w16_bytes(const oq_layer* L) { return round256((size_t)L->d_out * (size_t)L->d_in * 2); }

// the workspace of the large-batch route: the least workspace, the fused
// kernel's row-group flags, and the decoded weights
static size_t full_workspace(const oq_layer* L, int64_t T, size_t base) {
  return round256(base) + round256(fused_flag_bytes(T)) + fused_w16_bytes(L);
}

// the least workspace oq_linear_fused accepts (without the decoded weights)
static size_t min_workspace(const oq_layer* L, int64_t T) {
  if (!L || T <= 0 || L->int4_only) return 0;
  size_t a = fused_codes_bytes(L, T);
  if (L->d_out % 256 == 0) a = std::max(a, fused_f16_bytes(L, T));
  return round256(a) + (size_t)T * 4;
}

// the workspace of oq_linear_fused_decoded: the least workspace and the flags
static size_t decoded_workspace(const oq_layer* L, int64_t T) {
  return round256(min_workspace(L, T)) + round256(fused_flag_bytes(T));
}

size_t oq_linear_fused_workspace_size(const oq_layer* L, int64_t T) {
  const size_t base = min_workspace(L, T);
  if (base && fused_w16_route(L, OQ_DTYPE_BF16, T)) return full_workspace(L, T, base);
  return base;
}

static RQArgs rq_levels_args(const oq_layer* L, const void* x, int32_t x_dtype, int64_t T, uint16_t* a16,
                             float* s) {
  RQArgs a{};
  a.src = x;
  a.src_dtype = x_dtype;
  a.rows = T;
  a.d = L->d_in;
  a.h = L->h;
  a.log_h = L->log_h;
  a.bits = L->a_bits;
  a.gather = L->d_gather_a;
  a.signmask = L->d_signmask;
  a.bins = L->bins_a.d_levels;
  a.nb = L->bins_a.nb;
  a.b0 = L->bins_a.b0;
  a.kscale = L->bins_a.kscale;
  a.out16 = a16;
  a.norms = s;
  a.err = L->d_error;
  a.gather_tc = L->d_gather_tc;
  a.gather_cc = L->d_gather_cc;
  a.bins_full = L->bins_a_full.d_levels;
  a.nb_full = L->bins_a_full.nb;
  a.b0_full = L->bins_a_full.b0;
  return a;
}

static oq_status rq_levels(const oq_layer* L, const void* x, int32_t x_dtype, int64_t T, uint16_t* a16, float* s,
                           void* stream) {
  const RQArgs a = rq_levels_args(L, x, x_dtype, T, a16, s);
  if (rqtc_supported(a)) {
    const oq_status st = rqtc_launch(a, stream);
    if (st != OQ_ERR_UNSUPPORTED) return st;   // else (shared memory too small): the two-pass kernel
  }
  return rq_launch(a, stream);
}

oq_status oq_rotate_quantize_levels(const oq_layer* L, const void* x, int32_t x_dtype, int64_t T, uint16_t* a16,
                                    float* s, void* stream) {
  if (!L) return fail(OQ_ERR_INVALID_ARG, "oq_rotate_quantize_levels: layer is null");
  if (L->int4_only) return not_for_int4(L, "oq_rotate_quantize_levels");
  if (L->fp8) return fail(OQ_ERR_UNSUPPORTED, "oq_rotate_quantize_levels: the fp16-level route is not used in the FP8 mode");
  if (T < 0) return fail(OQ_ERR_INVALID_ARG, "oq_rotate_quantize_levels: T < 0");
  if (T == 0) return OQ_OK;
  oq_status st = check_rows_input(x, x_dtype, "oq_rotate_quantize_levels");
  if (st != OQ_OK) return st;
  if (x_dtype != OQ_DTYPE_BF16) return fail(OQ_ERR_UNSUPPORTED, "oq_rotate_quantize_levels: bf16 input only");
  if (!a16 || !s || !aligned(a16, 16) || !aligned(s, 4))
    return fail(OQ_ERR_INVALID_ARG, "oq_rotate_quantize_levels: a16 (16-byte) / s (4-byte) pointers invalid");
  return rq_levels(L, x, x_dtype, T, a16, s, stream);
}

oq_status oq_linear_levels(const oq_layer* L, const uint16_t* a16, const float* s, int64_t T, const uint32_t* Wcodes,
                           const float* r, void* y, int32_t y_dtype, void* stream) {
  if (!L) return fail(OQ_ERR_INVALID_ARG, "oq_linear_levels: layer is null");
  if (check_y_dtype(y_dtype, "oq_linear_levels") != OQ_OK) return OQ_ERR_INVALID_ARG;
  if (L->int4_only) return not_for_int4(L, "oq_linear_levels");
  if (L->fp8) return fail(OQ_ERR_UNSUPPORTED, "oq_linear_levels: the fp16-level route is not used in the FP8 mode");
  if (T < 0) return fail(OQ_ERR_INVALID_ARG, "oq_linear_levels: T < 0");
  if (T == 0) return OQ_OK;
  if (!a16 || !s || !Wcodes || !r || !y) return fail(OQ_ERR_INVALID_ARG, "oq_linear_levels: null pointer");
  if (!aligned(a16, 16) || !aligned(Wcodes, 16) || !aligned(y, 16) || !aligned(s, 4) || !aligned(r, 16))
    return fail(OQ_ERR_INVALID_ARG, "oq_linear_levels: misaligned pointer");
  if (L->d_out % 256 != 0) return fail(OQ_ERR_UNSUPPORTED, "oq_linear_levels: needs d_out % 256 == 0");
  return linear_impl(L, nullptr, s, T, Wcodes, r, y, y_dtype == OQ_DTYPE_BF16, stream, a16);
}

oq_status oq_weight_levels(const oq_layer* L, const uint32_t* Wcodes, uint16_t* w16, void* stream) {
  if (!L) return fail(OQ_ERR_INVALID_ARG, "oq_weight_levels: layer is null");
  if (L->int4_only) return not_for_int4(L, "oq_weight_levels");
  if (L->fp8) return fail(OQ_ERR_UNSUPPORTED, "oq_weight_levels: the fp16-level route is not used in the FP8 mode");
  if (!Wcodes || !w16 || !aligned(Wcodes, 16) || !aligned(w16, 16))
    return fail(OQ_ERR_INVALID_ARG, "oq_weight_levels: Wcodes / w16 must be 16-byte aligned device pointers");
  const oq_status st = levels_launch(Wcodes, L->d_out, L->d_in, L->w_bits, L->lv_w, L->d_levels_w, w16, stream);
  return st == OQ_ERR_UNSUPPORTED ? fail(st, "oq_weight_levels: unsupported shape") : st;
}

static GemmArgs w16_args(const oq_layer* L, const uint16_t* a16, const float* s, int64_t T, const uint16_t* w16,
                         const float* r, void* y, bool y_bf16) {
  GemmArgs g{};
  g.a_f16 = a16;
  g.b_f16 = w16;
  g.a_scale = s;
  g.b_scale = r;
  g.out_scale = (float)(1.0 / (L->a_scale * L->w_scale));
  g.y = y;
  g.y_bf16 = y_bf16;
  g.M = T;
  g.N = L->d_out;
  g.K = L->d_in;
  g.a_bits = L->a_bits;
  g.b_bits = L->w_bits;
  g.err = L->d_error;
  return g;
}

static oq_status linear_w16(const oq_layer* L, const uint16_t* a16, const float* s, int64_t T, const uint16_t* w16,
                            const float* r, void* y, bool y_bf16, void* stream) {
  if (T > MAX_TOKENS) return fail(OQ_ERR_UNSUPPORTED, "batch too large: at most 2^31 - 1024 tokens per call");
  const oq_status st = gemm_w16_launch(w16_args(L, a16, s, T, w16, r, y, y_bf16), stream);
  return st == OQ_ERR_UNSUPPORTED ? fail(st, "oq_linear_decoded: unsupported shape") : st;
}

oq_status oq_linear_decoded(const oq_layer* L, const uint16_t* a16, const float* s, int64_t T, const uint16_t* w16,
                            const float* r, void* y, int32_t y_dtype, void* stream) {
  if (!L) return fail(OQ_ERR_INVALID_ARG, "oq_linear_decoded: layer is null");
  if (check_y_dtype(y_dtype, "oq_linear_decoded") != OQ_OK) return OQ_ERR_INVALID_ARG;
  if (L->int4_only) return not_for_int4(L, "oq_linear_decoded");
  if (L->fp8) return fail(OQ_ERR_UNSUPPORTED, "oq_linear_decoded: the fp16-level route is not used in the FP8 mode");
  if (T < 0) return fail(OQ_ERR_INVALID_ARG, "oq_linear_decoded: T < 0");
  if (T == 0) return OQ_OK;
  if (!a16 || !s || !w16 || !r || !y) return fail(OQ_ERR_INVALID_ARG, "oq_linear_decoded: null pointer");
  if (!aligned(a16, 16) || !aligned(w16, 16) || !aligned(y, 16) || !aligned(s, 4) || !aligned(r, 16))
    return fail(OQ_ERR_INVALID_ARG, "oq_linear_decoded: misaligned pointer");
  if (L->d_out % 256 != 0) return fail(OQ_ERR_UNSUPPORTED, "oq_linear_decoded: needs d_out % 256 == 0");
  return linear_w16(L, a16, s, T, w16, r, y, y_dtype == OQ_DTYPE_BF16, stream);
}

// y = x (q r)^T for the INT4 weight-only layer: bf16 x straight into the
// small-batch kernel as its token operand, in launches of up to 256 tokens
static oq_status int4_linear(const oq_layer* L, const void* x, int32_t x_dtype, int64_t T, const uint32_t* Wcodes,
                             const float* r, float* y, void* stream) {
  if (x_dtype != OQ_DTYPE_BF16) return fail(OQ_ERR_UNSUPPORTED, "INT4 weight-only layer: bf16 activations only");
  if (!Wcodes || !r || !y) return fail(OQ_ERR_INVALID_ARG, "oq_linear_fused: null pointer");
  if (!aligned(Wcodes, 16) || !aligned(y, 16) || !aligned(r, 4))
    return fail(OQ_ERR_INVALID_ARG, "oq_linear_fused: misaligned pointer");
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  for (int64_t t0 = 0; t0 < T; t0 += SKINNY_MAX_T) {
    GemmArgs g{};
    g.a_f16 = xb + t0 * L->d_in;
    g.a_bf16 = true;
    g.b_codes = Wcodes;
    g.a_scale = nullptr;
    g.b_scale = r;
    g.b_levels_host = L->lv_w;
    g.out_scale = 1.f;
    g.y = y + t0 * L->d_out;
    g.M = std::min<int64_t>(SKINNY_MAX_T, T - t0);
    g.N = L->d_out;
    g.K = L->d_in;
    g.a_bits = 16;
    g.b_bits = 4;
    g.err = L->d_error;
    const oq_status st = gemm_skinny_launch(g, L->d_counters, stream);
    if (st != OQ_OK) return st == OQ_ERR_UNSUPPORTED ? fail(st, "INT4 weight-only layer: unsupported shape") : st;
  }
  return OQ_OK;
}

// x -> y with the weights' fp16 levels already decoded: the fused kernel
// where it applies, else the rotate-quantize kernel and the decoded-weight
// contraction in turn.  ws: [A operand | norms | row-group flags].
// Wcodes: the weight codes, decoded into w16 here first by the level kernel,
// or null when w16 already holds their levels.
// The fused kernel pays where rotate-quantize is a large share of the layer's
// work: the contraction's work per token row grows with d_out, the producers'
// with d_in.  (Measured: with d_out = d_in, 3-6 % below the two kernels in
// turn; with d_out = 4 d_in, 16 % above them, the producers' warps and shared
// memory slowing a contraction that runs long after they are done.)
static bool fused_kernel_pays(const oq_layer* L) { return L->d_out <= L->d_in; }

static oq_status fused_decoded(const oq_layer* L, const void* x, int32_t x_dtype, int64_t T, const uint32_t* Wcodes,
                               uint16_t* w16, const float* r, void* y, bool y_bf16, unsigned char* ws, void* stream) {
  if (T > MAX_TOKENS) return fail(OQ_ERR_UNSUPPORTED, "batch too large: at most 2^31 - 1024 tokens per call");
  const size_t need = min_workspace(L, T);
  uint16_t* a16 = reinterpret_cast<uint16_t*>(ws);
  float* s = reinterpret_cast<float*>(ws + round256(fused_f16_bytes(L, T)));
  const RQArgs ra = rq_levels_args(L, x, x_dtype, T, a16, s);
  oq_status st = OQ_OK;
  const bool fused = fused_kernel_pays(L) && fused_kernel_supported(ra, L->d_out);
  int* flags = reinterpret_cast<int*>(ws + round256(need));
  // with a weight decode, the fused kernel follows it directly as its
  // programmatic dependent, so its flags are cleared before the decode
  if (fused && Wcodes) {
    st = fused_clear_flags(flags, T, stream);
    if (st != OQ_OK) return st;
  }
  if (Wcodes) {
    st = levels_launch(Wcodes, L->d_out, L->d_in, L->w_bits, L->lv_w, L->d_levels_w, w16, stream);
    if (st != OQ_OK) return st == OQ_ERR_UNSUPPORTED ? fail(st, "oq_linear_fused: unsupported shape") : st;
  }
  if (fused) {
    st = fused_launch(ra, w16_args(L, a16, s, T, w16, r, y, y_bf16), flags, stream, Wcodes != nullptr);
    if (st != OQ_ERR_UNSUPPORTED) return st;
  }
  st = rq_levels(L, x, x_dtype, T, a16, s, stream);
  return st != OQ_OK ? st : linear_w16(L, a16, s, T, w16, r, y, y_bf16, stream);
}

// The fused call's body on checked arguments.  w16_ready: the weights' fp16
// levels, already decoded by the caller (oq_linear_fused_host decodes them
// once for all its chunks), or null.
static oq_status fused_device(const oq_layer* L, const void* x, int32_t x_dtype, int64_t T, const uint32_t* Wcodes,
                              const float* r, void* y, bool y_bf16, unsigned char* ws, size_t workspace_bytes,
                              void* stream, const uint16_t* w16_ready) {
  oq_status st;
  const size_t need = min_workspace(L, T);
  if (fused_f16_route(L, x_dtype)) {
    uint16_t* a16 = reinterpret_cast<uint16_t*>(ws);
    float* s = reinterpret_cast<float*>(ws + round256(fused_f16_bytes(L, T)));
    if (w16_ready)   // the same kernels as the one-call route, weights given
      return fused_decoded(L, x, x_dtype, T, nullptr, const_cast<uint16_t*>(w16_ready), r, y, y_bf16, ws, stream);
    // large batches with room for the decoded weights: decode them once, then
    // contract two fp16 operands -- in the fused kernel, whose producer teams
    // write the A operand while the contraction runs, where it applies;
    // otherwise decode weights inside the contraction
    if (fused_w16_route(L, x_dtype, T) && workspace_bytes >= full_workspace(L, T, need)) {
      // workspace: [A operand | norms | row-group flags | decoded weights]
      uint16_t* w16 = reinterpret_cast<uint16_t*>(ws + decoded_workspace(L, T));
      return fused_decoded(L, x, x_dtype, T, Wcodes, w16, r, y, y_bf16, ws, stream);
    }
    st = rq_levels(L, x, x_dtype, T, a16, s, stream);
    if (st != OQ_OK) return st;
    return linear_impl(L, nullptr, s, T, Wcodes, r, y, y_bf16, stream, a16);
  }
  uint32_t* codes = reinterpret_cast<uint32_t*>(ws);
  float* s = reinterpret_cast<float*>(ws + round256(fused_codes_bytes(L, T)));
  st = rq(L, x, x_dtype, T, L->a_bits, L->bins_a, codes, s, stream);
  if (st != OQ_OK) return st;
  return linear_impl(L, codes, s, T, Wcodes, r, y, y_bf16, stream);
}

static oq_status fused_checks(const oq_layer* L, const void* x, int32_t x_dtype, int64_t T, const uint32_t* Wcodes,
                              const float* r, const void* y, int32_t y_dtype, const void* workspace,
                              const char* who) {
  const std::string w(who);
  if (!L) return fail(OQ_ERR_INVALID_ARG, w + ": layer is null");
  if (T < 0) return fail(OQ_ERR_INVALID_ARG, w + ": T < 0");
  if (T == 0) return OQ_OK;
  oq_status st = check_rows_input(x, x_dtype, who);
  if (st != OQ_OK) return st;
  if ((st = check_y_dtype(y_dtype, who)) != OQ_OK) return st;
  if (L->int4_only) {
    if (y_dtype != OQ_DTYPE_F32) return fail(OQ_ERR_UNSUPPORTED, w + ": the INT4 weight-only layer writes fp32 y");
    return OQ_OK;
  }
  if (!Wcodes || !r || !y || !workspace) return fail(OQ_ERR_INVALID_ARG, w + ": null pointer");
  if (!aligned(Wcodes, 16) || !aligned(y, 16) || !aligned(r, 16) || !aligned(workspace, 256))
    return fail(OQ_ERR_INVALID_ARG, w + ": misaligned pointer (workspace needs 256 bytes)");
  return OQ_OK;
}

oq_status oq_linear_fused(const oq_layer* L, const void* x, int32_t x_dtype, int64_t T, const uint32_t* Wcodes,
                          const float* r, void* y, int32_t y_dtype, void* workspace, size_t workspace_bytes,
                          void* stream) {
  oq_status st = fused_checks(L, x, x_dtype, T, Wcodes, r, y, y_dtype, workspace, "oq_linear_fused");
  if (st != OQ_OK || T == 0) return st;
  if (L->int4_only) return int4_linear(L, x, x_dtype, T, Wcodes, r, static_cast<float*>(y), stream);
  if (workspace_bytes < min_workspace(L, T)) return fail(OQ_ERR_INVALID_ARG, "oq_linear_fused: workspace too small");
  return fused_device(L, x, x_dtype, T, Wcodes, r, y, y_dtype == OQ_DTYPE_BF16,
                      static_cast<unsigned char*>(workspace), workspace_bytes, stream, nullptr);
}

size_t oq_linear_fused_decoded_workspace_size(const oq_layer* L, int64_t T) {
  if (!L || T <= 0 || L->int4_only || L->fp8 || L->d_out % 256) return 0;
  return decoded_workspace(L, T);
}

oq_status oq_linear_fused_decoded(const oq_layer* L, const void* x, int32_t x_dtype, int64_t T, const uint16_t* w16,
                                  const float* r, void* y, int32_t y_dtype, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  const char* who = "oq_linear_fused_decoded";
  if (!L) return fail(OQ_ERR_INVALID_ARG, "oq_linear_fused_decoded: layer is null");
  if (L->int4_only) return not_for_int4(L, who);
  if (L->fp8) return fail(OQ_ERR_UNSUPPORTED, "oq_linear_fused_decoded: the fp16-level route is not used in the FP8 mode");
  if (L->d_out % 256 != 0) return fail(OQ_ERR_UNSUPPORTED, "oq_linear_fused_decoded: needs d_out % 256 == 0");
  oq_status st = fused_checks(L, x, x_dtype, T, reinterpret_cast<const uint32_t*>(w16), r, y, y_dtype, workspace, who);
  if (st != OQ_OK || T == 0) return st;
  if (x_dtype != OQ_DTYPE_BF16) return fail(OQ_ERR_UNSUPPORTED, "oq_linear_fused_decoded: bf16 input only");
  if (!aligned(w16, 16)) return fail(OQ_ERR_INVALID_ARG, "oq_linear_fused_decoded: w16 must be 16-byte aligned");
  if (workspace_bytes < decoded_workspace(L, T))
    return fail(OQ_ERR_INVALID_ARG, "oq_linear_fused_decoded: workspace too small");
  return fused_decoded(L, x, x_dtype, T, nullptr, const_cast<uint16_t*>(w16), r, y, y_dtype == OQ_DTYPE_BF16,
                       static_cast<unsigned char*>(workspace), stream);
}

oq_status oq_poll_error(const oq_layer* L) {
  if (!L) return fail(OQ_ERR_INVALID_ARG, "oq_poll_error: layer is null");
  oq_status st = cuda_check(cudaDeviceSynchronize(), "oq_poll_error: synchronize");
  if (st != OQ_OK) return st;
  int word = 0;
  st = cuda_check(cudaMemcpy(&word, L->d_error, sizeof(int), cudaMemcpyDeviceToHost), "oq_poll_error: read");
  if (st != OQ_OK) return st;
  if (word) cudaMemset(L->d_error, 0, sizeof(int));
  // a timed-out small-batch call can leave split counters mid-way
  if ((word & OQ_DEVERR_TIMEOUT) && L->d_counters) cudaMemset(L->d_counters, 0, (size_t)(L->d_out / 32) * sizeof(int));
  if (word & OQ_DEVERR_TIMEOUT) return fail(OQ_ERR_TIMEOUT, "a kernel's bounded wait ran out");
  if (word) return fail(OQ_ERR_DEVICE, "unknown bits in the device error word");
  return OQ_OK;
}

oq_status oq_check_wait_timeout(const oq_layer* L, uint32_t limit_us, void* stream) {
  if (!L) return fail(OQ_ERR_INVALID_ARG, "oq_check_wait_timeout: layer is null");
  if (limit_us < 1 || limit_us > 1000000)
    return fail(OQ_ERR_INVALID_ARG, "oq_check_wait_timeout: limit must be 1 .. 1000000 microseconds");
  return wait_timeout_launch(L->d_error, (uint64_t)limit_us * 1000u, stream);
}

}  // extern "C"

namespace oq {
size_t fused_min_workspace(const oq_layer* L, int64_t T) { return min_workspace(L, T); }
size_t fused_w16_workspace(const oq_layer* L, int64_t T) { return full_workspace(L, T, min_workspace(L, T)); }
size_t fused_decoded_min_workspace(const oq_layer* L, int64_t T) { return decoded_workspace(L, T); }
bool fused_decodes_weights(const oq_layer* L, int32_t x_dtype, int64_t T) { return fused_w16_route(L, x_dtype, T); }
oq_status fused_check_args(const oq_layer* L, const void* x, int32_t x_dtype, int64_t T, const uint32_t* Wcodes,
                           const float* r, const void* y, int32_t y_dtype, const void* workspace, const char* who) {
  return fused_checks(L, x, x_dtype, T, Wcodes, r, y, y_dtype, workspace, who);
}
oq_status fused_run(const oq_layer* L, const void* x, int32_t x_dtype, int64_t T, const uint32_t* Wcodes,
                    const float* r, void* y, bool y_bf16, void* ws, size_t ws_bytes, void* stream,
                    const uint16_t* w16_ready) {
  if (L->int4_only) return int4_linear(L, x, x_dtype, T, Wcodes, r, static_cast<float*>(y), stream);
  return fused_device(L, x, x_dtype, T, Wcodes, r, y, y_bf16, static_cast<unsigned char*>(ws), ws_bytes, stream,
                      w16_ready);
}
oq_status decode_weight_levels(const oq_layer* L, const uint32_t* Wcodes, uint16_t* w16, void* stream) {
  return levels_launch(Wcodes, L->d_out, L->d_in, L->w_bits, L->lv_w, L->d_levels_w, w16, stream);
}
}  // namespace oq
