// Internal declarations shared by the library's host and device sources.
#pragma once

#include <cstdint>
#include <string>
#include <vector>

#include "orbitquant.h"

// error word bit written by kernels into the layer's device word
#define OQ_DEVERR_TIMEOUT 1

// Threshold search table of one codebook for the rotate-quantize kernel: with
// g = K sqrt(d) u (u the unit-norm rotated coordinate, K a power of two bins
// per unit) every bin [m - 1/2, m + 1/2] holds at most one threshold
// TK_j = K sqrt(d) t_j, so code = base + (g > TK) with (TK, base) of the bin of
// rint(g); bins past the outermost thresholds clamp to the two end bins.
struct oq_bin_table {
  float kscale;        // K sqrt(d / h): g = z * kscale / s for the unnormalised FWHT output z
  int b0, nb;          // bin index = clamp(rint(g) + b0, 0, nb - 1)
  uint32_t* d_codes;   // device [nb] x {TK bits, base code}
  uint32_t* d_levels;  // device [nb] x {TK bits, fp16 level of base | fp16 level of base+1 << 16}
};

struct oq_layer {
  int d_in, d_out, h, k, log_h, a_bits, w_bits, flags;
  bool int4_only;                     // OQ_FLAG_WEIGHT_ONLY_INT4: AdaLN path (no rotation or codebooks)
  bool fp8;                           // OQ_FLAG_FP8_CONTRACTION: levels decoded to e4m3, kind::f8f6f4 MMAs
  double a8_scale, w8_scale;          // e4m3 decode scale per codebook (fp8 mode)
  double a8_err, w8_err;              // their worst relative level rounding
  uint8_t lv8_a[16], lv8_w[16];       // e4m3 bytes of the scaled levels (fp8 mode, 4-bit)
  uint64_t seed;
  int device;
  oq_codebook cb_a, cb_w;
  double a_scale, w_scale;            // fp16 decode scale per codebook
  std::vector<uint32_t> perm_host;    // gather: rotated position i <- channel perm[i]
  std::vector<int8_t> signs_host;     // +-1 by rotated position (OQ_FLAG_SIGNS)
  // device tables (owned)
  uint16_t* d_gather_a;               // rotate-quantize gather offsets, kernel order
  uint16_t* d_gather_tc;              // the same for the tensor-core FWHT kernel (h = 1024 or 512), or null
  uint16_t* d_gather_cc;              // the same for the CUDA-core block kernel (h = 1024), or null
  uint32_t* d_signmask;               // sign bits in kernel order, or null
  uint16_t* d_levels_a;               // fp16 bits of a_scale * activation levels
  uint16_t* d_levels_w;               // fp16 bits of w_scale * weight levels
  uint16_t lv_a[256], lv_w[256];      // host copies of the two level tables
  int* d_error;                       // device error word
  oq_bin_table bins_a, bins_w;       // threshold search tables (activation / weight codebook)
  oq_bin_table bins_a_full;           // activation table over the full range of g (levels only), or d_levels null
  int* d_counters;                    // split-K hand-off counters of the small-batch contraction (zero at rest)
  // host-buffer pipeline (oq_linear_fused_host): two copy streams and their
  // events, created on the first call (opaque CUDA handles)
  void* io_stream[2];
  void* io_event[8];
  bool io_ready;
};

namespace oq {

void set_error(const std::string& msg);

// host math (oq_host.cpp)
void make_permutation(int d, uint64_t seed, std::vector<uint32_t>& perm, std::vector<int8_t>* signs);
oq_status design_codebook(int d, int bits, int flags, oq_codebook* out);
oq_status get_codebook(int d, int bits, int flags, oq_codebook* out);
uint16_t f64_to_f16_bits(double v);
double f16_bits_to_f64(uint16_t h);
double choose_fp16_scale(const oq_codebook& cb);
uint8_t f64_to_e4m3_bits(double v);
double e4m3_bits_to_f64(uint8_t b);
double choose_fp8_scale(const oq_codebook& cb, double* worst);
// threshold search table of a codebook (host copies; words interleaved TK, payload)
constexpr int OQ_MAX_BINS = 4096;
oq_status build_bin_table(const oq_codebook& cb, int d, int h, const uint16_t* lv16, float* kscale, int* b0, int* nb,
                          std::vector<uint32_t>& codes, std::vector<uint32_t>& levels, bool full_range = false);

// rotate + quantize launch (oq_rotate_quantize.cu): rows of `src` -> packed codes + norms
struct RQArgs {
  const void* src;       // [rows, d] bf16 or fp32
  int src_dtype;
  int64_t rows;
  int d, h, log_h, bits;
  const uint16_t* gather;    // per-thread gather offsets (kernel order)
  const uint16_t* gather_tc; // offsets in the tensor-core kernel's order, or null
  const uint16_t* gather_cc; // offsets in the CUDA-core block kernel's order (h = 1024), or null
  const uint32_t* bins_full; // full-range levels table (no clamping needed), or null
  int nb_full, b0_full;
  const uint32_t* signmask;  // or null
  const uint32_t* bins;      // device threshold search table (codes, or levels for out16)
  int nb, b0;
  float kscale;
  uint32_t* codes;           // [rows, d*bits/32], or
  uint16_t* out16;           // fp16 levels [rows, d] (fused layer call); null otherwise
  float* norms;              // [rows]
  int* err;
};
int rq_elems_per_thread(int h);
// kernel-order gather table for a permutation (and optional signs)
void rq_build_gather(int d, int h, const std::vector<uint32_t>& perm, const std::vector<int8_t>* signs,
                     std::vector<uint16_t>& gather, std::vector<uint32_t>& signmask);
oq_status rq_launch(const RQArgs& a, void* stream);
// rotate-quantize with the block FWHT on the tensor cores (h = 1024 or 512,
// bf16 input, fp16-level output, no signs; oq_rotate_quantize_tc.cu)
void rqtc_build_gather(int d, int h, const std::vector<uint32_t>& perm, std::vector<uint16_t>& gather);
// the same for the fused kernel's CUDA-core block transform (h = 1024; oq_fused.cu)
void rqcc_build_gather(int d, const std::vector<uint32_t>& perm, std::vector<uint16_t>& gather);
bool rqtc_supported(const RQArgs& a);
oq_status rqtc_launch(const RQArgs& a, void* stream);

// codebook contraction launch (oq_gemm.cu)
struct GemmArgs {
  const uint32_t* a_codes;   // [M, K*a_bits/32]
  const uint16_t* a_f16;     // or: fp16 levels of A [M, K] (fused call), null otherwise
  bool a_bf16;               // a_f16 holds bf16 values (INT4 weight-only layer; b levels are bf16 too)
  bool fp8;                  // decode both operands to e4m3 and contract with kind::f8f6f4 (4-bit codes)
  const uint8_t* a_levels8;  // host e4m3 level bytes (fp8 mode)
  const uint8_t* b_levels8;
  const uint32_t* b_codes;   // [N, K*b_bits/32]
  const uint16_t* b_f16;     // or: fp16 levels of B [N, K] (decode-then-contract route), null otherwise
  const float* a_scale;      // [M] per-row magnitude s (null: 1)
  const float* b_scale;      // [N] per-row magnitude r
  const uint16_t* a_levels;       // device fp16 bits, 2^a_bits (8-bit table)
  const uint16_t* b_levels;       // device fp16 bits, 2^b_bits
  const uint16_t* a_levels_host;  // host copies (register decode tables)
  const uint16_t* b_levels_host;
  float out_scale;           // 1 / (alpha_a alpha_w)
  void* y;                   // [M, N] fp32, or bf16 with y_bf16
  bool y_bf16;
  int64_t M;
  int N, K, a_bits, b_bits;
  int* err;
};
oq_status gemm_launch(const GemmArgs& g, void* stream);
// paired-CTA contraction (oq_gemm_pair.cu); OQ_ERR_UNSUPPORTED unless N % 256 == 0
oq_status gemm_pair_launch(const GemmArgs& g, void* stream);
// small-batch contraction (oq_gemm_skinny.cu): fp16 A operand, T <= SKINNY_MAX_T,
// N % 128 == 0; `counters` holds N / 32 zeroed ints
constexpr int SKINNY_MAX_T = 256;
// GEMV contraction for up to GEMV_MAX_T tokens (oq_gemv.cu): fp16 A operand,
// weight codes of 2-4 bits decoded in registers, warp MMAs over up to three
// tiles of 8 tokens, no split across CTAs; N % 16 == 0, K % 32 == 0
constexpr int GEMV_MAX_T = 24;
oq_status gemv_launch(const GemmArgs& g, void* stream);
oq_status gemm_skinny_launch(const GemmArgs& g, int* counters, void* stream);
// INT4 weight-only round-to-nearest of weight rows (oq_int4.cu): per-row
// scale max|w| / 7 and 4-bit codes of q in [-7, 7] (q >= 0 -> q + 8, else q + 7)
oq_status rtn4_prepare_launch(const void* W, int w_dtype, int rows, int d, uint32_t* codes, float* scale,
                              void* stream);
// decode-then-contract route (oq_gemm_w16.cu): packed code rows [rows, K] ->
// fp16 levels [rows, K] (K % 32 == 0), and the CTA-pair contraction of two
// fp16 level operands (g.a_f16, g.b_f16; N % 256 == 0, K % 8 == 0)
oq_status levels_launch(const uint32_t* codes, int64_t rows, int K, int bits, const uint16_t* levels_host,
                        const uint16_t* levels_dev, uint16_t* out, void* stream);
oq_status gemm_w16_launch(const GemmArgs& g, void* stream);
// the fused call decodes the weights once per call from this many tokens on
constexpr int64_t W16_MIN_T = 1024;
// the fused layer kernel (oq_fused.cu): rotate-quantize producer teams inside
// the CTA-pair contraction of the decoded weights.  `flags` is workspace of
// fused_flag_bytes(T) bytes, cleared by the launch itself, or, with
// after_levels, by fused_clear_flags before the weight-level kernel that the
// fused kernel then follows directly as its programmatic dependent (its
// producers start while the weights are decoded; its TMA warp waits for them).
bool fused_kernel_supported(const RQArgs& a, int N);
size_t fused_flag_bytes(int64_t T);
oq_status fused_clear_flags(int* flags, int64_t T, void* stream);
oq_status fused_launch(const RQArgs& a, const GemmArgs& g, int* flags, void* stream, bool after_levels = false);
// the fused call's pieces for the host-buffer pipeline (oq_api.cu): the least
// workspace; the workspace with the decoded weights after it; whether the
// fused call decodes the weights once at this batch size; argument checks;
// the call on checked arguments (w16_ready: weights already decoded, or null)
size_t fused_min_workspace(const oq_layer* L, int64_t T);
size_t fused_w16_workspace(const oq_layer* L, int64_t T);
size_t fused_decoded_min_workspace(const oq_layer* L, int64_t T);   // operand, norms and fused-kernel flags
bool fused_decodes_weights(const oq_layer* L, int32_t x_dtype, int64_t T);
oq_status fused_check_args(const oq_layer* L, const void* x, int32_t x_dtype, int64_t T, const uint32_t* Wcodes,
                           const float* r, const void* y, int32_t y_dtype, const void* workspace, const char* who);
oq_status fused_run(const oq_layer* L, const void* x, int32_t x_dtype, int64_t T, const uint32_t* Wcodes,
                    const float* r, void* y, bool y_bf16, void* ws, size_t ws_bytes, void* stream,
                    const uint16_t* w16_ready);
oq_status decode_weight_levels(const oq_layer* L, const uint32_t* Wcodes, uint16_t* w16, void* stream);
// a one-warp kernel whose bounded wait (limit_ns) runs out (oq_diag.cu)
oq_status wait_timeout_launch(int* err, uint64_t limit_ns, void* stream);
// host-buffer pipeline resources of a layer (oq_host_io.cu)
void io_release(oq_layer* L);
// prmt decode tables of a codebook's fp16 levels (oq_gemm.cu)
void make_decode_tables(int bits, const uint16_t* levels, uint32_t* t);

}  // namespace oq
