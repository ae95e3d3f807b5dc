/*
 * orbitquant.h -- C ABI of the OrbitQuant quantized linear layer on B200.
 *
 * The method ("OrbitQuant: Data-Agnostic Quantization for Image and Video
 * Diffusion Transformers", arXiv 2607.02461), as described by the web pages
 * cited below:
 *   - per token, split the activation into its norm s and direction x/s
 *     (paper.gecl.asia reading notes, Method 1);
 *   - rotate the direction with the randomized permuted block-Hadamard
 *     (RPBH) rotation R = blockdiag(H_h/sqrt(h)) P_pi, h the largest power of
 *     two dividing d (gecl notes Method 4 and Key Insight; pith.science
 *     Supplementary A);
 *   - code every rotated coordinate with the Lloyd-Max codebook C_{d,b}
 *     designed for the fixed marginal f_d ~ N(0, 1/d) (gecl notes Method 3;
 *     pith Figure 2);
 *   - weight rows get the same rotation, norm split and quantizer offline, so
 *     the rotation cancels inside the layer (hotpaper.ai abstract; gecl notes
 *     Method 2; llmdb.app Mathematical Formulation y = Q_w(W R^-1) Q_a(R x)).
 *   y[t, o] = s_t r_o sum_i C_w[Wc[o, i]] C_a[Xc[t, i]].
 *
 * Conventions for every call below:
 *   - Pointers named "device" must point to CUDA device memory of the current
 *     device, be 16-byte aligned and be contiguous row-major.  The caller owns
 *     them.  The library owns what an oq_layer holds (the permutation and
 *     gather tables, codebook and threshold tables, split-K counters, an error
 *     word, and the copy streams of oq_linear_fused_host), and the fixed
 *     scratch array of oq_linear_fused_static on every GPU that loads it.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously; the return value reports
 *     argument checks and launch errors only.  No call allocates device memory
 *     except oq_layer_create; oq_linear_fused_host creates its layer's two
 *     copy streams and their events on its first call.
 *   - Every wait inside a kernel is bounded (1 s); a wait that runs out sets
 *     the layer's device error word, and the kernel ends without its result.
 *     oq_poll_error reads the word back (OQ_ERR_TIMEOUT).
 *   - Supported shapes: d_in % 32 == 0 with h = (largest power of two dividing
 *     d_in) in [32, 4096]; d_out % 16 == 0; a_bits in {2,3,4,8}; w_bits in
 *     {2,3,4}.  Anything else returns OQ_ERR_UNSUPPORTED.  T = 0 is a no-op.
 *   - Codes are packed per group of 32 consecutive rotated coordinates: the
 *     group is a little-endian bit stream of 32*b bits stored as b uint32
 *     words, low word first; code i of the group sits at bits [i*b, (i+1)*b).
 *     A row of d codes takes d*b/32 words.  Codes are unsigned and ascend with
 *     the level value.
 */
#ifndef ORBITQUANT_H
#define ORBITQUANT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  OQ_OK = 0,
  OQ_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer     */
  OQ_ERR_UNSUPPORTED = 2,   /* shape or bit width outside the supported set  */
  OQ_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed          */
  OQ_ERR_TIMEOUT = 4,       /* a kernel's bounded wait ran out (device word) */
  OQ_ERR_NOMEM = 5,         /* oq_layer_create could not allocate            */
  OQ_ERR_DEVICE = 6         /* the device error word holds a bit this version
                               does not define (reserved)                    */
} oq_status;

/* Element types of x, W and y.  y (the contraction calls' output) is fp32 or
 * bf16 (rounded to nearest even in the epilogue, from the fp32 result). */
enum { OQ_DTYPE_F32 = 0, OQ_DTYPE_BF16 = 1 };

/* Layer / codebook flags. */
enum {
  OQ_FLAG_SIGNS = 1,              /* Rademacher signs D_j before each block
                                     Hadamard (pith Supplementary A);
                                     off by default                          */
  OQ_FLAG_GAUSSIAN_MARGINAL = 2,  /* design the codebook on N(0, 1/d) (pith
                                     Figure 2) instead of the exact sphere
                                     marginal f_d                            */
  OQ_FLAG_WEIGHT_ONLY_INT4 = 4,   /* the AdaLN exception path (gecl notes
                                     Method 5: INT4 weight-only RTN, no
                                     rotation, 16-bit activations); see
                                     oq_layer_create                         */
  OQ_FLAG_FP8_CONTRACTION = 8     /* lower-precision contraction mode: both
                                     operands' 4-bit codes decode to e4m3 and
                                     multiply on kind::f8f6f4 tensor cores
                                     (twice the fp16 rate).  Same codes, but y
                                     carries the e4m3 rounding of the levels
                                     and does not meet the 1e-3 bound of the
                                     default mode; see oq_layer_create       */
};

/*
 * oq_codebook_build -- the Lloyd-Max codebook C_{d,b} (gecl notes Method 3;
 * pith Figure 2: one codebook per input dimension and bit width, built
 * offline without data).  Host-only; needs no GPU.
 *   d      input dimension (>= 3); the marginal is that of one coordinate of
 *          a uniform point on the unit sphere S^{d-1},
 *          f_d(t) = Gamma(d/2)/(sqrt(pi) Gamma((d-1)/2)) (1-t^2)^((d-3)/2),
 *          or N(0, 1/d) with OQ_FLAG_GAUSSIAN_MARGINAL.
 *   bits   1..8; the codebook has L = 2^bits levels.
 *   out    caller-owned; receives ascending levels[0..L), the L-1 midpoint
 *          thresholds, the designed MSE per coordinate (units of the unit-norm
 *          coordinate) and the solver's iteration count.
 * Deterministic.  Results are cached per (d, bits, flags) inside the library.
 * Errors: OQ_ERR_INVALID_ARG for a null `out` or d < 3; OQ_ERR_UNSUPPORTED for
 * bits outside 1..8.
 */
typedef struct {
  int32_t d, bits, flags, iterations;
  double levels[256];
  double thresholds[255];
  double mse;
} oq_codebook;

oq_status oq_codebook_build(int32_t d, int32_t bits, int32_t flags, oq_codebook* out);

/*
 * oq_rotation_build -- the seeded rotation's random parts, host-only (needs no
 * GPU).  The permutation pi of RPBH (gecl notes Method 4; pith Supplementary
 * A, y = P_pi x) as a gather: rotated position i takes input channel perm[i].
 * Drawn with SplitMix64(seed) driving a descending Fisher-Yates shuffle
 * (j = high 64 bits of next() * (i + 1), i = d-1 .. 1); the pages fix no
 * generator.  With OQ_FLAG_SIGNS in `flags` and a non-null `signs`, also the
 * Rademacher signs D_j of pith Supplementary A by rotated position (+1/-1,
 * -1 when bit 63 of the next draw is set), drawn after the shuffle.
 *   perm   caller-owned host array of d entries.
 *   signs  caller-owned host array of d entries, or NULL.
 * Errors: OQ_ERR_INVALID_ARG for d < 1 or a null perm.
 */
oq_status oq_rotation_build(int32_t d, uint64_t seed, int32_t flags, uint32_t* perm, int8_t* signs);

/*
 * oq_layer_create -- a layer's shared rotation and codebooks.  Builds the
 * seeded permutation pi (SplitMix64(seed) driving a descending Fisher-Yates
 * shuffle; the pages fix no generator), optional signs, both codebooks, and
 * uploads the device tables.  Allocates device memory on the current device.
 * `*out` is library-owned; release it with oq_layer_destroy.
 * Errors: OQ_ERR_INVALID_ARG (null out), OQ_ERR_UNSUPPORTED (shape/bits),
 * OQ_ERR_NOMEM / OQ_ERR_CUDA (allocation or upload failed).
 *
 * With OQ_FLAG_WEIGHT_ONLY_INT4 (alone in `flags`) the layer is the AdaLN
 * modulation projection that the pages keep at INT4 weight-only round-to-
 * nearest because a static rotation cannot fold into it (gecl notes Method 5):
 *   a_bits must be 16 and w_bits 4, d_in % 32 == 0, d_out % 128 == 0;
 *   oq_weight_prepare stores per row r_o = max_i |w_oi| / 7 and codes of
 *     q = round-half-even(w / r_o) in [-7, 7] (fp32, IEEE division), in the
 *     4-bit code format (q >= 0 -> q + 8, q < 0 -> q + 7);
 *   oq_linear_fused with bf16 x gives y = x (q r)^T in fp32 (bf16 operands on
 *     the tensor cores, fp32 accumulation); its workspace size is 0;
 *   the rotation and activation-code calls return OQ_ERR_UNSUPPORTED.
 *
 * With OQ_FLAG_FP8_CONTRACTION (combinable with the two codebook/rotation
 * flags) a_bits and w_bits must be 4 and d_out % 256 == 0: the codes and
 * norms are those of the default mode, while oq_linear and oq_linear_fused
 * decode both operands' levels to e4m3 (each codebook scaled so its levels
 * land closest to e4m3 values) and accumulate in fp32.  The fp16-level calls
 * (oq_rotate_quantize_levels, oq_linear_levels) return OQ_ERR_UNSUPPORTED.
 */
typedef struct oq_layer oq_layer;

oq_status oq_layer_create(int32_t d_in, int32_t d_out, uint64_t seed, int32_t a_bits,
                          int32_t w_bits, int32_t flags, oq_layer** out);
void oq_layer_destroy(oq_layer* layer);

typedef struct {
  int32_t d_in, d_out, h, k, a_bits, w_bits, flags, reserved;
  uint64_t seed;
  int64_t a_words_per_row;   /* d_in * a_bits / 32 */
  int64_t w_words_per_row;   /* d_in * w_bits / 32 */
  double a_scale, w_scale;   /* fp16 decode scale of each codebook's levels */
} oq_layer_info;

oq_status oq_layer_get_info(const oq_layer* layer, oq_layer_info* out);

/* Host copy of the permutation as a gather: rotated position i takes input
 * channel perm[i].  `perm` is a caller-owned host array of d_in entries. */
oq_status oq_layer_get_perm(const oq_layer* layer, uint32_t* perm);

/*
 * oq_weight_save / oq_weight_load -- prepared weights on disk, so that the
 * offline step (oq_weight_prepare; hotpaper.ai abstract: the rotation is
 * folded into the weight rows once) need not run again in a later process.
 * The file carries the layer's d_in, d_out, a_bits, w_bits, flags and seed
 * and a hash of both codebooks, then r [d_out] fp32 and Wcodes [d_out,
 * d_in*w_bits/32] uint32 (little-endian, format version 1).
 *   oq_weight_save  copies Wcodes and r (device, from oq_weight_prepare) to
 *                   the host and writes `path` (through a temporary file that
 *                   is renamed into place).  Synchronous.
 *   oq_weight_load  reads `path`, checks every header field against `layer`,
 *                   and copies the weights into Wcodes and r (device,
 *                   caller-owned, the sizes oq_weight_prepare fills).
 *                   Synchronous.
 * Errors: OQ_ERR_INVALID_ARG for a null argument, a file that cannot be
 * opened or written, a file that is not a prepared-weight file, is truncated
 * or was prepared for a layer with other settings or codebooks;
 * OQ_ERR_UNSUPPORTED for an unknown format version; OQ_ERR_CUDA for a failed
 * copy.
 */
oq_status oq_weight_save(const oq_layer* layer, const uint32_t* Wcodes, const float* r, const char* path);
oq_status oq_weight_load(const oq_layer* layer, const char* path, uint32_t* Wcodes, float* r);

/*
 * oq_rotate_quantize -- online activation codec (gecl notes Method 1, 2, 4):
 *   s[t] = ||x[t]||_2,  u = R x[t] / s[t],  codes[t, i] = #{j : t_j < u_i}.
 *   x      device [T, d_in], bf16 (OQ_DTYPE_BF16) or fp32 (OQ_DTYPE_F32).
 *   codes  device [T, d_in*a_bits/32] uint32, packed as described above.
 *   s      device [T] fp32.
 * A token of zeros gets s = 0 and every code = 2^(a_bits-1) - 1.
 */
oq_status oq_rotate_quantize(const oq_layer* layer, const void* x, int32_t x_dtype, int64_t T,
                             uint32_t* codes, float* s, void* stream);

/*
 * oq_weight_prepare -- offline weight rows (hotpaper.ai abstract: the same
 * quantizer extended to weight rows, rotation absorbed; gecl notes Method 2):
 *   r[o] = ||W[o]||_2, Wcodes[o] = codes of R W[o] / r[o] with the weight
 *   codebook C_{d_in, w_bits}.
 *   W       device [d_out, d_in], fp32 or bf16.
 *   Wcodes  device [d_out, d_in*w_bits/32] uint32.
 *   r       device [d_out] fp32.
 */
oq_status oq_weight_prepare(const oq_layer* layer, const void* W, int32_t W_dtype,
                            uint32_t* Wcodes, float* r, void* stream);

/*
 * oq_linear -- codebook contraction in the shared rotated basis with the
 * magnitudes restored (llmdb.app Mathematical Formulation; gecl notes
 * Method 1-2; pith Figure 2):
 *   y[t, o] = s[t] r[o] sum_i C_w[Wcodes[o, i]] C_a[codes[t, i]]
 *   codes, s   from oq_rotate_quantize; Wcodes, r from oq_weight_prepare.
 *   y          device [T, d_out], fp32 (y_dtype OQ_DTYPE_F32) or bf16
 *              (OQ_DTYPE_BF16: the fp32 result rounded to nearest even).
 * Runs on the tcgen05 tensor cores: both operands are decoded to fp16 levels
 * (scaled per codebook for exact-as-possible fp16 values), accumulated in
 * fp32 in tensor memory, and rescaled in the epilogue.
 */
oq_status oq_linear(const oq_layer* layer, const uint32_t* codes, const float* s, int64_t T,
                    const uint32_t* Wcodes, const float* r, void* y, int32_t y_dtype, void* stream);

/*
 * oq_linear_fused -- x -> y in one call: the rotate-quantize step produces
 * the A operand of the contraction.  With bf16 x and d_out % 256 == 0 the
 * rotate-quantize kernel writes the fp16 levels of the activation codes (as
 * oq_rotate_quantize_levels), which the contraction reads with TMA (only the
 * weight codes are decoded in the contraction); otherwise the packed codes of
 * oq_rotate_quantize pass through the workspace and y is that of oq_linear
 * (bit for bit).  `workspace` is
 * caller-owned device scratch, 256-byte aligned, that may be reused between
 * calls on one stream.  oq_linear_fused_workspace_size(layer, T) gives the
 * bytes of the fastest route: the A operand and the norms, and from 1024
 * tokens on (bf16 x, d_out % 256 == 0) also 2 d_out d_in bytes for the
 * weights' fp16 levels, which are then decoded once per call
 * (oq_weight_levels), and about T bytes of row-group flags.  That route
 * contracts the two fp16 operands on CTA pairs; where the block size is 1024
 * or 512 (at most 12 warps per token row) and d_out <= d_in one kernel does
 * both steps, its rotate-quantize warps writing the A operand while the
 * contraction of earlier tiles runs (it is launched as a programmatic
 * dependent of the weight decode, whose output only its TMA warp waits for),
 * otherwise oq_rotate_quantize_levels' kernel and oq_linear_decoded's kernel
 * run in turn.  A
 * smaller workspace that still holds the A operand and the norms (the least
 * size: 2 T d_in bytes rounded up to a multiple of 256, plus 4 T, on the
 * fp16-level route) is accepted and decodes the weights inside the
 * contraction instead; the y values are the same up to fp32 summation
 * order.  On the fp16-level route the workspace starts with the A operand
 * (fp16 levels [T, d_in] as oq_rotate_quantize_levels writes them, 2 T d_in
 * bytes rounded up to a multiple of 256) followed by the norms s [T] fp32:
 * after the call they hold the codes' levels and norms that gave y.  Where
 * the fused kernel runs with the block transform on the CUDA cores (h =
 * 1024), its fp32 rounding differs from oq_rotate_quantize_levels', so a code
 * may differ from that call's where the coordinate lies within rounding of a
 * decision threshold, and s in the last bits; y is then oq_linear_decoded's
 * on the workspace's operands, bit for bit.  Errors: OQ_ERR_INVALID_ARG when
 * the workspace is below that least size.
 */
size_t oq_linear_fused_workspace_size(const oq_layer* layer, int64_t T);
oq_status oq_linear_fused(const oq_layer* layer, const void* x, int32_t x_dtype, int64_t T,
                          const uint32_t* Wcodes, const float* r, void* y, int32_t y_dtype,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * The two stages of oq_linear_fused's fp16 route, as separate calls (for
 * callers that schedule or time them separately; pith Figure 2 and gecl notes
 * Method 2: the codes' levels are what the contraction multiplies):
 *
 * oq_rotate_quantize_levels -- oq_rotate_quantize, but instead of packed
 * codes it writes each coordinate's codebook level as the fp16 A operand of
 * the contraction:
 *   a16[t, i] = fp16(a_scale * C_a[code_{t,i}])   (a_scale from
 *               oq_layer_get_info: the per-codebook factor that makes the
 *               levels close to exact in fp16)
 *   x    device [T, d_in] bf16 (OQ_DTYPE_BF16 only, else OQ_ERR_UNSUPPORTED).
 *   a16  device [T, d_in] uint16 (fp16 bits), 16-byte aligned.
 *   s    device [T] fp32 token norms.
 * For h = 1024 (d_in <= 8192) or h = 512 (d_in <= 16384) without
 * OQ_FLAG_SIGNS the block transform runs on the tensor cores (H_h =
 * H_{h/32} (x) H_32 as two passes of warp MMAs, the second on a two-term tf32
 * split of the fp32 intermediate): its fp32 rounding differs
 * from oq_rotate_quantize's, so a code may differ from that call's where the
 * coordinate lies within rounding of a decision threshold, and s may differ
 * in the last bits.  Both meet the same bounds against the exact transform.
 *
 * oq_linear_levels -- oq_linear with the A operand given as those fp16
 * levels (read by TMA; only the weight codes are decoded):
 *   y[t, o] = s[t] r[o] / (a_scale w_scale) sum_i a16[t, i] fp16(w_scale C_w[Wcodes[o, i]])
 *   Needs d_out % 256 == 0 (else OQ_ERR_UNSUPPORTED); y 16-byte aligned,
 *   fp32 or bf16 as y_dtype says.
 *
 * oq_weight_levels -- the weights' operand as fp16 levels, decoded once
 * (gecl notes Limitation 3: the centroid lookup of every code):
 *   w16[o, i] = fp16(w_scale * C_w[Wcodes[o, i]])
 *   Wcodes  device [d_out, d_in*w_bits/32] from oq_weight_prepare, 16-byte aligned.
 *   w16     device [d_out, d_in] uint16 (fp16 bits), 16-byte aligned, caller-owned.
 *   Reads the codes once and writes 2 d_out d_in bytes.
 *
 * oq_linear_decoded -- the contraction of the two fp16 level operands, both
 * read by TMA (no decoding in the contraction; the route oq_linear_fused takes
 * for large batches):
 *   y[t, o] = s[t] r[o] / (a_scale w_scale) sum_i a16[t, i] w16[o, i]
 *   a16, s from oq_rotate_quantize_levels; w16 from oq_weight_levels; r from
 *   oq_weight_prepare (16-byte aligned); y device [T, d_out], fp32 or bf16
 *   as y_dtype says, 16-byte aligned.  Needs d_out % 256 == 0 (else
 *   OQ_ERR_UNSUPPORTED).
 *
 * oq_rotate_quantize_levels followed by oq_linear_levels gives exactly the y
 * of oq_linear_fused for T < 1024, and followed by oq_weight_levels +
 * oq_linear_decoded exactly its y for T >= 1024 with the full workspace (and
 * the y of oq_rotate_quantize + oq_linear up to fp32 summation order).
 *
 * Batches of up to 24 tokens (d_out % 16 == 0, d_in % 32 == 0; the batch-1 /
 * GEMV end of the workload sweep) take a kernel that streams the weight codes
 * once, decodes them in registers and multiplies them with warp MMAs; each
 * CTA owns 16 weight rows and adds its warps' partial sums in a fixed order,
 * so results repeat bit for bit, for fp32 and bf16 y alike.  Larger small
 * batches (T <= 256, d_out % 128 == 0) take a kernel whose M dimension is 128
 * weight rows and whose N is the padded batch, with the K range split across
 * the SMs; the splits of a tile add into y in a fixed order through per-layer
 * counters, so results repeat bit for bit, and calls on one layer must not
 * overlap on the GPU (different streams or host threads).  With bf16 y those
 * batches take the CTA-pair kernel instead (the splits add in fp32 in y
 * itself).
 */
/*
 * oq_linear_fused_decoded -- oq_linear_fused with the weights' fp16 levels
 * already decoded (w16 from oq_weight_levels, kept by the caller across
 * calls or decoded just before): the large-batch route of oq_linear_fused
 * without its first step.  Where the block size is 1024 or 512 (at most 12
 * warps per token row) and d_out <= d_in (where rotate-quantize is a share of
 * the work large enough for the overlap to pay) one kernel rotates, quantizes
 * and contracts: its
 * rotate-quantize warps claim groups of 4 token rows from a queue, write
 * their fp16 levels and norms to the workspace and publish each group with a
 * flag, while its contraction warps load a tile's rows as soon as their
 * groups are published (gecl notes Method 2: the codes of R x meet the
 * pre-rotated weight codes in one pass).  Elsewhere the rotate-quantize
 * kernel and oq_linear_decoded's kernel run in turn.  The workspace then holds
 * the A operand and the norms as for oq_linear_fused, and y is that of
 * oq_linear_decoded on them, bit for bit (and that of
 * oq_rotate_quantize_levels + oq_linear_decoded where the transform is the
 * same: every case but h = 1024 inside the fused kernel, see
 * oq_linear_fused).
 *   x          device [T, d_in] bf16 (else OQ_ERR_UNSUPPORTED).
 *   w16        device [d_out, d_in] fp16 levels, 16-byte aligned.
 *   r          device [d_out] fp32, 16-byte aligned.
 *   y          device [T, d_out], fp32 or bf16 as y_dtype says.
 *   workspace  device scratch of oq_linear_fused_decoded_workspace_size(layer,
 *              T) bytes (0 when the call is not available for the layer),
 *              256-byte aligned; reusable between calls on one stream.
 * Needs d_out % 256 == 0.  Calls that share a workspace must not overlap on
 * the GPU.  Errors: as oq_linear_fused.
 */
size_t oq_linear_fused_decoded_workspace_size(const oq_layer* layer, int64_t T);
oq_status oq_linear_fused_decoded(const oq_layer* layer, const void* x, int32_t x_dtype, int64_t T,
                                  const uint16_t* w16, const float* r, void* y, int32_t y_dtype, void* workspace,
                                  size_t workspace_bytes, void* stream);

oq_status oq_rotate_quantize_levels(const oq_layer* layer, const void* x, int32_t x_dtype, int64_t T,
                                    uint16_t* a16, float* s, void* stream);
oq_status oq_linear_levels(const oq_layer* layer, const uint16_t* a16, const float* s, int64_t T,
                           const uint32_t* Wcodes, const float* r, void* y, int32_t y_dtype, void* stream);
oq_status oq_weight_levels(const oq_layer* layer, const uint32_t* Wcodes, uint16_t* w16, void* stream);
oq_status oq_linear_decoded(const oq_layer* layer, const uint16_t* a16, const float* s, int64_t T,
                            const uint16_t* w16, const float* r, void* y, int32_t y_dtype, void* stream);

/*
 * oq_linear_fused_static -- the same computation as oq_linear_fused for
 * callers that cannot allocate device memory: inference runtimes that give
 * plug-ins no allocator, deployments whose device memory is fixed at start-
 * up, loops where an allocation or the synchronisation it implies is not
 * allowed.  (The pages have no counterpart; this is an interface for such
 * callers.)
 *   The scratch that oq_linear_fused takes as `workspace` comes instead from a
 *   fixed array of OQ_STATIC_SCRATCH_BYTES bytes in device memory that the
 *   library reserves on every GPU that loads it, until the process exits.
 *   No call allocates or frees memory.
 *   The first call on each device looks up the array's device address (with
 *   that device current); make that first call before any stream capture.
 *   Every call shares the array: calls that overlap on the GPU (different
 *   streams or host threads) race and give wrong results.
 *   Arguments as for oq_linear_fused, with fp32 y.  The array serves as its least
 *   workspace (the A operand and the norms), so the weights are decoded
 *   inside the contraction at every batch size and y is that of
 *   oq_linear_fused given that least workspace, bit for bit.  Errors:
 *   OQ_ERR_INVALID_ARG when the batch needs more scratch than the array holds
 *   (2 d_in + 4 bytes per token with bf16 x and d_out % 256 == 0: about 2700
 *   tokens at d_in = 3072).
 */
#define OQ_STATIC_SCRATCH_BYTES (16u << 20)
oq_status oq_linear_fused_static(const oq_layer* layer, const void* x, int32_t x_dtype, int64_t T,
                                 const uint32_t* Wcodes, const float* r, float* y, void* stream);

/*
 * oq_linear_fused_host -- oq_linear_fused with x and y in HOST memory (page-
 * locked for the copies to overlap; pageable memory works but serialises
 * them).  The pages have no counterpart; this is the interface for callers
 * whose activations live in host memory.
 *   x_host     host [T, d_in] bf16 (OQ_DTYPE_BF16) or fp32 (OQ_DTYPE_F32).
 *   y_host     host [T, d_out], fp32 or bf16 as y_dtype says.
 *   Wcodes, r  device, from oq_weight_prepare.
 *   workspace  device scratch of oq_linear_fused_host_workspace_size(layer,
 *              x_dtype, T) bytes, 256-byte aligned.
 * The batch runs in chunks of 1024 tokens: the copy of chunk i + 1 into the
 * device, the computation of chunk i (on `stream`) and the copy of chunk i - 1
 * out to the host overlap, on two copy streams that the layer creates on its
 * first such call and keeps until oq_layer_destroy (make that first call before
 * any stream capture).  Work queued on `stream` before the call runs first;
 * work queued after it waits for y to be in host memory (synchronise `stream`
 * before reading y_host).  y is exactly the y of oq_linear_fused on the whole
 * batch.  Calls on one layer must not overlap (they share its copy streams).
 * Errors: as oq_linear_fused; OQ_ERR_UNSUPPORTED on an INT4 weight-only layer.
 */
size_t oq_linear_fused_host_workspace_size(const oq_layer* layer, int32_t x_dtype, int64_t T);
oq_status oq_linear_fused_host(const oq_layer* layer, const void* x_host, int32_t x_dtype, int64_t T,
                               const uint32_t* Wcodes, const float* r, void* y_host, int32_t y_dtype,
                               void* workspace, size_t workspace_bytes, void* stream);

/* Reads and clears the layer's device error word.  Synchronizes the device.
 * Returns OQ_OK or OQ_ERR_TIMEOUT (OQ_ERR_DEVICE for a bit this version does
 * not define). */
oq_status oq_poll_error(const oq_layer* layer);

/*
 * oq_check_wait_timeout -- a self-test of the failure path shared by every
 * kernel (the pages have no counterpart).  Launches one warp that waits, with
 * the library's bounded-wait routine and a bound of `limit_us` microseconds
 * (1 .. 1000000), on an mbarrier that no thread ever arrives on.  The wait runs
 * out, sets the timeout bit of the layer's error word and returns; the kernel
 * ends normally and the CUDA context stays usable.  The next oq_poll_error
 * returns OQ_ERR_TIMEOUT and clears the word.  Asynchronous on `stream`.
 * Errors: OQ_ERR_INVALID_ARG for a null layer or a bound out of range.
 */
oq_status oq_check_wait_timeout(const oq_layer* layer, uint32_t limit_us, void* stream);

/* Message for the last error on the calling thread ("" if none). */
const char* oq_last_error(void);
const char* oq_status_string(oq_status status);

#ifdef __cplusplus
}
#endif

#endif /* ORBITQUANT_H */
