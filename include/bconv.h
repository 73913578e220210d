/*
 * bconv.h -- C ABI of the B200 binary convolution library (libbconv.so).
 *
 * The operation is the binary convolution of the Apple page "MPSCNNBinaryConvolution",
 * Overview:
 *
 *     out[i,x,y,c] = act( (sum_{dx,dy,f} in[i,x+dx,y+dy,f] (op) B[c,dx,dy,f])
 *                         * scale[c] * beta[i,x,y] + bias[c] )
 *
 * with three operators (the MPSCNNBinaryConvolutionType bullets): binaryWeights (input
 * not binarized, weights [0,1] -> {-1,1}), XNOR (input binarized by bin(x) = x<0 ? -1 : 1,
 * each 32-bit word contributes 32 - 2*popcount(x^y)) and AND (same binarization, each word
 * contributes popcount(x&y)); optional input terms applied before binarization and before
 * beta ("inputScaleTerms"/"inputBiasTerms"); and optional beta scaling (the beta and A
 * formulas, enabled by the useBetaScaling flag).  The bfc_* entry points are the
 * fully-connected special case of the page "MPSCNNFullyConnected" (kernel = source size,
 * a 1x1xNo output).
 *
 * Conventions for every entry point:
 *   - Tensors are fp32, NHWC, contiguous.  in[n][y][x][f], out[n][oy][ox][c].
 *   - Packed bits are LSB-first: channel f is bit (f % 32) of word (f / 32); each pixel
 *     (or weight tap) holds ceil(Ni/32) words; bits at or beyond Ni are ignored.
 *     Bit 1 means +1 (XNOR, binaryWeights) or 1 (AND).
 *   - Pointers documented as "host" are read during the call only.  Pointers documented
 *     as "device" must be device memory on the device the handle was created on, are
 *     owned by the caller, and must stay valid until the work on `stream` completes.
 *   - A stream argument is a cudaStream_t (NULL = the legacy default stream).
 *   - Every call returns a status; nothing aborts the process.  Launch failures come back
 *     from the call that launched; device-side failures (an error word the kernels set)
 *     come back from *_sync_status.
 *   - A handle's workspace is used by one stream at a time: forwards on one handle that
 *     overlap on the GPU race.
 */
#ifndef BCONV_H_
#define BCONV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st; /* the type behind cudaStream_t */

/* Status of a call. */
typedef enum {
  BCONV_OK = 0,
  BCONV_ERR_INVALID_ARG = 1, /* NULL where a pointer is required, bad size, bad enum     */
  BCONV_ERR_UNSUPPORTED = 2, /* a valid request this library does not do (groups > 1)  */
  BCONV_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed            */
  BCONV_ERR_OOM = 4,         /* device allocation failed                               */
  BCONV_ERR_TIMEOUT = 5,     /* a kernel gave up a bounded wait and set the error word */
  BCONV_ERR_NO_DEVICE = 6    /* no CUDA device is visible                              */
} bconv_status_t;

/* The convolution operator (MPSCNNBinaryConvolutionType). */
typedef enum {
  BCONV_TYPE_BINARY_WEIGHTS = 0,
  BCONV_TYPE_XNOR = 1,
  BCONV_TYPE_AND = 2
} bconv_type_t;

/* Flags (MPSCNNBinaryConvolutionFlags). */
enum { BCONV_FLAG_NONE = 0u, BCONV_FLAG_USE_BETA_SCALING = 1u };

/* The activation neuron applied last (the closing sentence of the Overview). */
typedef enum { BCONV_NEURON_NONE = 0, BCONV_NEURON_RELU = 1 } bconv_neuron_t;

/* Kernel family used for the contraction.  AUTO picks the fastest one available for the layer. */
typedef enum {
  BCONV_ALGO_AUTO = 0,
  BCONV_ALGO_POPC = 1,     /* XNOR/AND: LOP3 XOR/AND + POPC into int32 registers     */
  BCONV_ALGO_SIMT_F32 = 2, /* binaryWeights: FP32 signed-add contraction on the SIMT */
  BCONV_ALGO_TCGEN05 = 3   /* tcgen05 tensor cores, for out_channels % 4 == 0:
                              XNOR/AND as +-1 / {0,1} int8 codes with int32 accumulation in
                              TMEM (exact, like the POPC family); binaryWeights as three exact
                              bf16 parts of the input against +-1 bf16 weights, fp32
                              accumulation */
} bconv_algo_t;

/*
 * Convolution descriptor.  Output extent: Ho = ceil(in_h/stride_y), Wo = ceil(in_w/stride_x);
 * output (oy, ox) is centred on input (oy*stride_y, ox*stride_x) and its window covers rows
 * dy in [-floor(kernel_h/2), floor((kernel_h-1)/2)] (columns likewise).  Taps outside the
 * image contribute 0.  `groups` must be 1 (the Note on the MPSCNNBinaryConvolution page).
 * `scale_value` is used for every output channel when no scale array is given (the
 * init(device:convolutionData:scaleValue:type:flags:) form).
 */
typedef struct {
  int32_t batch, in_h, in_w, in_channels, out_channels;
  int32_t kernel_h, kernel_w, stride_y, stride_x, groups;
  int32_t neuron; /* bconv_neuron_t */
  float scale_value;
} bconv_desc_t;

typedef struct bconv_handle_s* bconv_handle_t;

/*
 * Create a convolution (MPSCNNBinaryConvolution initializer with outputBiasTerms,
 * outputScaleTerms, inputBiasTerms, inputScaleTerms, type and flags).
 *   desc            host; copied.
 *   packed_weights  host uint32 [out_channels][kernel_h][kernel_w][ceil(in_channels/32)];
 *                   required; copied to the device (bits beyond in_channels are cleared).
 *   scale           host float [out_channels] or NULL (then desc->scale_value for all).
 *   bias            host float [out_channels] or NULL (then 0).
 *   in_scale        host float [in_channels] or NULL (then 1).
 *   in_bias         host float [in_channels] or NULL (then 0).
 *   flags           BCONV_FLAG_* bits; unknown bits are rejected.
 *   out             host; receives the handle.
 * Allocates on the current device every buffer the forward needs (weights, terms and
 * workspace), so forwards never allocate.  Errors: INVALID_ARG, UNSUPPORTED (groups != 1),
 * OOM, CUDA, NO_DEVICE; *out is left NULL on any error.
 */
bconv_status_t bconv_create(const bconv_desc_t* desc, const uint32_t* packed_weights, const float* scale,
                            const float* bias, const float* in_scale, const float* in_bias, bconv_type_t type,
                            uint32_t flags, bconv_handle_t* out);

/*
 * Run the layer: in (device fp32 [batch][in_h][in_w][in_channels]) -> out (device fp32
 * [batch][Ho][Wo][out_channels]).  Asynchronous on `stream`; allocates nothing.
 */
bconv_status_t bconv_forward(bconv_handle_t h, const float* in, float* out, struct CUstream_st* stream);

/*
 * Same as bconv_forward with HOST buffers: copies host_in to the device, runs the layer
 * and copies the result into host_out, then waits for all of it.  Batches of 8 MB or more
 * (input plus output) run as 4 (else 2) image chunks where that divides the batch and keeps
 * 2 MB or more per chunk: a chunk's copy in (on an internal stream), its compute (on
 * `stream`, after the work already queued there) and its copy out (on a second internal
 * stream) overlap with the neighbouring chunks'.  Use page-locked host memory for full copy
 * bandwidth.  The first call on a handle allocates the device staging buffers and the chunk
 * layers (about the layer's own working memory again, plus one more copy of its device
 * weights, which all chunks share) and keeps them until bconv_destroy.
 */
bconv_status_t bconv_forward_host(bconv_handle_t h, const float* host_in, float* host_out,
                                  struct CUstream_st* stream);

/* ------------------------------------------------------------------------------------
 * Chained binary layers.  A binary layer uses its input only through the step before the
 * sum (MPSCNNBinaryConvolution Overview: the input terms act before binarization and
 * before the beta image; bin(x) = x < 0 ? -1 : 1; A of the beta formula): per pixel and
 * channel the sign of x~ = in_scale[c] * x + in_bias[c], and per pixel the mean over the
 * channels of |x~|.  When one binary layer feeds another, the first can therefore emit
 * that form from its epilogue and the second read it in place of fp32 activations: 32x
 * fewer bytes per activation in each direction.  (The pages describe single layers; this
 * form is what the next layer's definition reads of the previous layer's output.)
 *
 * Bit-packed activations of an [N][H][W][C] image:
 *   bits  uint32 [N][H][W][ceil(C/32)]: channel c is bit c % 32 of word c / 32, 1 for
 *         x~ >= 0 (bin = +1) and 0 for x~ < 0; bits past C in a pixel's last word are
 *         written 0 and ignored on input.
 *   a     float [N][H][W]: sum over the C channels of |x~|, divided by C.
 * Signs are decided on x~ in fp32 (x~ = fmaf(y, in_scale, in_bias) of the fp32 output y).
 * ------------------------------------------------------------------------------------ */

/*
 * The input terms of the layer that reads this layer's output: host float [out_channels]
 * each, NULL meaning 1 (scale) or 0 (bias); copied.  Required before a forward with
 * out_bits; may be called again to change them.  Allocates what the bit-packed output
 * needs with the current kernel family (slice partials of A, or an fp32 output buffer
 * for families that binarize in a separate pass; bconv_set_algo may allocate it later).
 * Errors: INVALID_ARG, OOM, CUDA.
 */
bconv_status_t bconv_set_output_terms(bconv_handle_t h, const float* next_in_scale, const float* next_in_bias);

/* Input and output forms of bconv_forward_io: exactly one of in / in_bits and exactly one
 * of out / out_bits is non-NULL.  All pointers are device memory owned by the caller. */
typedef struct {
  const float* in;          /* fp32 [batch][in_h][in_w][in_channels] */
  const uint32_t* in_bits;  /* bit-packed input, in_channels channels */
  const float* in_a;        /* with in_bits: its A [batch][in_h][in_w]; required when the layer uses beta */
  float* out;               /* fp32 [batch][Ho][Wo][out_channels] */
  uint32_t* out_bits;       /* bit-packed output (binarized with the terms of bconv_set_output_terms) */
  float* out_a;             /* with out_bits: its A [batch][Ho][Wo]; required */
} bconv_io_t;

/*
 * bconv_forward with a choice of forms.  Bit-packed input: XNOR and AND layers created
 * without input terms only (the producer applied them): UNSUPPORTED for binaryWeights,
 * INVALID_ARG with input terms.  Bit-packed output: the layer output y (after the neuron)
 * is binarized with the next layer's terms; INVALID_ARG before bconv_set_output_terms.
 * Asynchronous on `stream`; allocates nothing.  When a pixel's output channels are
 * computed by several work items, A is added in a fixed order, so results do not depend
 * on timing.
 */
bconv_status_t bconv_forward_io(bconv_handle_t h, const bconv_io_t* io, struct CUstream_st* stream);

/* Output dimensions (n, Ho, Wo, out_channels).  Any pointer may be NULL. */
bconv_status_t bconv_get_output_dims(bconv_handle_t h, int32_t* n, int32_t* ho, int32_t* wo, int32_t* c);

/* The inputFeatureChannels / outputFeatureChannels properties; -1 for a NULL handle. */
int32_t bconv_input_feature_channels(bconv_handle_t h);
int32_t bconv_output_feature_channels(bconv_handle_t h);

/* Choose the kernel family (BCONV_ALGO_*).  UNSUPPORTED if the family does not do this type. */
bconv_status_t bconv_set_algo(bconv_handle_t h, bconv_algo_t algo);

/* Kernel launches one bconv_forward makes with the current settings. */
int32_t bconv_launches_per_forward(bconv_handle_t h);

/* The kernel family (BCONV_ALGO_*, never AUTO) the next forward will use; -1 for a bad handle. */
int32_t bconv_effective_algo(bconv_handle_t h);

/*
 * How the tensor-core contraction spreads over the SMs, for layers created after the call
 * (process-wide; a layer keeps what it was created with, and its weights are laid out for it).
 *   SINGLE  one CTA per 128-pixel tile on one SM; each weight stage is one bulk copy.
 *   PAIR    a cluster of two CTAs per 256-pixel tile (tcgen05 cta_group::2), each CTA
 *           loading half of every weight stage; an FC needs batch > 128 for it.  XNOR/AND
 *           layers then use int8 codes (see bconv_set_tc_codes).
 *   AUTO    SINGLE for e2m1 codes.  Otherwise PAIR for an FC with batch > 128, and PAIR for a
 *           convolution when the busiest SM of the pair plan runs under 95 % (binaryWeights:
 *           80 %) of the k-block stages of the busiest SM of the one-SM plan (e.g. where the
 *           pairs' balanced split evens out a ragged last wave); otherwise SINGLE.
 * A forced family that the layer or device cannot use falls back to the other one.
 * Returns INVALID_ARG for an unknown mode.
 */
typedef enum { BCONV_CTA_AUTO = 0, BCONV_CTA_SINGLE = 1, BCONV_CTA_PAIR = 2 } bconv_cta_mode_t;
bconv_status_t bconv_set_cta_mode(bconv_cta_mode_t mode);

/* The spread a layer's tensor-core contraction runs with (BCONV_CTA_SINGLE or BCONV_CTA_PAIR);
 * 0 when the layer has no tensor-core path, -1 for a bad handle. */
int32_t bconv_cta_mode(bconv_handle_t h);

/*
 * Operand codes of the XNOR / AND tensor-core contraction, for layers created after the call
 * (process-wide, like bconv_set_cta_mode).
 *   FP4   e2m1 values, two per byte: +-1.0 (XNOR) or 1.0 / 0 (AND), multiplied by
 *         tcgen05.mma kind::mxf4 with unit block scales and summed in fp32 -- exact, since
 *         every product is -1, 0 or 1 and the sums stay below 2^24; half the operand bytes
 *         and twice the MMA rate of INT8; one SM per tile, tiles of up to 128 channels.
 *   INT8  int8 codes, kind::i8, int32 sums (single SMs or pairs).
 *   AUTO  FP4, unless the spread is forced onto SM pairs (then INT8).
 * binaryWeights layers always use three bf16 parts.  Returns INVALID_ARG for an unknown value.
 */
typedef enum { BCONV_CODES_AUTO = 0, BCONV_CODES_INT8 = 1, BCONV_CODES_FP4 = 2, BCONV_CODES_BF16X3 = 3 } bconv_tc_codes_t;
bconv_status_t bconv_set_tc_codes(bconv_tc_codes_t codes);

/* The codes a layer's tensor-core contraction uses (BCONV_CODES_INT8 / FP4 / BF16X3); 0 when
 * the layer has no tensor-core path, -1 for a bad handle. */
int32_t bconv_tc_codes(bconv_handle_t h);

/*
 * How the tensor-core contraction brings the activations into shared memory, for layers
 * created after the call (process-wide, like bconv_set_cta_mode).
 *   PER_TAP  for every tap of the window, a box of the tile's pixels shifted by the tap offset
 *            (each activation code is loaded once per tap); binaryWeights: of the three bf16
 *            parts of x~ that a pack kernel wrote to memory before the contraction.
 *   ROWS     the codes sit in a zero-bordered copy of the image; a tile is 128 consecutive
 *            positions of that grid, and one load of them plus the window's reach serves every
 *            tap (the taps differ only in where their operand starts in shared memory); the
 *            weights of a CTA's output channels stay in shared memory when they fit.  Needs
 *            (kernel_h - 1) * (in_w + kernel_w - 1) + kernel_w - 1 <= 896 and an fp32 output;
 *            a bit-packed output (bconv_set_output_terms) moves the layer to PER_TAP.
 *   INPUT    binaryWeights convolutions: per tap, a box of the fp32 input itself; converting
 *            warps of the contraction form x~ = in_scale * x + in_bias and its three bf16 parts
 *            in shared memory, so no parts buffer is written or read (no pack kernel runs).
 *            Needs no beta, in_c % 4 == 0, at most 128 output channels and an fp32 output; a
 *            bit-packed output (bconv_set_output_terms) moves the layer to PER_TAP.  A forward
 *            whose input is not 16-byte aligned runs on the SIMT family (that call only).
 *   AUTO     ROWS or INPUT where they apply, else PER_TAP.
 * Returns INVALID_ARG for an unknown value.
 */
typedef enum {
  BCONV_STAGING_AUTO = 0,
  BCONV_STAGING_PER_TAP = 1,
  BCONV_STAGING_ROWS = 2,
  BCONV_STAGING_INPUT = 3
} bconv_staging_t;
bconv_status_t bconv_set_staging(bconv_staging_t staging);

/* The staging a layer's tensor-core contraction uses (BCONV_STAGING_PER_TAP, ROWS or INPUT); 0
 * when the layer has no tensor-core path, -1 for a bad handle. */
int32_t bconv_staging(bconv_handle_t h);

/*
 * Wait for `stream`, then read and clear the handle's device error word.  Returns OK,
 * TIMEOUT (a kernel gave up a bounded wait), or CUDA (a pending CUDA error).
 */
bconv_status_t bconv_sync_status(bconv_handle_t h, struct CUstream_st* stream);

/*
 * Timing of the contraction kernel.  After bconv_profile_begin(h, n), each of the next n
 * forwards records a CUDA event pair around its contraction kernel on its own stream;
 * bconv_profile_end waits for the events and returns the summed milliseconds and the
 * number of launches timed, then stops recording.
 */
bconv_status_t bconv_profile_begin(bconv_handle_t h, int32_t max_launches);
bconv_status_t bconv_profile_end(bconv_handle_t h, float* total_ms, int32_t* launches);
/*
 * Called after bconv_profile_begin: time only every `every`-th forward (>= 1; each window
 * starts at 1) of that window, beginning with the next one; max_launches still counts the
 * timed ones.  Each event pair serialises the stream
 * around the timed kernel (several microseconds per forward), so a sparse sample keeps the
 * measurement out of the back-to-back throughput.  INVALID_ARG for every < 1.
 */
bconv_status_t bconv_profile_stride(bconv_handle_t h, int32_t every);

/* Free everything the handle owns (waits for the device first).  NULL is a no-op (OK). */
bconv_status_t bconv_destroy(bconv_handle_t h);

/* ------------------------------------------------------------------------------------
 * Fully-connected special case (MPSCNNFullyConnected Overview and Note): the kernel is
 * the whole source image, the output is 1x1xNo per image, and the result equals the
 * flattened (y, x, f) input vector times an No x (H*W*Ni) weight matrix.  Stride and
 * groups must be 1.  With beta, beta_n = sum over all pixels of A / (H*W).
 * ------------------------------------------------------------------------------------ */
typedef struct {
  int32_t batch, in_h, in_w, in_channels, out_channels;
  int32_t stride_y, stride_x, groups; /* each must be 1 */
  int32_t neuron;                     /* bconv_neuron_t */
  float scale_value;
} bfc_desc_t;

typedef struct bfc_handle_s* bfc_handle_t;

/*
 * packed_weights: host uint32 [out_channels][in_h][in_w][ceil(in_channels/32)].
 * Other arguments and errors as for bconv_create; stride or groups != 1 -> INVALID_ARG
 * and UNSUPPORTED respectively.
 */
bconv_status_t bfc_create(const bfc_desc_t* desc, const uint32_t* packed_weights, const float* scale,
                          const float* bias, const float* in_scale, const float* in_bias, bconv_type_t type,
                          uint32_t flags, bfc_handle_t* out);
/* in: device fp32 [batch][in_h][in_w][in_channels]; out: device fp32 [batch][out_channels]. */
bconv_status_t bfc_forward(bfc_handle_t h, const float* in, float* out, struct CUstream_st* stream);
bconv_status_t bfc_forward_host(bfc_handle_t h, const float* host_in, float* host_out, struct CUstream_st* stream);
/* Chained layers (as bconv_set_output_terms / bconv_forward_io): the bit-packed input is
 * [batch][in_h][in_w][ceil(in_channels/32)] words with A [batch][in_h][in_w] (a binary
 * convolution's bit-packed output); the bit-packed output is [batch][ceil(out_channels/32)]
 * words with A [batch]. */
bconv_status_t bfc_set_output_terms(bfc_handle_t h, const float* next_in_scale, const float* next_in_bias);
bconv_status_t bfc_forward_io(bfc_handle_t h, const bconv_io_t* io, struct CUstream_st* stream);
int32_t bfc_input_feature_channels(bfc_handle_t h);
int32_t bfc_output_feature_channels(bfc_handle_t h);
bconv_status_t bfc_set_algo(bfc_handle_t h, bconv_algo_t algo);
int32_t bfc_launches_per_forward(bfc_handle_t h);
int32_t bfc_effective_algo(bfc_handle_t h);
int32_t bfc_cta_mode(bfc_handle_t h);
int32_t bfc_tc_codes(bfc_handle_t h);
bconv_status_t bfc_sync_status(bfc_handle_t h, struct CUstream_st* stream);
bconv_status_t bfc_profile_begin(bfc_handle_t h, int32_t max_launches);
bconv_status_t bfc_profile_end(bfc_handle_t h, float* total_ms, int32_t* launches);
bconv_status_t bfc_profile_stride(bfc_handle_t h, int32_t every);
bconv_status_t bfc_destroy(bfc_handle_t h);

/* ------------------------------------------------------------------------------------
 * Host helpers
 * ------------------------------------------------------------------------------------ */

/* A short English description of a status. */
const char* bconv_status_string(bconv_status_t s);

/*
 * Pack 0/1 bytes into LSB-first words: bits (host uint8 [rows][nbits], each byte 0 or
 * nonzero) -> out (host uint32 [rows][ceil(nbits/32)]); bit f of a row goes to bit
 * (f % 32) of word (f / 32), unused high bits are 0.  For weights, rows = out_channels *
 * kernel_h * kernel_w and nbits = in_channels.
 */
bconv_status_t bconv_pack_bits(const uint8_t* bits, int64_t rows, int32_t nbits, uint32_t* out);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int32_t bconv_version(void);

/*
 * Measured peak of an instruction the contraction kernels are bound by, on the current
 * device: kind 0 = POPC (32-bit population count, reported as bit-ops/s = 32 x
 * instructions/s), 1 = LOP3 (32-bit logic op, instructions/s x 32), 2 = b1 tensor MMA
 * mma.sync m16n8k256 .xor.popc (bit multiply-accumulates/s), 3 = tcgen05.mma kind::i8
 * M128 N256 K32 from shared memory into TMEM (multiply-accumulates/s), 4 = tcgen05.mma
 * kind::f16 with bf16 operands, M128 N256 K16 (multiply-accumulates/s); kinds 3 and 4 run on
 * zero operands, 5 and 6 are the same on pseudo-random +-1 operands; 7 = tcgen05.mma
 * kind::mxf4 on pseudo-random e2m1 +-1.0 operands with unit block scales, M128 N128 K64
 * (multiply-accumulates/s).  Runs a few short kernels
 * (milliseconds) and waits for them.  *sm_mhz receives the SM clock the kernels saw,
 * derived from clock64() over the event-timed interval (may be NULL).
 */
bconv_status_t bconv_measure_peak(int32_t kind, double* ops_per_s, double* sm_mhz);

/*
 * Check of the failure path every tensor-core kernel relies on (no counterpart on the pages):
 * a kernel waits, with the kernels' own bounded-wait routine, on an mbarrier that nothing
 * completes; after limit_ms (0 < limit_ms <= 1000) it gives up and records a timeout, and the
 * device stays usable.  Returns TIMEOUT when the wait ended as designed, OK if it did not
 * (which would mean the barrier completed), INVALID_ARG, NO_DEVICE or CUDA.
 */
bconv_status_t bconv_check_wait_timeout(double limit_ms);

/* ------------------------------------------------------------------------------------
 * Forward without any allocation.  (The pages have no counterpart to this entry point; it
 * exists for callers of this library that cannot allocate device memory when they run a
 * layer: code whose device memory is all owned by its own pool allocator, or real-time loops
 * where an allocation may stall on a device-wide synchronisation.  Such callers cannot use
 * bconv_create, which allocates the weights and the workspace.)
 * ------------------------------------------------------------------------------------ */

/* Size of the one fixed scratch array this entry point works in (16 MiB).  Every device that
 * loads the library holds it until the process exits. */
#define BCONV_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * XNOR or AND convolution (the same result as bconv_create + bconv_forward with the same
 * arguments), computed with no cudaMalloc, cudaFree or other allocating call.  It runs the
 * SIMT (POPC) kernel family -- a weight-layout kernel, pack, beta, then the XOR/AND + POPC
 * contraction with int32 sums -- not the tensor cores, whose weight layout is prepared on
 * the host at creation: on large layers it is several times slower than a created layer
 * (batch 16, 56x56, 256 -> 256, 3x3: about 8x).
 *   desc            host; as for bconv_create (groups must be 1).
 *   type            BCONV_TYPE_XNOR or BCONV_TYPE_AND (binaryWeights -> INVALID_ARG).
 *   flags           BCONV_FLAG_* bits.
 *   packed_weights  DEVICE uint32 [out_channels][kernel_h][kernel_w][ceil(in_channels/32)],
 *                   LSB-first as for bconv_create; bits beyond in_channels are ignored.
 *   scale, bias     DEVICE float [out_channels] or NULL (desc->scale_value / 0).
 *   in_scale, in_bias DEVICE float [in_channels] or NULL (1 / 0).
 *   in, out         DEVICE fp32 NHWC input and output, as for bconv_forward.
 *   stream          the stream all work is queued on (asynchronous).
 * Working buffers come from the library's fixed scratch array.  Their total is
 *   P*W + T*W*C + No*T*4 [+ P*4 + N*Ho*Wo*4 with beta] [+ 4*No per missing scale/bias]
 *   [+ 4*Ni if exactly one of in_scale/in_bias is given]
 * bytes, each piece rounded up to 256, with P = batch*in_h*in_w, W = 4*round_up(ceil(Ni/32), 8),
 * T = kernel_h*kernel_w, C = round_up(out_channels, 128); a call needing more than
 * BCONV_NOALLOC_SCRATCH_BYTES returns BCONV_ERR_UNSUPPORTED before queuing any work.  Each call
 * rewrites every part of the scratch it reads, so no state carries over from earlier calls,
 * but all calls share the one array: calls whose GPU work can overlap (different streams or
 * host threads without ordering between them) race and corrupt each other's results.
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress, with
 * that device current) and caches it; make that first call before any stream capture begins.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA, NO_DEVICE.
 */
bconv_status_t bconv_forward_noalloc(const bconv_desc_t* desc, bconv_type_t type, uint32_t flags,
                                     const uint32_t* packed_weights, const float* scale, const float* bias,
                                     const float* in_scale, const float* in_bias, const float* in, float* out,
                                     struct CUstream_st* stream);

#ifdef __cplusplus
}
#endif

#endif /* BCONV_H_ */
