/*
 * bconv_oracle.c -- TEST INFRASTRUCTURE ONLY (the oracle).
 *
 * A plain, slow, CPU restatement of the binary convolution defined on the Apple
 * documentation page "MPSCNNBinaryConvolution" (Overview: the output formula
 * out = (sum in (op) B) * scale * beta + bias, the sign function bin(), the
 * binaryWeights / XNOR / AND operator bullets, the paragraph on input pre-offset and
 * scaling, the two beta formulas, and the closing sentence on the activation neuron),
 * and of the fully-connected special case on the page "MPSCNNFullyConnected"
 * (Overview: kernel = source size, result = matrix-vector product of the flattened
 * image; Note: equivalent convolution with offset (kW/2, kH/2) and a 1x1 clip).
 *
 * Rules this file keeps:
 *   - one multiply per bit, on +-1 or {0,1} values (or on the full-precision input for
 *     binaryWeights), accumulated in double;
 *   - no bit packing, no popcount, no tiling, no reordering beyond the definition;
 *   - no code shared with the CUDA library, and it includes none of its headers.
 * Only the tests, the smoke check and the bench's CPU-baseline leg may call it.
 *
 * Readings of points the pages leave open (each is listed in the design notes):
 *   - x~ = inScale[f] * x + inBias[f]; the product of two floats is exact in double.
 *   - bin(v) = v < 0 ? -1 : +1, so bin(+-0) = +1.  The sign is decided on x~ rounded to
 *     fp32, the precision the device path computes x~ in (the pages fix none).
 *   - weight bit 1 -> +1 and 0 -> -1 (XNOR, binaryWeights); AND counts positions where
 *     both the input bit and the weight bit are 1.
 *   - window dy in [-floor(kh/2), floor((kh-1)/2)], dx likewise, around the centre
 *     (oy*sy, ox*sx); taps outside the image contribute 0; output size ceil(H/s).
 *   - A[n,y,x] = sum_f |x~| / Ni over the transformed input; beta sums in-image A over
 *     the window and divides by kh*kw.
 *   - the neuron is identity or ReLU, applied after the bias.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_BINARY_WEIGHTS 0
#define ORACLE_XNOR 1
#define ORACLE_AND 2

typedef struct {
  int32_t batch, in_h, in_w, in_channels, out_channels;
  int32_t kernel_h, kernel_w, stride_y, stride_x;
  int32_t type;     /* ORACLE_BINARY_WEIGHTS / ORACLE_XNOR / ORACLE_AND */
  int32_t use_beta; /* useBetaScaling flag */
  int32_t relu;     /* neuron: 0 identity, 1 ReLU */
} oracle_conv_t;

/* Output extent: the output pixel o looks at input centre o*s, so ceil(in/s) of them. */
static int32_t out_extent(int32_t in, int32_t s) { return (in + s - 1) / s; }

/* Input pre-offset and scale ("inputScaleTerms" / "inputBiasTerms"), applied before
 * binarization and before the beta image.  Missing terms mean scale 1 and offset 0. */
static double transformed_input(const float* in, const float* in_scale, const float* in_bias,
                                int64_t pixel, int32_t ni, int32_t f) {
  double x = (double)in[pixel * ni + f];
  double s = in_scale ? (double)in_scale[f] : 1.0;
  double b = in_bias ? (double)in_bias[f] : 0.0;
  return s * x + b;
}

/* bin(x) = x < 0 ? -1 : 1, decided on the fp32 value of x~. */
static double bin_pm1(double xt) { return ((float)xt < 0.0f) ? -1.0 : 1.0; }

/* The same sign as a {0,1} value (AND mode: +1 -> 1, -1 -> 0). */
static double bin_01(double xt) { return ((float)xt < 0.0f) ? 0.0 : 1.0; }

/* One term of the sum over (dx, dy, f): in (op) B, per the operator bullets. */
static double op_term(int32_t type, double xt, uint8_t wbit) {
  if (type == ORACLE_XNOR) return bin_pm1(xt) * (wbit ? 1.0 : -1.0);
  if (type == ORACLE_AND) return bin_01(xt) * (wbit ? 1.0 : 0.0);
  return xt * (wbit ? 1.0 : -1.0); /* binaryWeights: [0,1] -> {-1,1}, input not binarized */
}

/* A[n,y,x] = sum_c |x~[n,y,x,c]| / Nc  (second beta formula). */
static double channel_mean_abs(const float* in, const float* in_scale, const float* in_bias,
                               int64_t pixel, int32_t ni) {
  double acc = 0.0;
  for (int32_t f = 0; f < ni; ++f) acc += fabs(transformed_input(in, in_scale, in_bias, pixel, ni, f));
  return acc / (double)ni;
}

/*
 * Convolution output for a list of output pixels.
 *   in       [N][H][W][Ni] fp32 (NHWC)
 *   wbits    [No][kh][kw][Ni] uint8, each 0 or 1
 *   scale    [No], bias [No]   (the caller expands a single scaleValue)
 *   in_scale [Ni] or NULL, in_bias [Ni] or NULL
 *   pix      flattened output pixel indices n*Ho*Wo + oy*Wo + ox, or NULL for all of them
 *   S_out    [npix][No] the sum over the window (exact integers for XNOR/AND), may be NULL
 *   beta_out [npix] beta (1.0 when the flag is off), may be NULL
 *   y_out    [npix][No] the layer output, may be NULL
 * Returns 0, or -1 on a bad argument.
 */
int oracle_bconv(const oracle_conv_t* d, const float* in, const uint8_t* wbits, const float* scale,
                 const float* bias, const float* in_scale, const float* in_bias, const int64_t* pix,
                 int64_t npix, double* S_out, double* beta_out, double* y_out) {
  if (!d || !in || !wbits || !scale || !bias) return -1;
  if (d->batch < 0 || d->in_h <= 0 || d->in_w <= 0 || d->in_channels <= 0 || d->out_channels <= 0 ||
      d->kernel_h <= 0 || d->kernel_w <= 0 || d->stride_y <= 0 || d->stride_x <= 0)
    return -1;
  const int32_t H = d->in_h, W = d->in_w, Ni = d->in_channels, No = d->out_channels;
  const int32_t kh = d->kernel_h, kw = d->kernel_w;
  const int32_t Ho = out_extent(H, d->stride_y), Wo = out_extent(W, d->stride_x);
  const int64_t total = (int64_t)d->batch * Ho * Wo;
  if (!pix) npix = total;

#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t p = 0; p < npix; ++p) {
    const int64_t o = pix ? pix[p] : p;
    const int32_t n = (int32_t)(o / ((int64_t)Ho * Wo));
    const int32_t oy = (int32_t)((o / Wo) % Ho);
    const int32_t ox = (int32_t)(o % Wo);
    const int32_t cy = oy * d->stride_y, cx = ox * d->stride_x;

    /* beta[i,x,y] = sum over the window of A / (kx*ky), A = 0 outside the image. */
    double beta = 1.0;
    if (d->use_beta) {
      double acc = 0.0;
      for (int32_t dy = -(kh / 2); dy <= (kh - 1) / 2; ++dy)
        for (int32_t dx = -(kw / 2); dx <= (kw - 1) / 2; ++dx) {
          const int32_t y = cy + dy, x = cx + dx;
          if (y < 0 || y >= H || x < 0 || x >= W) continue;
          acc += channel_mean_abs(in, in_scale, in_bias, ((int64_t)n * H + y) * W + x, Ni);
        }
      beta = acc / ((double)kh * (double)kw);
    }
    if (beta_out) beta_out[p] = beta;

    for (int32_t c = 0; c < No; ++c) {
      double acc = 0.0;
      for (int32_t dy = -(kh / 2); dy <= (kh - 1) / 2; ++dy)
        for (int32_t dx = -(kw / 2); dx <= (kw - 1) / 2; ++dx) {
          const int32_t y = cy + dy, x = cx + dx;
          if (y < 0 || y >= H || x < 0 || x >= W) continue; /* out-of-image taps add 0 */
          const int64_t ipix = ((int64_t)n * H + y) * W + x;
          const int32_t ky = dy + kh / 2, kx = dx + kw / 2;
          const uint8_t* wrow = wbits + (((int64_t)c * kh + ky) * kw + kx) * Ni;
          for (int32_t f = 0; f < Ni; ++f)
            acc += op_term(d->type, transformed_input(in, in_scale, in_bias, ipix, Ni, f), wrow[f]);
        }
      if (S_out) S_out[p * No + c] = acc;
      double yv = acc * (double)scale[c] * beta + (double)bias[c];
      if (d->relu && yv < 0.0) yv = 0.0;
      if (y_out) y_out[p * No + c] = yv;
    }
  }
  return 0;
}

/*
 * Binary fully-connected layer: kernel = source size, 1x1xNo output.  The image of
 * image n is flattened to a vector of length H*W*Ni in (y, x, f) order and multiplied
 * by the No x (H*W*Ni) weight matrix, one (op) term per element.  With beta, the window
 * is the whole image, so beta_n = sum over all pixels of A / (H*W).
 *   in    [N][H][W][Ni] fp32;  wbits [No][H][W][Ni] uint8 0/1
 *   rows  image indices to compute, or NULL for all N
 *   S_out/y_out [nrows][No], beta_out [nrows]; any may be NULL.
 */
int oracle_bfc(int32_t batch, int32_t H, int32_t W, int32_t Ni, int32_t No, int32_t type,
               int32_t use_beta, int32_t relu, const float* in, const uint8_t* wbits,
               const float* scale, const float* bias, const float* in_scale, const float* in_bias,
               const int64_t* rows, int64_t nrows, double* S_out, double* beta_out, double* y_out) {
  if (!in || !wbits || !scale || !bias) return -1;
  if (batch < 0 || H <= 0 || W <= 0 || Ni <= 0 || No <= 0) return -1;
  const int64_t K = (int64_t)H * W * Ni;
  if (!rows) nrows = batch;

#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < nrows; ++r) {
    const int64_t n = rows ? rows[r] : r;
    const float* img = in + n * K; /* flattened vector v[k], k = (y*W + x)*Ni + f */

    double beta = 1.0;
    if (use_beta) {
      double acc = 0.0;
      for (int64_t p = 0; p < (int64_t)H * W; ++p) acc += channel_mean_abs(img, in_scale, in_bias, p, Ni);
      beta = acc / ((double)H * (double)W);
    }
    if (beta_out) beta_out[r] = beta;

    for (int32_t c = 0; c < No; ++c) {
      const uint8_t* wrow = wbits + (int64_t)c * K;
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        const int32_t f = (int32_t)(k % Ni);
        acc += op_term(type, transformed_input(img, in_scale, in_bias, k / Ni, Ni, f), wrow[k]);
      }
      if (S_out) S_out[r * No + c] = acc;
      double yv = acc * (double)scale[c] * beta + (double)bias[c];
      if (relu && yv < 0.0) yv = 0.0;
      if (y_out) y_out[r * No + c] = yv;
    }
  }
  return 0;
}

/*
 * The binarized form of an fp32 image, as the next binary layer sees it: per pixel and
 * channel x~ = inScale[c] * x + inBias[c], the sign bit bin(x~) as 1 (x~ >= 0) or 0, and the
 * per-pixel mean of |x~| over the channels (the "A" of the beta formula).  This is what a
 * binary convolution does to its input before the sum (same page, same paragraphs as
 * above); applied to one layer's output with the following layer's input terms it gives
 * the following layer's view of that output.
 *   x       [npix][C] fp32
 *   bits    [npix][C] uint8 0/1, may be NULL
 *   A       [npix] mean |x~|, may be NULL
 *   xt      [npix][C] x~ in double (before the sign decision), may be NULL
 */
int oracle_binarize(const float* x, int64_t npix, int32_t C, const float* in_scale, const float* in_bias,
                    uint8_t* bits, double* A, double* xt) {
  if (!x || npix < 0 || C <= 0) return -1;
#pragma omp parallel for schedule(static)
  for (int64_t p = 0; p < npix; ++p) {
    for (int32_t c = 0; c < C; ++c) {
      const double v = transformed_input(x, in_scale, in_bias, p, C, c);
      if (bits) bits[p * C + c] = (uint8_t)bin_01(v);
      if (xt) xt[p * C + c] = v;
    }
    if (A) A[p] = channel_mean_abs(x, in_scale, in_bias, p, C);
  }
  return 0;
}

/* Number of threads an OpenMP parallel region of the oracle uses (1 without OpenMP). */
int oracle_num_threads(void) {
  int n = 1;
#pragma omp parallel
  {
#pragma omp single
    {
#ifdef _OPENMP
      n = omp_get_num_threads();
#endif
    }
  }
  return n;
}
