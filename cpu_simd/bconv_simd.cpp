// A vectorised CPU binary convolution: the stated CPU baseline that the benchmark times beside
// the oracle.  It is not part of the CUDA library and never serves a forward of it.
//
// What it computes (Apple page "MPSCNNBinaryConvolution", Overview): x~ = inScale * x + inBias
// (one fp32 fused multiply-add), bin(x~) = x~ < 0 ? -1 : +1 packed as LSB-first bits (bit 1 for
// +1); per output and channel the window sum over the valid taps of the per-word forms of the
// XNOR bullet (32 - 2 * popcount(x ^ y) per full word) or of the AND bullet (popcount(x & y));
// beta = the window sum of A = mean_c |x~| over (kh * kw) with the useBetaScaling flag; and
// y = act(S * scale[c] * beta + bias[c]).  binaryWeights (input not binarized, weights
// [0,1] -> {-1,+1}) is an fp32 dot product of the window's x~ with +-1.0.  The fully-connected
// case (page "MPSCNNFullyConnected") is one output whose window is the whole image.
//
// The bit-packed sums are what the Bitwise XNOR page's CPU SIMD paragraph describes: XOR (or
// AND) and population count on wide vector registers.  Three code paths, chosen at run time:
// AVX-512 with VPOPCNTQ (8 x 64-bit counts per instruction), AVX2 with the nibble-lookup
// population count (VPSHUFB on the two 4-bit halves of every byte, VPSADBW to sum the bytes),
// and scalar 64-bit POPCNT.  Out-of-image taps read zero words; for XNOR their (nonzero)
// contribution popcount(0 ^ w) is taken back out with the per-tap weight popcounts, so the
// inner loop runs over the whole window without branches.  OpenMP over output pixels.
#include <immintrin.h>
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <vector>

namespace {

enum { kBinaryWeights = 0, kXnor = 1, kAnd = 2 };
enum { kIsaScalar = 0, kIsaAvx2 = 1, kIsaAvx512 = 2 };

struct Desc {
  int32_t batch, in_h, in_w, in_channels, out_channels;
  int32_t kernel_h, kernel_w, stride_y, stride_x;
  int32_t type, use_beta, relu, fc;
};

// ---- population count of (a op w) summed over n 64-bit words (n a multiple of 8) ----

int64_t popc_scalar(const uint64_t* a, const uint64_t* w, int64_t n, bool xnor) {
  int64_t s = 0;
  for (int64_t i = 0; i < n; ++i) s += __builtin_popcountll(xnor ? (a[i] ^ w[i]) : (a[i] & w[i]));
  return s;
}

__attribute__((target("avx2"))) int64_t popc_avx2(const uint64_t* a, const uint64_t* w, int64_t n, bool xnor) {
  const __m256i lut = _mm256_setr_epi8(0, 1, 1, 2, 1, 2, 2, 3, 1, 2, 2, 3, 2, 3, 3, 4, 0, 1, 1, 2, 1, 2, 2, 3, 1, 2, 2,
                                       3, 2, 3, 3, 4);
  const __m256i low = _mm256_set1_epi8(0x0F);
  __m256i acc = _mm256_setzero_si256();
  for (int64_t i = 0; i < n; i += 4) {
    const __m256i va = _mm256_loadu_si256(reinterpret_cast<const __m256i*>(a + i));
    const __m256i vw = _mm256_loadu_si256(reinterpret_cast<const __m256i*>(w + i));
    const __m256i v = xnor ? _mm256_xor_si256(va, vw) : _mm256_and_si256(va, vw);
    const __m256i cnt = _mm256_add_epi8(_mm256_shuffle_epi8(lut, _mm256_and_si256(v, low)),
                                        _mm256_shuffle_epi8(lut, _mm256_and_si256(_mm256_srli_epi16(v, 4), low)));
    acc = _mm256_add_epi64(acc, _mm256_sad_epu8(cnt, _mm256_setzero_si256()));
  }
  alignas(32) int64_t t[4];
  _mm256_store_si256(reinterpret_cast<__m256i*>(t), acc);
  return t[0] + t[1] + t[2] + t[3];
}

__attribute__((target("avx512f,avx512vpopcntdq"))) int64_t popc_avx512(const uint64_t* a, const uint64_t* w,
                                                                       int64_t n, bool xnor) {
  __m512i acc = _mm512_setzero_si512();
  for (int64_t i = 0; i < n; i += 8) {
    const __m512i va = _mm512_loadu_si512(a + i);
    const __m512i vw = _mm512_loadu_si512(w + i);
    acc = _mm512_add_epi64(acc, _mm512_popcnt_epi64(xnor ? _mm512_xor_si512(va, vw) : _mm512_and_si512(va, vw)));
  }
  return _mm512_reduce_add_epi64(acc);
}

// ---- fp32 dot product over n floats (n a multiple of 16), binaryWeights ----

float dot_scalar(const float* a, const float* w, int64_t n) {
  float lane[16] = {0.f};
  for (int64_t i = 0; i < n; ++i) lane[i % 16] = fmaf(a[i], w[i], lane[i % 16]);
  float s = 0.f;
  for (int j = 0; j < 16; ++j) s += lane[j];
  return s;
}

__attribute__((target("avx2,fma"))) float dot_avx2(const float* a, const float* w, int64_t n) {
  __m256 s0 = _mm256_setzero_ps(), s1 = _mm256_setzero_ps();
  for (int64_t i = 0; i < n; i += 16) {
    s0 = _mm256_fmadd_ps(_mm256_loadu_ps(a + i), _mm256_loadu_ps(w + i), s0);
    s1 = _mm256_fmadd_ps(_mm256_loadu_ps(a + i + 8), _mm256_loadu_ps(w + i + 8), s1);
  }
  alignas(32) float t[16];
  _mm256_store_ps(t, s0);
  _mm256_store_ps(t + 8, s1);
  float s = 0.f;
  for (int j = 0; j < 16; ++j) s += t[j];
  return s;
}

__attribute__((target("avx512f"))) float dot_avx512(const float* a, const float* w, int64_t n) {
  __m512 s = _mm512_setzero_ps();
  for (int64_t i = 0; i < n; i += 16) s = _mm512_fmadd_ps(_mm512_loadu_ps(a + i), _mm512_loadu_ps(w + i), s);
  return _mm512_reduce_add_ps(s);
}

// Sign bits and sum of |x~| of one pixel's channels, 16 at a time (AVX-512): x~ by one fused
// multiply-add, the bits from a "less than zero" compare mask (bit 1 for x~ >= 0, NaN included).
__attribute__((target("avx512f"))) float pack_pixel_avx512(const float* row, const float* sc, const float* bi, int ni,
                                                           uint32_t* bits) {
  __m512 acc = _mm512_setzero_ps();
  int f = 0;
  for (; f + 16 <= ni; f += 16) {
    __m512 v = _mm512_loadu_ps(row + f);
    if (sc) v = _mm512_fmadd_ps(v, _mm512_loadu_ps(sc + f), _mm512_loadu_ps(bi + f));
    acc = _mm512_add_ps(acc, _mm512_abs_ps(v));
    const uint32_t neg = _mm512_cmp_ps_mask(v, _mm512_setzero_ps(), _CMP_LT_OQ);
    bits[f / 32] |= (~neg & 0xFFFFu) << (f % 32);
  }
  float asum = _mm512_reduce_add_ps(acc);
  for (; f < ni; ++f) {  // the channels past the last full 16
    const float v = sc ? fmaf(row[f], sc[f], bi[f]) : row[f];
    asum += fabsf(v);
    if (!(v < 0.f)) bits[f / 32] |= 1u << (f % 32);
  }
  return asum;
}

int best_isa() {
  __builtin_cpu_init();
  if (__builtin_cpu_supports("avx512f") && __builtin_cpu_supports("avx512vpopcntdq")) return kIsaAvx512;
  if (__builtin_cpu_supports("avx2") && __builtin_cpu_supports("fma")) return kIsaAvx2;
  return kIsaScalar;
}

int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

}  // namespace

extern "C" {

// The vector path this CPU supports: 2 AVX-512 VPOPCNTDQ, 1 AVX2, 0 scalar.
int simd_best_isa(void) { return best_isa(); }

int simd_num_threads(void) { return omp_get_max_threads(); }

/*
 * x         float [N][H][W][Ni];  wpacked uint32 [No][kh][kw][ceil(Ni/32)] (LSB-first, bit 1 = +1
 *           or 1; bits at or past Ni ignored); for the FC kh = H, kw = W.
 * scale, bias [No] (required); in_scale, in_bias [Ni] or NULL.
 * pixels    optional flattened output indices (n*Ho*Wo + oy*Wo + ox; the image index for the
 *           FC), npix of them; NULL = every output.
 * S_out     optional int32 [npix][No] window sums (XNOR / AND) or fp32 sums (binaryWeights,
 *           stored as float bits); y_out float [npix][No].
 * isa       the vector path to use (at most simd_best_isa()); -1 = the best one.
 * Returns 0, or -1 for bad arguments.
 */
int simd_bconv(const Desc* d, const float* x, const uint32_t* wpacked, const float* scale, const float* bias,
               const float* in_scale, const float* in_bias, const int64_t* pixels, int64_t npix, int32_t* S_out,
               float* y_out, int isa) {
  if (!d || !x || !wpacked || !scale || !bias || !y_out) return -1;
  const int N = d->batch, H = d->in_h, W = d->in_w, Ni = d->in_channels, No = d->out_channels;
  const int kh = d->fc ? H : d->kernel_h, kw = d->fc ? W : d->kernel_w;
  const int sy = d->fc ? 1 : d->stride_y, sx = d->fc ? 1 : d->stride_x;
  if (N < 0 || H <= 0 || W <= 0 || Ni <= 0 || No <= 0 || kh <= 0 || kw <= 0 || sy <= 0 || sx <= 0) return -1;
  if (d->type != kBinaryWeights && d->type != kXnor && d->type != kAnd) return -1;
  if (isa < 0 || isa > best_isa()) isa = best_isa();
  const int Ho = d->fc ? 1 : (H + sy - 1) / sy, Wo = d->fc ? 1 : (W + sx - 1) / sx;
  const int64_t total = static_cast<int64_t>(N) * Ho * Wo;
  if (!pixels) npix = total;
  const int taps = kh * kw;
  const int nw = (Ni + 31) / 32;
  const int64_t npx = static_cast<int64_t>(N) * H * W;
  const bool bw = d->type == kBinaryWeights;

  // 1. input transform, sign bits (LSB-first, words padded to an even count) and A
  const int nw2 = static_cast<int>(round_up(nw, 2));  // 32-bit words per pixel, a whole number of uint64
  std::vector<uint32_t> bits(bw ? 0 : static_cast<size_t>(npx) * nw2, 0u);
  std::vector<float> xt(bw ? static_cast<size_t>(npx) * Ni : 0);
  std::vector<float> A(d->use_beta ? npx : 0);
  // both input terms, with the defaults filled in, for the vector pack
  std::vector<float> sc_full, bi_full;
  if (in_scale || in_bias) {
    sc_full.assign(Ni, 1.f);
    bi_full.assign(Ni, 0.f);
    for (int f = 0; f < Ni; ++f) {
      if (in_scale) sc_full[f] = in_scale[f];
      if (in_bias) bi_full[f] = in_bias[f];
    }
  }
  if (!bw && isa == kIsaAvx512) {
#pragma omp parallel for schedule(static)
    for (int64_t p = 0; p < npx; ++p) {
      const float asum = pack_pixel_avx512(x + p * Ni, sc_full.empty() ? nullptr : sc_full.data(),
                                           bi_full.empty() ? nullptr : bi_full.data(), Ni,
                                           bits.data() + static_cast<size_t>(p) * nw2);
      if (d->use_beta) A[p] = asum / static_cast<float>(Ni);
    }
  } else {
#pragma omp parallel for schedule(static)
  for (int64_t p = 0; p < npx; ++p) {
    const float* row = x + p * Ni;
    float asum = 0.f;
    for (int f = 0; f < Ni; ++f) {
      const float v = in_scale || in_bias ? fmaf(row[f], in_scale ? in_scale[f] : 1.f, in_bias ? in_bias[f] : 0.f)
                                          : row[f];
      asum += fabsf(v);
      if (bw)
        xt[static_cast<size_t>(p) * Ni + f] = v;
      else if (!(v < 0.f))
        bits[static_cast<size_t>(p) * nw2 + f / 32] |= 1u << (f % 32);
    }
    if (d->use_beta) A[p] = asum / static_cast<float>(Ni);
  }
  }

  // 2. weights: per channel the whole window as one contiguous row, padded to 8 uint64 (the
  //    bits) or 16 floats (binaryWeights); per (channel, tap) popcounts for the XNOR correction
  const int64_t kwords = round_up(static_cast<int64_t>(taps) * nw2 / 2, 8);  // uint64 per window
  const int64_t kfl = round_up(static_cast<int64_t>(taps) * Ni, 16);        // floats per window
  std::vector<uint64_t> wrow(bw ? 0 : static_cast<size_t>(No) * kwords, 0u);
  std::vector<float> wf(bw ? static_cast<size_t>(No) * kfl : 0, 0.f);
  std::vector<int32_t> wpop(static_cast<size_t>(No) * taps, 0);
  const uint32_t tail_mask = (Ni % 32) ? ((1u << (Ni % 32)) - 1u) : 0xFFFFFFFFu;
  for (int c = 0; c < No; ++c)
    for (int t = 0; t < taps; ++t)
      for (int k = 0; k < nw; ++k) {
        uint32_t v = wpacked[(static_cast<int64_t>(c) * taps + t) * nw + k];
        if (k == nw - 1) v &= tail_mask;
        wpop[static_cast<size_t>(c) * taps + t] += __builtin_popcount(v);
        if (bw) {
          for (int b = 0; b < 32 && k * 32 + b < Ni; ++b)
            wf[static_cast<size_t>(c) * kfl + static_cast<int64_t>(t) * Ni + k * 32 + b] = ((v >> b) & 1u) ? 1.f : -1.f;
        } else {
          reinterpret_cast<uint32_t*>(wrow.data() + static_cast<size_t>(c) * kwords)[t * nw2 + k] = v;
        }
      }

  // 3. per output pixel: gather the window (zero words / floats for out-of-image taps), then
  //    one vector reduction per output channel, beta and the epilogue
  const int oy0 = d->fc ? H / 2 : 0, ox0 = d->fc ? W / 2 : 0;
  const bool xnor = d->type == kXnor;
#pragma omp parallel
  {
    std::vector<uint64_t> win(bw ? 0 : kwords);
    std::vector<float> winf(bw ? kfl : 0);
    std::vector<char> valid(taps);
#pragma omp for schedule(dynamic, 16)
    for (int64_t i = 0; i < npix; ++i) {
      const int64_t o = pixels ? pixels[i] : i;
      if (o < 0 || o >= total) continue;
      const int n = static_cast<int>(o / (static_cast<int64_t>(Ho) * Wo));
      const int r = static_cast<int>(o % (static_cast<int64_t>(Ho) * Wo));
      const int cy = d->fc ? oy0 : (r / Wo) * sy, cx = d->fc ? ox0 : (r % Wo) * sx;
      int n_valid = 0;
      float asum = 0.f;
      if (bw) std::fill(winf.begin(), winf.end(), 0.f);
      else std::fill(win.begin(), win.end(), 0ull);
      for (int t = 0; t < taps; ++t) {
        const int y = cy + t / kw - kh / 2, xx = cx + t % kw - kw / 2;
        valid[t] = y >= 0 && y < H && xx >= 0 && xx < W;
        if (!valid[t]) continue;
        ++n_valid;
        const int64_t p = (static_cast<int64_t>(n) * H + y) * W + xx;
        if (d->use_beta) asum += A[p];
        if (bw)
          memcpy(winf.data() + static_cast<int64_t>(t) * Ni, xt.data() + p * Ni, sizeof(float) * Ni);
        else
          memcpy(reinterpret_cast<uint32_t*>(win.data()) + t * nw2, bits.data() + p * nw2, sizeof(uint32_t) * nw2);
      }
      const float beta = d->use_beta ? asum / static_cast<float>(kh * kw) : 1.f;
      for (int c = 0; c < No; ++c) {
        float s;
        if (bw) {
          const float* wc = wf.data() + static_cast<size_t>(c) * kfl;
          s = isa == kIsaAvx512 ? dot_avx512(winf.data(), wc, kfl)
              : isa == kIsaAvx2 ? dot_avx2(winf.data(), wc, kfl)
                                : dot_scalar(winf.data(), wc, kfl);
          if (S_out) memcpy(S_out + i * No + c, &s, sizeof(float));
        } else {
          const uint64_t* wc = wrow.data() + static_cast<size_t>(c) * kwords;
          int64_t pc = isa == kIsaAvx512 ? popc_avx512(win.data(), wc, kwords, xnor)
                       : isa == kIsaAvx2 ? popc_avx2(win.data(), wc, kwords, xnor)
                                         : popc_scalar(win.data(), wc, kwords, xnor);
          int64_t S;
          if (xnor) {
            // zero words of the out-of-image taps still counted popcount(w) there: take it back
            for (int t = 0; t < taps; ++t)
              if (!valid[t]) pc -= wpop[static_cast<size_t>(c) * taps + t];
            S = static_cast<int64_t>(Ni) * n_valid - 2 * pc;
          } else {
            S = pc;
          }
          if (S_out) S_out[i * No + c] = static_cast<int32_t>(S);
          s = static_cast<float>(S);
        }
        float y = d->use_beta ? fmaf(s * scale[c], beta, bias[c]) : fmaf(s, scale[c], bias[c]);
        if (d->relu) y = fmaxf(y, 0.f);
        y_out[i * No + c] = y;
      }
    }
  }
  return 0;
}

}  // extern "C"
