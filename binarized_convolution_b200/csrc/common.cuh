// Internal declarations shared by the library's translation units (not installed).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "bconv.h"

namespace bconv {

// Shape checks of a convolution descriptor shared by every entry point that takes one (neuron,
// positive sizes, groups == 1, window and channel limits, int32 window sums); OK, INVALID_ARG
// or UNSUPPORTED.
bconv_status_t check_conv_shape(const bconv_desc_t* d);

enum Op : int { kBinaryWeights = 0, kXnor = 1, kAnd = 2 };

// Error word bits the kernels may set (read by *_sync_status).
enum : uint32_t { kErrTimeout = 1u, kErrLayout = 2u };

constexpr int kWordBits = 32;
// Words per pixel are padded to this many (32 bytes) so that a pixel's words start on a
// 16-byte boundary and every pipeline stage of the POPC contraction reads whole chunks.
constexpr int kWordPad = 8;

inline int words_for(int bits) { return (bits + kWordBits - 1) / kWordBits; }
inline int round_up(int v, int m) { return (v + m - 1) / m * m; }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Multiprocessor count of the current device (cached per device).
int current_sm_count();

// Per-CTA timeline of a kernel's phases, for diagnosis: compiled in only when the library is
// built with -DBCONV_TIMELINE, where BCONV_STAMP(slot) writes %globaltimer into a device array
// (64 slots per CTA, one array per source file) that the host reads through the function
// BCONV_TIMELINE_READER(name) defines; otherwise both are empty.
#ifdef BCONV_TIMELINE
static __device__ unsigned long long g_bconv_timeline[1024 * 64];  // one array per source file
#define BCONV_TIMELINE_READER(name)                                                       \
  extern "C" int name(unsigned long long* host, int n) {                                 \
    return static_cast<int>(cudaMemcpyFromSymbol(host, bconv::g_bconv_timeline, sizeof(unsigned long long) * n)); \
  }
#define BCONV_STAMP(slot)                                                                              \
  do {                                                                                                 \
    unsigned long long t_;                                                                             \
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                                            \
    if (blockIdx.x < 1024) g_bconv_timeline[blockIdx.x * 64 + (slot)] = t_;                            \
  } while (0)
#else
#define BCONV_TIMELINE_READER(name)
#define BCONV_STAMP(slot) \
  do {                    \
  } while (0)
#endif

// x~ as three bf16 parts whose sum is x~ exactly, for the binaryWeights contraction (which
// multiplies each part by the same +-1 weights on the bf16 tensor cores): hi = x~ with the low
// 16 bits of its fp32 encoding cleared (its leading 8 significant bits), r = x~ - hi (exact: a
// subset of x~'s bits), mid = r cut the same way, lo = r - mid (exact, and with at most 8
// significant bits left, itself a bf16 with zero low bits).  Every part is a normal bf16 (or 0)
// for |x~| >= 2^-103.  Two values at a time as bf16x2 words (x0 in the low half); bit
// operations and exact subtractions (both values in one packed f32x2 subtraction, round to
// nearest, no flush to zero) only, no conversion instructions.
__device__ __forceinline__ void sub_f32x2(float a0, float a1, float b0, float b1, float& d0, float& d1) {
  asm("{\n .reg .b64 a, b, d;\n mov.b64 a, {%2, %3};\n mov.b64 b, {%4, %5};\n sub.rn.f32x2 d, a, b;\n"
      " mov.b64 {%0, %1}, d;\n}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

__device__ __forceinline__ void split3_bf16x2(float x0, float x1, uint32_t& hi, uint32_t& mid, uint32_t& lo) {
  const uint32_t u0 = __float_as_uint(x0), u1 = __float_as_uint(x1);
  hi = __byte_perm(u0, u1, 0x7632);  // the high halves of both
  float r0, r1;
  sub_f32x2(x0, x1, __uint_as_float(u0 & 0xffff0000u), __uint_as_float(u1 & 0xffff0000u), r0, r1);
  const uint32_t v0 = __float_as_uint(r0), v1 = __float_as_uint(r1);
  mid = __byte_perm(v0, v1, 0x7632);
  float q0, q1;
  sub_f32x2(r0, r1, __uint_as_float(v0 & 0xffff0000u), __uint_as_float(v1 & 0xffff0000u), q0, q1);
  lo = __byte_perm(__float_as_uint(q0), __float_as_uint(q1), 0x7632);
}

// Programmatic dependent launch, used by the kernels of the tensor-core forward: a kernel
// started with launch_overlapped may be scheduled while the previous kernel of the stream is
// finishing.  It calls wait_prior_grid() before it touches global memory (the previous kernel
// may be writing its input), and allow_next_grid() so that the next kernel can be scheduled
// in turn.  Both are no-ops for an ordinary launch.
__device__ __forceinline__ void wait_prior_grid() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_next_grid() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_overlapped(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Where pixel p = (n, y, x) of an [N][h][w] image lands in a zero-bordered [N][hp][wp] grid
// (at (n, y + pad_t, x + pad_l)); hp == 0 means no border (the pixel keeps its index).
struct PadMap {
  int h, w, hp, wp, pad_t, pad_l;
  // (A zero-bordered grid is only planned when N * hp * wp < 2^31, so p fits 32 bits then.)
  __host__ __device__ __forceinline__ int64_t operator()(int64_t p) const {
    if (hp == 0) return p;
    const uint32_t pp = static_cast<uint32_t>(p), hw = static_cast<uint32_t>(h) * static_cast<uint32_t>(w);
    const uint32_t n = pp / hw, r = pp - n * hw;
    const uint32_t y = r / static_cast<uint32_t>(w), x = r - y * static_cast<uint32_t>(w);
    return (static_cast<int64_t>(n) * hp + y + pad_t) * wp + x + pad_l;
  }
  // The place of pixel p + 1 from that of pixel p, whose column and row are x and y (updated).
  __host__ __device__ __forceinline__ int64_t next(int64_t q, int& y, int& x) const {
    if (hp == 0) return q + 1;
    ++q;
    if (++x == w) {
      x = 0;
      q += wp - w;
      if (++y == h) {
        y = 0;
        q += static_cast<int64_t>(hp - h) * wp;
      }
    }
    return q;
  }
  // Column and row of pixel p.
  __host__ __device__ __forceinline__ void yx(int64_t p, int& y, int& x) const {
    if (hp == 0) return;
    const uint32_t pp = static_cast<uint32_t>(p), hw = static_cast<uint32_t>(h) * static_cast<uint32_t>(w);
    const uint32_t r = pp % hw;
    y = static_cast<int>(r / static_cast<uint32_t>(w));
    x = static_cast<int>(r - static_cast<uint32_t>(y) * static_cast<uint32_t>(w));
  }
};

// ------------------------------------------------------------------------------------
// Input transform, sign and pack (one pass over the fp32 input).
// ------------------------------------------------------------------------------------
struct PackArgs {
  const float* in;        // [npix][ni] fp32
  int64_t npix;
  int ni;
  int nw_pad;             // words written per pixel (>= ceil(ni/32), multiple of kWordPad)
  const float* in_scale;  // [ni] or nullptr
  const float* in_bias;   // [ni] or nullptr
  uint32_t* bits;         // [npix][nw_pad] or nullptr (A only)
  float* A;               // [npix] or nullptr (no beta)
};
cudaError_t launch_pack(const PackArgs& a, cudaStream_t s);

// Bit-packed activations u32 [npix][ceil(ni/32)] (bits at or past ni ignored) into the POPC
// layout [npix][nw_pad] (tail bits cleared, padding words 0), or into int8 operand codes
// [npix][cip] (XNOR: bit 1 -> +1, 0 -> -1; AND: 1 -> 1, 0 -> 0; channels >= ni -> 0;
// codes 16-byte aligned, cip a multiple of 16).
cudaError_t launch_repack_bits(const uint32_t* bits, int64_t npix, int ni, int nw_pad, uint32_t* out, cudaStream_t s);
cudaError_t launch_unpack_bits_i8(const uint32_t* bits, int64_t npix, int ni, int cip, int op, int8_t* codes,
                                  cudaStream_t s);
// ... or into e2m1 (fp4) codes [npix][cip / 2] bytes, two channels per byte (XNOR: 1 -> +1.0
// = 0x2, 0 -> -1.0 = 0xA; AND: 1 -> 0x2, 0 -> 0; channels >= ni -> 0; cip a multiple of 32).
cudaError_t launch_unpack_bits_f4(const uint32_t* bits, int64_t npix, int ni, int cip, int op, int8_t* codes,
                                  cudaStream_t s, PadMap pad = PadMap{});
// Copy an [N][h][w] float image into the same pixels of a zero-bordered grid.
cudaError_t launch_pad_copy(const float* src, int64_t npix, PadMap pad, float* dst, cudaStream_t s);

// ------------------------------------------------------------------------------------
// Beta: box filter of A over the window (conv) or mean of A over the image (FC).
// ------------------------------------------------------------------------------------
struct BetaArgs {
  const float* A;  // [N][H][W]
  float* beta;     // [N][Ho][Wo] (conv) or [N] (FC)
  int N, H, W, Ho, Wo, kh, kw, sy, sx;
};
cudaError_t launch_beta_conv(const BetaArgs& a, cudaStream_t s);
cudaError_t launch_beta_image_mean(const BetaArgs& a, cudaStream_t s);

// ------------------------------------------------------------------------------------
// POPC implicit-GEMM contraction with the fused epilogue (XNOR / AND).
// Geometry of the convolution as a GEMM: rows = output pixels, columns = output
// channels, reduction = taps x words.  The FC case is a 1x1 "convolution" whose single
// pixel per image holds all H*W*nw words.
// ------------------------------------------------------------------------------------
struct PopcArgs {
  const uint32_t* bits;   // [N][H][W][nw] packed input bits
  const uint32_t* wt;     // [kh*kw*nw][no_pad] packed weights, reduction-major
  const int32_t* wpop;    // [no][kh*kw] weight popcount per tap (XNOR border correction)
  const float* scale;     // [no]
  const float* bias;      // [no]
  const float* beta;      // [N*Ho*Wo] or nullptr
  float* out;             // [N*Ho*Wo][no]
  int N, H, W, Ho, Wo, kh, kw, sy, sx;
  int nw;                 // words per pixel (multiple of kWordPad)
  int nbits;              // real bits per tap (Ni, or H*W*Ni for the FC)
  int no, no_pad;
  int op;                 // kXnor or kAnd
  int relu;
  int split_k;            // 1, or CTAs of a cluster sharing one output tile
  int vec_out;            // out is 16-byte aligned and no % 4 == 0: float4 stores
};
cudaError_t launch_popc_gemm(const PopcArgs& a, cudaStream_t s);
int popc_split_k_for(int64_t m_tiles, int64_t n_tiles, int ksteps, int sm_count);

// ------------------------------------------------------------------------------------
// binaryWeights: FP32 signed-add contraction with the transform fused into the loads.
// ------------------------------------------------------------------------------------
struct BwArgs {
  const float* in;        // [N][H][W][ni] raw input
  const float* in_scale;  // [ni] or nullptr
  const float* in_bias;   // [ni] or nullptr
  const float* wf;        // [kh*kw*ni_pad][no_pad] weights as +-1.0f (0 in padding)
  const float* scale;     // [no]
  const float* bias;      // [no]
  const float* beta;      // [N*Ho*Wo] or nullptr
  float* out;             // [N*Ho*Wo][no]
  int N, H, W, Ho, Wo, kh, kw, sy, sx;
  int ni, ni_pad, no, no_pad;
  int relu;
  int vec_out;            // out is 16-byte aligned and no % 4 == 0: float4 stores
};
cudaError_t launch_bw_conv(const BwArgs& a, cudaStream_t s);
constexpr int kBwChanPad = 32;  // channels per pipeline stage of the FP32 kernel
constexpr int kTileN = 128;     // output channels per CTA tile (both contraction kernels)

// ------------------------------------------------------------------------------------
// Peak probes.
// ------------------------------------------------------------------------------------
cudaError_t probe_peak(int kind, double* ops_per_s, double* sm_mhz);
// Runs the kernels' bounded mbarrier wait on a barrier nothing completes, with the given limit;
// *status receives the error word it left (kErrTimeout expected).
cudaError_t wait_check(double limit_ms, uint32_t* status);

}  // namespace bconv
