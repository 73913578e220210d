// bconv_forward_noalloc: an XNOR / AND convolution forward that allocates no memory.
//
// Who needs it: code that must not call cudaMalloc at the moment it runs a layer -- for
// example a caller that has handed all device memory to its own pool allocator, or a
// real-time loop where an allocation could block on a device-wide synchronisation.  Such
// callers cannot create a handle (bconv_create allocates the weights and the workspace), so
// this entry point takes every operand as caller-owned device memory and keeps its working
// buffers in one fixed array that lives in this library's device image.
//
// The scratch array is `g_noalloc_scratch` below (BCONV_NOALLOC_SCRATCH_BYTES).  It is
// allocated by the CUDA runtime when the library's module is loaded on a device and is held
// by every device that loads the library until the process exits.  Host code cannot use the
// array's name as a device address (on the host it names a host-side stand-in), so the
// device address is looked up once per device with cudaGetSymbolAddress, with that device
// current, on the first call made on that device.
//
// It runs the SIMT kernel family -- the library's own pack, beta and POPC contraction (int32
// window sums), not the tensor cores, whose weight layout is prepared on the host when a layer
// is created -- and adds one small kernel that lays the caller's packed weights out for the
// contraction.  Every call rewrites
// all of the scratch it reads, so nothing carries over between calls; but all calls share the
// one array, so calls whose GPU work overlaps (two streams, or two host threads) race.
#include <mutex>

#include "bconv.h"
#include "common.cuh"

namespace bconv {
namespace {

__device__ __align__(256) static unsigned char g_noalloc_scratch[BCONV_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device (looked up once per device).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

// Bump allocator over the scratch array (256-byte aligned pieces); no device calls.
struct Carve {
  unsigned char* base;
  size_t used = 0;
  template <typename T>
  T* take(size_t count) {
    T* p = reinterpret_cast<T*>(base + used);
    used += (count * sizeof(T) + 255) / 256 * 256;
    return p;
  }
};

constexpr size_t piece(size_t bytes) { return (bytes + 255) / 256 * 256; }

// Caller weights [No][taps][nw] -> reduction-major [taps*nw_pad][no_pad] with zero padding
// (bits at or beyond Ni cleared), and per-(channel, tap) popcounts.  One thread per
// (column c < no_pad, tap t).
__global__ void noalloc_weight_layout(const uint32_t* __restrict__ w, int no, int no_pad, int taps, int nw,
                                      int nw_pad, uint32_t last_mask, uint32_t* __restrict__ wt,
                                      int32_t* __restrict__ wpop) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<int64_t>(no_pad) * taps) return;
  const int c = static_cast<int>(i % no_pad), t = static_cast<int>(i / no_pad);
  int32_t pc = 0;
  for (int k = 0; k < nw_pad; ++k) {
    uint32_t v = 0u;
    if (c < no && k < nw) {
      v = w[(static_cast<int64_t>(c) * taps + t) * nw + k];
      if (k == nw - 1) v &= last_mask;
    }
    wt[(static_cast<int64_t>(t) * nw_pad + k) * no_pad + c] = v;
    pc += __popc(v);
  }
  if (c < no) wpop[static_cast<int64_t>(c) * taps + t] = pc;
}

// Fill n floats with one value (defaults for operands the caller left out).
__global__ void noalloc_fill(float* __restrict__ p, int n, float v) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = v;
}

}  // namespace
}  // namespace bconv

using namespace bconv;

extern "C" bconv_status_t bconv_forward_noalloc(const bconv_desc_t* d, bconv_type_t type, uint32_t flags,
                                                const uint32_t* packed_weights, const float* scale,
                                                const float* bias, const float* in_scale, const float* in_bias,
                                                const float* in, float* out, struct CUstream_st* stream) {
  if (!d || !packed_weights) return BCONV_ERR_INVALID_ARG;
  if (type != BCONV_TYPE_XNOR && type != BCONV_TYPE_AND) return BCONV_ERR_INVALID_ARG;
  if (flags & ~static_cast<uint32_t>(BCONV_FLAG_USE_BETA_SCALING)) return BCONV_ERR_INVALID_ARG;
  const bconv_status_t shape = check_conv_shape(d);  // the same shapes bconv_create accepts
  if (shape != BCONV_OK) return shape;
  if (d->batch > 0 && (!in || !out)) return BCONV_ERR_INVALID_ARG;

  const int N = d->batch, H = d->in_h, W = d->in_w, Ni = d->in_channels, No = d->out_channels;
  const int kh = d->kernel_h, kw = d->kernel_w, sy = d->stride_y, sx = d->stride_x;
  const int Ho = (H + sy - 1) / sy, Wo = (W + sx - 1) / sx;
  const int taps = kh * kw;
  const int nw = words_for(Ni), nw_pad = round_up(nw, kWordPad), no_pad = round_up(No, kTileN);
  const bool beta = (flags & BCONV_FLAG_USE_BETA_SCALING) != 0;
  const int64_t npix = static_cast<int64_t>(N) * H * W;

  // Scratch needed by this call; larger requests are refused before any device work.
  size_t need = piece(static_cast<size_t>(npix) * nw_pad * 4) +
                piece(static_cast<size_t>(taps) * nw_pad * no_pad * 4) + piece(static_cast<size_t>(No) * taps * 4);
  if (beta) need += piece(static_cast<size_t>(npix) * 4) + piece(static_cast<size_t>(N) * Ho * Wo * 4);
  if (!scale) need += piece(static_cast<size_t>(No) * 4);
  if (!bias) need += piece(static_cast<size_t>(No) * 4);
  if ((in_scale != nullptr) != (in_bias != nullptr)) need += piece(static_cast<size_t>(Ni) * 4);
  if (need > static_cast<size_t>(BCONV_NOALLOC_SCRATCH_BYTES)) return BCONV_ERR_UNSUPPORTED;
  if (N == 0) return BCONV_OK;

  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
    cudaGetLastError();
    return BCONV_ERR_NO_DEVICE;
  }
  void* base = nullptr;
  if (scratch_address(&base) != cudaSuccess) return BCONV_ERR_CUDA;
  Carve carve{static_cast<unsigned char*>(base)};
  uint32_t* bits = carve.take<uint32_t>(static_cast<size_t>(npix) * nw_pad);
  uint32_t* wt = carve.take<uint32_t>(static_cast<size_t>(taps) * nw_pad * no_pad);
  int32_t* wpop = carve.take<int32_t>(static_cast<size_t>(No) * taps);
  float* A = beta ? carve.take<float>(npix) : nullptr;
  float* beta_img = beta ? carve.take<float>(static_cast<size_t>(N) * Ho * Wo) : nullptr;
  cudaStream_t s = stream;

  // Defaults for operands left out (the same defaults bconv_create uses).
  if (!scale) {
    float* p = carve.take<float>(No);
    noalloc_fill<<<(No + 255) / 256, 256, 0, s>>>(p, No, d->scale_value);
    scale = p;
  }
  if (!bias) {
    float* p = carve.take<float>(No);
    noalloc_fill<<<(No + 255) / 256, 256, 0, s>>>(p, No, 0.f);
    bias = p;
  }
  if (in_scale && !in_bias) {
    float* p = carve.take<float>(Ni);
    noalloc_fill<<<(Ni + 255) / 256, 256, 0, s>>>(p, Ni, 0.f);
    in_bias = p;
  } else if (in_bias && !in_scale) {
    float* p = carve.take<float>(Ni);
    noalloc_fill<<<(Ni + 255) / 256, 256, 0, s>>>(p, Ni, 1.f);
    in_scale = p;
  }

  const int tail = Ni % kWordBits;
  const uint32_t last_mask = tail ? ((1u << tail) - 1u) : 0xffffffffu;
  const int64_t wthreads = static_cast<int64_t>(no_pad) * taps;
  noalloc_weight_layout<<<static_cast<unsigned>((wthreads + 255) / 256), 256, 0, s>>>(
      packed_weights, No, no_pad, taps, nw, nw_pad, last_mask, wt, wpop);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return BCONV_ERR_CUDA;

  PackArgs p{};
  p.in = in;
  p.npix = npix;
  p.ni = Ni;
  p.nw_pad = nw_pad;
  p.in_scale = in_scale;
  p.in_bias = in_bias;
  p.bits = bits;
  p.A = A;
  if (launch_pack(p, s) != cudaSuccess) return BCONV_ERR_CUDA;
  if (beta) {
    BetaArgs b{A, beta_img, N, H, W, Ho, Wo, kh, kw, sy, sx};
    if (launch_beta_conv(b, s) != cudaSuccess) return BCONV_ERR_CUDA;
  }
  PopcArgs g{};
  g.bits = bits;
  g.wt = wt;
  g.wpop = wpop;
  g.scale = scale;
  g.bias = bias;
  g.beta = beta_img;
  g.out = out;
  g.N = N; g.H = H; g.W = W; g.Ho = Ho; g.Wo = Wo; g.kh = kh; g.kw = kw; g.sy = sy; g.sx = sx;
  g.nw = nw_pad;
  g.nbits = Ni;
  g.no = No;
  g.no_pad = no_pad;
  g.op = type;
  g.relu = d->neuron == BCONV_NEURON_RELU;
  g.vec_out = (No % 4 == 0) && (reinterpret_cast<uintptr_t>(out) & 15) == 0;
  const int64_t m_tiles = ceil_div(static_cast<int64_t>(N) * Ho * Wo, 128);
  g.split_k = popc_split_k_for(m_tiles, no_pad / kTileN, taps * (nw_pad / kWordPad), current_sm_count());
  if (launch_popc_gemm(g, s) != cudaSuccess) return BCONV_ERR_CUDA;
  return BCONV_OK;
}
