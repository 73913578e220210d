// Beta image for XNOR-Net style scaling.
//
// The Apple page "MPSCNNBinaryConvolution", Overview, defines
//   beta[i,x,y] = sum_{dx,dy} A[i, x+dx, y+dy] / (kx * ky)
// over the filter window [-kx/2, (kx-1)/2] x [-ky/2, (ky-1)/2], with A the per-pixel
// channel mean of |x~| (computed by the pack pass).  Window rows are
// dy in [-floor(kh/2), floor((kh-1)/2)]; positions outside the image hold A = 0 and the
// divisor stays kh*kw.  The output pixel (oy, ox) is centred on input (oy*sy, ox*sx).
// For the fully-connected case the window is the whole image, so beta_n is the sum of A
// over all pixels divided by H*W.
//
// A is tiny (one float per pixel) and stays in L2 after the pack pass; these kernels are
// launch-latency bound.
#include "common.cuh"

namespace bconv {
namespace {

constexpr int kBetaThreads = 256;

__global__ void __launch_bounds__(kBetaThreads) beta_conv_kernel(BetaArgs a) {
  const int64_t total = static_cast<int64_t>(a.N) * a.Ho * a.Wo;
  const int64_t o = static_cast<int64_t>(blockIdx.x) * kBetaThreads + threadIdx.x;
  if (o >= total) return;
  const int n = static_cast<int>(o / (static_cast<int64_t>(a.Ho) * a.Wo));
  const int oy = static_cast<int>((o / a.Wo) % a.Ho);
  const int ox = static_cast<int>(o % a.Wo);
  const int cy = oy * a.sy, cx = ox * a.sx;
  const float* An = a.A + static_cast<int64_t>(n) * a.H * a.W;
  float acc = 0.f;
  for (int dy = -(a.kh / 2); dy <= (a.kh - 1) / 2; ++dy) {
    const int y = cy + dy;
    if (y < 0 || y >= a.H) continue;
    for (int dx = -(a.kw / 2); dx <= (a.kw - 1) / 2; ++dx) {
      const int x = cx + dx;
      if (x < 0 || x >= a.W) continue;
      acc += __ldg(An + static_cast<int64_t>(y) * a.W + x);
    }
  }
  a.beta[o] = acc / static_cast<float>(a.kh * a.kw);
}

// One CTA per image: tree sum of A over the image, divided by H*W.
__global__ void __launch_bounds__(kBetaThreads) beta_image_mean_kernel(BetaArgs a) {
  __shared__ float part[kBetaThreads / 32];
  const int n = blockIdx.x;
  const int64_t hw = static_cast<int64_t>(a.H) * a.W;
  const float* An = a.A + n * hw;
  float acc = 0.f;
  for (int64_t p = threadIdx.x; p < hw; p += kBetaThreads) acc += __ldg(An + p);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    acc = threadIdx.x < kBetaThreads / 32 ? part[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (threadIdx.x == 0) a.beta[n] = acc / static_cast<float>(hw);
  }
}

}  // namespace

cudaError_t launch_beta_conv(const BetaArgs& a, cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(a.N) * a.Ho * a.Wo;
  if (total == 0) return cudaSuccess;
  beta_conv_kernel<<<static_cast<unsigned>(ceil_div(total, kBetaThreads)), kBetaThreads, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_beta_image_mean(const BetaArgs& a, cudaStream_t s) {
  if (a.N == 0) return cudaSuccess;
  beta_image_mean_kernel<<<a.N, kBetaThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace bconv
