// binaryWeights convolution: full-precision input against +-1 weights, FP32 accumulation.
//
// Apple page "MPSCNNBinaryConvolution", Overview, binaryWeights bullet: the input image is
// not binarized and the weights are read as [0,1] -> {-1,1}.  With the input terms
// ("inputScaleTerms" / "inputBiasTerms") the operand is x~ = inScale[f]*x + inBias[f], one
// fused multiply-add, applied only to in-image taps (out-of-image taps contribute 0).  Then
// out = act(S * scale[c] * beta + bias[c]).
//
// An implicit GEMM on the SIMT FP32 pipe: the weights are expanded once (at create) to
// +-1.0f in a reduction-major matrix [taps*ni_pad][no_pad], so that every product is one
// FFMA with a +-1 operand (exactly a signed add).  A CTA of 256 threads owns a 128 x 128
// output tile, a thread 8 x 8.  Each pipeline step covers one tap and 32 channels: the input
// tile is loaded into registers with 128-byte coalesced reads (8 threads per pixel),
// transformed, and stored k-major into shared memory with a 16-byte-chunk XOR swizzle that
// keeps both the transposing stores and the 128-bit compute loads free of bank conflicts;
// the weight tile arrives by cp.async.  Two stages, double-buffered.
#include "common.cuh"

namespace bconv {
namespace {

constexpr int BM = 128;
constexpr int BN = kTileN;
constexpr int BKC = kBwChanPad;  // channels per step
constexpr int kThreads = 256;
constexpr int kStageFloats = BKC * BM + BKC * BN;
constexpr int kSmemBytes = 2 * kStageFloats * 4;

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::); }

// Physical float index of A element (k, m) in a [BKC][BM] stage (16-byte chunks of m
// permuted by k so that both access patterns hit 32 distinct banks).
__device__ __forceinline__ int a_index(int k, int m) {
  return k * BM + ((((m >> 2) ^ ((k >> 2) & 7)) << 2) | (m & 3));
}

__device__ __forceinline__ int tile_row(int ty, int i) { return (i < 4 ? 0 : 64) + ty * 4 + (i & 3); }

template <bool kTerms, bool kVec4>
__global__ void __launch_bounds__(kThreads, 2) bw_conv_kernel(BwArgs a) {
  extern __shared__ __align__(16) float smem_f[];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int64_t M = static_cast<int64_t>(a.N) * a.Ho * a.Wo;
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * BM;
  const int n0 = blockIdx.y * BN;
  const int cpt = a.ni_pad / BKC;
  const int ksteps = a.kh * a.kw * cpt;

  // Staging role: 8 threads per pixel, 4 channels each; 32 pixels per pass, 4 passes.
  const int s_q = tid & 7;   // channel quad within the 32-channel step
  const int s_p = tid >> 3;  // pixel within a pass (0..31)
  int p_n[4], p_cy[4], p_cx[4];
  bool p_ok[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int64_t m = m0 + r * 32 + s_p;
    p_ok[r] = m < M;
    const int64_t hw = static_cast<int64_t>(a.Ho) * a.Wo;
    const int64_t mm = p_ok[r] ? m : 0;
    p_n[r] = static_cast<int>(mm / hw);
    p_cy[r] = static_cast<int>((mm % hw) / a.Wo) * a.sy;
    p_cx[r] = static_cast<int>(mm % a.Wo) * a.sx;
  }

  float4 stage[4];
  auto load_regs = [&](int ks) {
    const int t = ks / cpt, ch = ks - t * cpt;
    const int ky = t / a.kw, kx = t - ky * a.kw;
    const int f0 = ch * BKC + s_q * 4;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int y = p_cy[r] + ky - a.kh / 2, x = p_cx[r] + kx - a.kw / 2;
      const bool ok = p_ok[r] && y >= 0 && y < a.H && x >= 0 && x < a.W;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (ok) {
        const float* src = a.in + ((static_cast<int64_t>(p_n[r]) * a.H + y) * a.W + x) * a.ni + f0;
        if constexpr (kVec4) {
          if (f0 < a.ni) v = __ldg(reinterpret_cast<const float4*>(src));
        } else {
          v.x = f0 + 0 < a.ni ? __ldg(src + 0) : 0.f;
          v.y = f0 + 1 < a.ni ? __ldg(src + 1) : 0.f;
          v.z = f0 + 2 < a.ni ? __ldg(src + 2) : 0.f;
          v.w = f0 + 3 < a.ni ? __ldg(src + 3) : 0.f;
        }
        if constexpr (kTerms) {
          // x~ = inScale*x + inBias for real channels only; padding channels stay 0.
          if (f0 + 0 < a.ni) v.x = fmaf(v.x, __ldg(a.in_scale + f0 + 0), __ldg(a.in_bias + f0 + 0));
          if (f0 + 1 < a.ni) v.y = fmaf(v.y, __ldg(a.in_scale + f0 + 1), __ldg(a.in_bias + f0 + 1));
          if (f0 + 2 < a.ni) v.z = fmaf(v.z, __ldg(a.in_scale + f0 + 2), __ldg(a.in_bias + f0 + 2));
          if (f0 + 3 < a.ni) v.w = fmaf(v.w, __ldg(a.in_scale + f0 + 3), __ldg(a.in_bias + f0 + 3));
        }
      }
      stage[r] = v;
    }
  };
  auto store_regs = [&](int buf) {
    float* As = smem_f + buf * kStageFloats;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int m = r * 32 + s_p;
      const int k = s_q * 4;
      As[a_index(k + 0, m)] = stage[r].x;
      As[a_index(k + 1, m)] = stage[r].y;
      As[a_index(k + 2, m)] = stage[r].z;
      As[a_index(k + 3, m)] = stage[r].w;
    }
  };
  auto load_b = [&](int buf, int ks) {
    float* Bs = smem_f + buf * kStageFloats + BKC * BM;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int chunk = r * kThreads + tid;  // 0..1023: row = chunk / 32, col quad = chunk % 32
      const int k = chunk >> 5, c4 = (chunk & 31) * 4;
      cp_async16(Bs + k * BN + c4, a.wf + static_cast<int64_t>(ks * BKC + k) * a.no_pad + n0 + c4);
    }
  };

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  if (ksteps > 0) {
    load_regs(0);
    load_b(0, 0);
    cp_async_commit();
    store_regs(0);
    cp_async_wait_all();
    __syncthreads();
  }
  for (int ks = 0; ks < ksteps; ++ks) {
    const int buf = ks & 1;
    const bool more = ks + 1 < ksteps;
    if (more) {
      load_regs(ks + 1);
      load_b(buf ^ 1, ks + 1);
      cp_async_commit();
    }
    const float* As = smem_f + buf * kStageFloats;
    const float* Bs = As + BKC * BM;
#pragma unroll 8
    for (int k = 0; k < BKC; ++k) {
      const int f = (k >> 2) & 7;
      const float4 a0 = *reinterpret_cast<const float4*>(As + k * BM + ((ty ^ f) << 2));
      const float4 a1 = *reinterpret_cast<const float4*>(As + k * BM + (((16 + ty) ^ f) << 2));
      const float4 b0 = *reinterpret_cast<const float4*>(Bs + k * BN + tx * 4);
      const float4 b1 = *reinterpret_cast<const float4*>(Bs + k * BN + 64 + tx * 4);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    if (more) {
      store_regs(buf ^ 1);
      cp_async_wait_all();
    }
    __syncthreads();
  }

  const bool vec_ok = a.vec_out != 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t m = m0 + tile_row(ty, i);
    if (m >= M) continue;
    const float beta = a.beta ? __ldg(a.beta + m) : 1.f;
    float* orow = a.out + m * a.no;
#pragma unroll
    for (int jg = 0; jg < 2; ++jg) {
      const int c0 = n0 + jg * 64 + tx * 4;
      float v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int c = c0 + q;
        if (c < a.no) {
          const float S = acc[i][jg * 4 + q];
          const float sc = __ldg(a.scale + c), bi = __ldg(a.bias + c);
          float y = a.beta ? fmaf(S * sc, beta, bi) : fmaf(S, sc, bi);
          if (a.relu) y = fmaxf(y, 0.f);
          v[q] = y;
        } else {
          v[q] = 0.f;
        }
      }
      if (vec_ok && c0 + 3 < a.no) {
        *reinterpret_cast<float4*>(orow + c0) = make_float4(v[0], v[1], v[2], v[3]);
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (c0 + q < a.no) orow[c0 + q] = v[q];
      }
    }
  }
}

template <bool kTerms, bool kVec4>
cudaError_t launch_t(const BwArgs& a, cudaStream_t s) {
  const int64_t M = static_cast<int64_t>(a.N) * a.Ho * a.Wo;
  auto kern = bw_conv_kernel<kTerms, kVec4>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(ceil_div(M, BM)), static_cast<unsigned>(a.no_pad / BN));
  kern<<<grid, kThreads, kSmemBytes, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bw_conv(const BwArgs& a, cudaStream_t s) {
  const int64_t M = static_cast<int64_t>(a.N) * a.Ho * a.Wo;
  if (M == 0 || a.no == 0) return cudaSuccess;
  const bool vec = (a.ni & 3) == 0 && (reinterpret_cast<uintptr_t>(a.in) & 15) == 0;
  if (a.in_scale) return vec ? launch_t<true, true>(a, s) : launch_t<true, false>(a, s);
  return vec ? launch_t<false, true>(a, s) : launch_t<false, false>(a, s);
}

}  // namespace bconv
