// Binary convolution as an implicit GEMM on packed bits: LOP3 XOR/AND + POPC into int32
// registers, with the scale / beta / bias / neuron epilogue fused.
//
// What it computes (Apple page "MPSCNNBinaryConvolution", Overview, XNOR and AND bullets):
// for 32-bit words x (input bits) and y (weight bits) a dot product contributes
// 32 - 2*popcount(x^y) (XNOR) or popcount(x&y) (AND).  Summed over the window:
//   XNOR: S = sum_{valid taps} (Ni - 2 * sum_words popcount(a ^ w))
//   AND:  S = sum_{valid taps} sum_words popcount(a & w)
// and out = act(S * scale[c] * beta + bias[c]).  The fully-connected layer (page
// "MPSCNNFullyConnected", Overview) is the same contraction with one tap that spans the
// whole image.
//
// Out-of-image taps are loaded as zero words (cp.async zero-fill), which adds 0 for AND.
// For XNOR popcount(0 ^ w) = popcount(w), so the epilogue subtracts the weight popcount of
// every invalid tap, wpop[c][t], and counts Ni per valid tap only.  Padding bits (channels
// at or beyond Ni in the last word, and the zero words that pad a pixel to kWordPad) are
// zero in both operands and add 0.
//
// Tiling: a CTA of 256 threads owns a 128 (pixels) x 128 (channels) output tile; each
// thread an 8 x 8 register tile.  The reduction runs over (tap, 8-word chunk) steps that a
// 3-stage cp.async pipeline stages in shared memory: A as [pixel][8 words], B as
// [word][128 channels].  Per word a thread issues 64 POPC, 64 LOP3 and 32 IADD3 against 4
// shared loads, so the POPC pipe (16 lanes/clk/SM) is the bound.  When output tiles are
// too few to fill the GPU (the FC layer), the reduction is split over the CTAs of a
// thread-block cluster whose partial sums are added through distributed shared memory;
// int32 sums are exact in any order.
#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace bconv {
namespace {

constexpr int BM = 128;
constexpr int BN = kTileN;
constexpr int BK = kWordPad;  // words per pipeline stage
constexpr int kThreads = 256;
constexpr int kStages = 3;
constexpr int kStageWords = BM * BK + BK * BN;
constexpr int kPipeBytes = kStages * kStageWords * 4;
constexpr int kReduceBytes = BM * BN * 4;

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  const int n = valid ? 16 : 0;  // 0 bytes read -> the 16 bytes are zero-filled
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

template <int kOp>
__device__ __forceinline__ uint32_t bitop(uint32_t a, uint32_t b) {
  if constexpr (kOp == kXnor) return a ^ b;
  return a & b;
}

__device__ __forceinline__ uint32_t comp(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// Row i (0..7) of a thread's register tile -> row within the CTA tile.
__device__ __forceinline__ int tile_row(int ty, int i) { return (i < 4 ? 0 : 64) + ty * 4 + (i & 3); }

struct Epilogue {
  const PopcArgs& a;
  // y = act(S * scale[c] * beta + bias[c]) with one rounding per product.
  __device__ __forceinline__ float apply(int32_t S, int c, float beta, bool has_beta) const {
    const float sc = __ldg(a.scale + c), bi = __ldg(a.bias + c);
    float y = has_beta ? fmaf(static_cast<float>(S) * sc, beta, bi) : fmaf(static_cast<float>(S), sc, bi);
    if (a.relu) y = fmaxf(y, 0.f);
    return y;
  }
};

// Pixel geometry of output row m for the XNOR count and border correction.
struct RowInfo {
  int cy, cx;    // input-space centre
  int nvalid;    // taps inside the image
  bool all_valid;
  float beta;
};

__device__ __forceinline__ RowInfo row_info(const PopcArgs& a, int64_t m) {
  RowInfo r;
  const int64_t hw = static_cast<int64_t>(a.Ho) * a.Wo;
  const int oy = static_cast<int>((m % hw) / a.Wo), ox = static_cast<int>(m % a.Wo);
  r.cy = oy * a.sy;
  r.cx = ox * a.sx;
  const int y0 = max(r.cy - a.kh / 2, 0), y1 = min(r.cy + (a.kh - 1) / 2, a.H - 1);
  const int x0 = max(r.cx - a.kw / 2, 0), x1 = min(r.cx + (a.kw - 1) / 2, a.W - 1);
  r.nvalid = max(y1 - y0 + 1, 0) * max(x1 - x0 + 1, 0);
  r.all_valid = r.nvalid == a.kh * a.kw;
  r.beta = a.beta ? __ldg(a.beta + m) : 1.f;
  return r;
}

// S for one (row, channel) from the raw popcount sum P over all taps.
template <int kOp>
__device__ __forceinline__ int32_t finish_sum(const PopcArgs& a, const RowInfo& r, int c, int32_t P) {
  if constexpr (kOp == kAnd) {
    return P;
  } else {
    int32_t corr = 0;
    if (!r.all_valid) {
      const int32_t* wp = a.wpop + static_cast<int64_t>(c) * a.kh * a.kw;
      for (int ky = 0; ky < a.kh; ++ky) {
        const int y = r.cy + ky - a.kh / 2;
        for (int kx = 0; kx < a.kw; ++kx) {
          const int x = r.cx + kx - a.kw / 2;
          if (y < 0 || y >= a.H || x < 0 || x >= a.W) corr += __ldg(wp + ky * a.kw + kx);
        }
      }
    }
    return a.nbits * r.nvalid - 2 * (P - corr);
  }
}

template <int kOp, bool kSplit>
__global__ void __launch_bounds__(kThreads, 2) popc_gemm_kernel(PopcArgs a) {
  extern __shared__ __align__(16) uint32_t smem[];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int64_t M = static_cast<int64_t>(a.N) * a.Ho * a.Wo;
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * BM;
  const int n0 = blockIdx.y * BN;
  const int taps = a.kh * a.kw;
  const int cpt = a.nw / BK;  // chunks per tap
  const int ksteps = taps * cpt;
  int ks_begin = 0, ks_end = ksteps;
  if constexpr (kSplit) {
    const int per = (ksteps + a.split_k - 1) / a.split_k;
    ks_begin = min(static_cast<int>(blockIdx.z) * per, ksteps);
    ks_end = min(ks_begin + per, ksteps);
  }

  // The A row (output pixel) and 16-byte half this thread stages every step.
  const int a_row = tid >> 1, a_half = tid & 1;
  const int64_t a_m = m0 + a_row;
  const bool a_row_ok = a_m < M;
  int a_n = 0, a_cy = 0, a_cx = 0;
  if (a_row_ok) {
    const int64_t hw = static_cast<int64_t>(a.Ho) * a.Wo;
    a_n = static_cast<int>(a_m / hw);
    a_cy = static_cast<int>((a_m % hw) / a.Wo) * a.sy;
    a_cx = static_cast<int>(a_m % a.Wo) * a.sx;
  }
  const int b_k = tid >> 5, b_c = tid & 31;

  auto load_stage = [&](int buf, int ks) {
    uint32_t* As = smem + buf * kStageWords;
    uint32_t* Bs = As + BM * BK;
    const int t = ks / cpt, ch = ks - t * cpt;
    const int ky = t / a.kw, kx = t - ky * a.kw;
    const int y = a_cy + ky - a.kh / 2, x = a_cx + kx - a.kw / 2;
    const bool ok = a_row_ok && y >= 0 && y < a.H && x >= 0 && x < a.W;
    const uint32_t* src = a.bits;
    if (ok) src = a.bits + ((static_cast<int64_t>(a_n) * a.H + y) * a.W + x) * a.nw + ch * BK + a_half * 4;
    cp_async16(As + a_row * BK + a_half * 4, src, ok);
    const uint32_t* wsrc = a.wt + static_cast<int64_t>(ks * BK + b_k) * a.no_pad + n0 + b_c * 4;
    cp_async16(Bs + b_k * BN + b_c * 4, wsrc, true);
  };

  int32_t acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0;

#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (ks_begin + s < ks_end) load_stage(s, ks_begin + s);
    cp_async_commit();
  }

  for (int ks = ks_begin; ks < ks_end; ++ks) {
    const int it = ks - ks_begin;
    cp_async_wait<kStages - 2>();
    __syncthreads();
    if (ks + kStages - 1 < ks_end) load_stage((it + kStages - 1) % kStages, ks + kStages - 1);
    cp_async_commit();

    const uint32_t* As = smem + (it % kStages) * kStageWords;
    const uint32_t* Bs = As + BM * BK;
#pragma unroll
    for (int k4 = 0; k4 < BK / 4; ++k4) {
      uint4 av[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        av[i] = *reinterpret_cast<const uint4*>(As + tile_row(ty, i) * BK + k4 * 4);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint4 b0 = *reinterpret_cast<const uint4*>(Bs + (k4 * 4 + kk) * BN + tx * 4);
        const uint4 b1 = *reinterpret_cast<const uint4*>(Bs + (k4 * 4 + kk) * BN + 64 + tx * 4);
        const uint32_t bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t av_k = comp(av[i], kk);
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[i][j] += __popc(bitop<kOp>(av_k, bv[j]));
        }
      }
    }
  }
  cp_async_wait<0>();

  const Epilogue ep{a};
  const bool vec_ok = a.vec_out != 0;

  if constexpr (!kSplit) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t m = m0 + tile_row(ty, i);
      if (m >= M) continue;
      const RowInfo r = row_info(a, m);
      float* orow = a.out + m * a.no;
#pragma unroll
      for (int jg = 0; jg < 2; ++jg) {
        const int c0 = n0 + jg * 64 + tx * 4;
        float v[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int c = c0 + q;
          v[q] = c < a.no ? ep.apply(finish_sum<kOp>(a, r, c, acc[i][jg * 4 + q]), c, r.beta, a.beta != nullptr)
                          : 0.f;
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
  } else {
    // Split reduction: every CTA of the cluster parks its partial tile in its own shared
    // memory; CTA r then sums rows [r*BM/split, (r+1)*BM/split) over all CTAs and writes them.
    cg::cluster_group cluster = cg::this_cluster();
    __syncthreads();
    int32_t* red = reinterpret_cast<int32_t*>(smem);
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int jg = 0; jg < 2; ++jg)
        *reinterpret_cast<int4*>(red + tile_row(ty, i) * BN + jg * 64 + tx * 4) =
            make_int4(acc[i][jg * 4 + 0], acc[i][jg * 4 + 1], acc[i][jg * 4 + 2], acc[i][jg * 4 + 3]);
    cluster.sync();
    const int split = a.split_k;
    const int rank = static_cast<int>(cluster.block_rank());
    const int rows = BM / split;
    const int groups = rows * (BN / 4);
    for (int g = tid; g < groups; g += kThreads) {
      const int lr = rank * rows + g / (BN / 4);
      const int lc = (g % (BN / 4)) * 4;
      int4 s = make_int4(0, 0, 0, 0);
      for (int q = 0; q < split; ++q) {
        const int32_t* peer = cluster.map_shared_rank(red, q);
        const int4 p = *reinterpret_cast<const int4*>(peer + lr * BN + lc);
        s.x += p.x;
        s.y += p.y;
        s.z += p.z;
        s.w += p.w;
      }
      const int64_t m = m0 + lr;
      if (m >= M) continue;
      const RowInfo r = row_info(a, m);
      const int c0 = n0 + lc;
      const int32_t P[4] = {s.x, s.y, s.z, s.w};
      float v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int c = c0 + q;
        v[q] = c < a.no ? ep.apply(finish_sum<kOp>(a, r, c, P[q]), c, r.beta, a.beta != nullptr) : 0.f;
      }
      float* orow = a.out + m * a.no;
      if (vec_ok && c0 + 3 < a.no) {
        *reinterpret_cast<float4*>(orow + c0) = make_float4(v[0], v[1], v[2], v[3]);
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (c0 + q < a.no) orow[c0 + q] = v[q];
      }
    }
    cluster.sync();  // peers may still be reading this CTA's shared memory
  }
}

template <int kOp, bool kSplit>
cudaError_t launch_t(const PopcArgs& a, cudaStream_t s) {
  const int64_t M = static_cast<int64_t>(a.N) * a.Ho * a.Wo;
  const int smem = kSplit ? (kPipeBytes > kReduceBytes ? kPipeBytes : kReduceBytes) : kPipeBytes;
  auto kern = popc_gemm_kernel<kOp, kSplit>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ceil_div(M, BM)), static_cast<unsigned>(a.no_pad / BN),
                     kSplit ? static_cast<unsigned>(a.split_k) : 1u);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  if (kSplit) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = static_cast<unsigned>(a.split_k);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  e = cudaLaunchKernelEx(&cfg, kern, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

int popc_split_k_for(int64_t m_tiles, int64_t n_tiles, int ksteps, int sm_count) {
  const int64_t tiles = m_tiles * n_tiles;
  const int64_t slots = static_cast<int64_t>(sm_count) * 2;
  int best = 1;
  double best_eff = 0.0;
  for (int s = 1; s <= 8; s *= 2) {
    if (s > 1 && ksteps / s < 8) break;
    const int64_t ctas = tiles * s;
    const int64_t waves = ceil_div(ctas, slots);
    const double eff = static_cast<double>(ctas) / static_cast<double>(waves * slots);
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = s;
    }
  }
  return best;
}

cudaError_t launch_popc_gemm(const PopcArgs& a, cudaStream_t s) {
  const int64_t M = static_cast<int64_t>(a.N) * a.Ho * a.Wo;
  if (M == 0 || a.no == 0) return cudaSuccess;
  const bool split = a.split_k > 1;
  if (a.op == kXnor) return split ? launch_t<kXnor, true>(a, s) : launch_t<kXnor, false>(a, s);
  return split ? launch_t<kAnd, true>(a, s) : launch_t<kAnd, false>(a, s);
}

}  // namespace bconv
