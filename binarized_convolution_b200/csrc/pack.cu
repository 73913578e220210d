// Input transform + sign + bit-pack + channel mean |x~|, in one pass over the fp32 input.
//
// Follows the Apple page "MPSCNNBinaryConvolution", Overview: the input is pre-offset and
// scaled by inputScaleTerms / inputBiasTerms before binarization and before the beta image
// ("The scaling of input values happens before possible beta-image computation"), is
// binarized by bin(x) = x < 0 ? -1 : 1 (bit 1 <-> +1), and A[i,x,y] = sum_c |in| / Nc feeds
// beta.  x~ is one fused multiply-add, so its sign is the sign of the exact affine value.
//
// Layout: one warp per pixel.  Lane l takes channel 32*w + l of word w, so a warp load is
// one coalesced 128-byte line and __ballot_sync assembles the word in channel order
// (LSB = lowest channel).  Eight words are loaded before any is used so that each warp
// keeps a kilobyte in flight; the kernel is bound by the fp32 read.

#include <algorithm>

#include "common.cuh"
#include "pack_stage.cuh"
#include "tc_device.cuh"

namespace bconv {
namespace {

constexpr int kPackThreads = 256;
constexpr int kWordsInFlight = 8;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <bool kTerms, bool kBits, bool kA>
__global__ void __launch_bounds__(kPackThreads) pack_kernel(PackArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kPackThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kPackThreads) >> 5;
  const int ni = a.ni;
  const int nw = (ni + kWordBits - 1) / kWordBits;

  for (int64_t p = warp; p < a.npix; p += nwarps) {
    const float* row = a.in + p * ni;
    uint32_t* brow = kBits ? a.bits + p * a.nw_pad : nullptr;
    float asum = 0.f;
    for (int w0 = 0; w0 < nw; w0 += kWordsInFlight) {
      float x[kWordsInFlight];
#pragma unroll
      for (int j = 0; j < kWordsInFlight; ++j) {
        const int f = (w0 + j) * kWordBits + lane;
        x[j] = (f < ni) ? __ldcs(row + f) : 0.f;
      }
#pragma unroll
      for (int j = 0; j < kWordsInFlight; ++j) {
        const int w = w0 + j;
        if (w >= nw) break;  // warp-uniform
        const int f = w * kWordBits + lane;
        const bool valid = f < ni;
        float xt = x[j];
        if (kTerms && valid) xt = fmaf(xt, __ldg(a.in_scale + f), __ldg(a.in_bias + f));
        if (kA) asum += valid ? fabsf(xt) : 0.f;
        if (kBits) {
          const uint32_t word = __ballot_sync(0xffffffffu, valid && !(xt < 0.f));
          if (lane == 0) brow[w] = word;
        }
      }
    }
    if (kBits)
      for (int w = nw + lane; w < a.nw_pad; w += 32) brow[w] = 0u;
    if (kA) {
      asum = warp_sum(asum);
      if (lane == 0) a.A[p] = asum / static_cast<float>(ni);
    }
  }
}

template <bool kTerms>
cudaError_t launch_pack_t(const PackArgs& a, cudaStream_t s) {
  const int sms = current_sm_count();
  const int64_t warps_per_block = kPackThreads / 32;
  int64_t blocks = ceil_div(a.npix, warps_per_block);
  const int64_t cap = static_cast<int64_t>(sms) * 8;  // 8 x 256 threads = 64 warps per SM
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  const dim3 grid(static_cast<unsigned>(blocks));
  if (a.bits && a.A)
    pack_kernel<kTerms, true, true><<<grid, kPackThreads, 0, s>>>(a);
  else if (a.bits)
    pack_kernel<kTerms, true, false><<<grid, kPackThreads, 0, s>>>(a);
  else if (a.A)
    pack_kernel<kTerms, false, true><<<grid, kPackThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pack(const PackArgs& a, cudaStream_t s) {
  if (a.npix == 0 || (!a.bits && !a.A)) return cudaSuccess;
  if (a.in_scale) return launch_pack_t<true>(a, s);
  return launch_pack_t<false>(a, s);
}

}  // namespace bconv

// ------------------------------------------------------------------------------------
// int8 operand codes for the tensor-core contraction, with the same transform and A.
// A warp per pixel; with 4-aligned channels each lane turns one float4 into 4 codes (one
// 32-bit store), so a warp writes 128 contiguous code bytes per step.
// ------------------------------------------------------------------------------------
#include "tc_conv.cuh"

namespace bconv {
namespace {

// Codes for 4 transformed values as one little-endian word.
template <int kOp>
__device__ __forceinline__ uint32_t codes4(const float4& v) {
  constexpr uint32_t kPos = 0x01u;
  constexpr uint32_t kNeg = kOp == kXnor ? 0xFFu : 0x00u;
  return ((v.x < 0.f) ? kNeg : kPos) | (((v.y < 0.f) ? kNeg : kPos) << 8) | (((v.z < 0.f) ? kNeg : kPos) << 16) |
         (((v.w < 0.f) ? kNeg : kPos) << 24);
}

// The same 4 values as e2m1 (fp4) codes in one 16-bit word, element j in bits 4j..4j+3:
// +1.0 = 0x2; -1.0 = 0xA (XNOR) or 0 (AND).
template <int kOp>
__device__ __forceinline__ uint32_t nibbles4(const float4& v) {
  constexpr uint32_t kPos = 0x2u;
  constexpr uint32_t kNeg = kOp == kXnor ? 0xAu : 0x0u;
  return ((v.x < 0.f) ? kNeg : kPos) | (((v.y < 0.f) ? kNeg : kPos) << 4) | (((v.z < 0.f) ? kNeg : kPos) << 8) |
         (((v.w < 0.f) ? kNeg : kPos) << 12);
}

template <bool kTerms>
__device__ __forceinline__ float4 transform4(float4 v, const float* __restrict__ sc, const float* __restrict__ bi,
                                             int f) {
  if (kTerms) {
    const float4 s = __ldg(reinterpret_cast<const float4*>(sc + f));
    const float4 b = __ldg(reinterpret_cast<const float4*>(bi + f));
    v.x = fmaf(v.x, s.x, b.x);
    v.y = fmaf(v.y, s.y, b.y);
    v.z = fmaf(v.z, s.z, b.z);
    v.w = fmaf(v.w, s.w, b.w);
  }
  return v;
}

// Vector path: kC chunks of 128 channels per pixel (a compile-time 1, 2 or 4), a group of
// 8 / kC pixels per warp step (8 float4 loads per lane).  The loads of the next group are
// issued before the current one is converted, so two groups per warp are in flight.
// Lane l always handles channels chunk*128 + 4l .. 4l+3, so its input terms stay in registers.
template <int kG, int kC>
__device__ __forceinline__ void load_group(float4 (&v)[kG][kC], const float* __restrict__ in, int64_t p0, int64_t npix,
                                           int ni, const bool (&live)[kC], int lane) {
#pragma unroll
  for (int g = 0; g < kG; ++g)
#pragma unroll
    for (int c = 0; c < kC; ++c) {
      const int64_t p = p0 + g;
      v[g][c] = (p < npix && live[c]) ? __ldcs(reinterpret_cast<const float4*>(in + p * ni + c * 128 + lane * 4))
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

template <bool kTerms, bool kA, int kOp, int kC, bool kF4>
__global__ void __launch_bounds__(kPackThreads, 2) pack_i8_vec_kernel(PackI8Args a) {
  constexpr int kG = 8 / kC;  // pixels per warp step
  constexpr int kLanesPerPix = 32 / kG;  // lanes holding one pixel's A after warp_sum_multi
  wait_prior_grid();
  allow_next_grid();
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kPackThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kPackThreads) >> 5;
  const int ni = a.ni;
  const float* __restrict__ in = a.in;
  int8_t* __restrict__ codes = a.codes;
  const int64_t pbytes = kF4 ? a.cip / 2 : a.cip;  // code bytes per pixel
  float4 sc[kC], bi[kC];
  bool live[kC];
#pragma unroll
  for (int c = 0; c < kC; ++c) {
    const int f = c * 128 + lane * 4;
    live[c] = f < ni;
    sc[c] = make_float4(1.f, 1.f, 1.f, 1.f);
    bi[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (kTerms && live[c]) {
      sc[c] = __ldg(reinterpret_cast<const float4*>(a.in_scale + f));
      bi[c] = __ldg(reinterpret_cast<const float4*>(a.in_bias + f));
    }
  }
  // Each warp packs one contiguous range of whole steps: a pixel's place in the code grid then
  // follows from the previous pixel's (one division per warp, none per pixel), and each warp
  // streams one stretch of the input.
  const int64_t steps = (a.npix + kG - 1) / kG;
  const int64_t per_warp = (steps + nwarps - 1) / nwarps;
  int64_t p0 = warp * per_warp * kG;
  const int64_t p_end = min(a.npix, p0 + per_warp * kG);
  if (p0 >= p_end) return;
  int py = 0, px = 0;
  a.pad.yx(p0, py, px);
  int64_t q = a.pad(p0);  // place of the next pixel to pack
  float4 v[kG][kC];
  load_group<kG, kC>(v, in, p0, p_end, ni, live, lane);
  for (; p0 < p_end; p0 += kG) {
    float4 nxt[kG][kC];
    if (p0 + kG < p_end) load_group<kG, kC>(nxt, in, p0 + kG, p_end, ni, live, lane);
    float asum[kG];
    int64_t qa = q;  // place of this lane's pixel for A (set below)
#pragma unroll
    for (int g = 0; g < kG; ++g) {
      asum[g] = 0.f;
      if (p0 + g >= p_end) continue;  // warp-uniform
      if (g == lane / kLanesPerPix) qa = q;
      int8_t* crow = codes + q * pbytes;
#pragma unroll
      for (int c = 0; c < kC; ++c) {
        uint32_t word = 0u;
        if (live[c]) {
          float4 t = v[g][c];
          if (kTerms) {
            t.x = fmaf(t.x, sc[c].x, bi[c].x);
            t.y = fmaf(t.y, sc[c].y, bi[c].y);
            t.z = fmaf(t.z, sc[c].z, bi[c].z);
            t.w = fmaf(t.w, sc[c].w, bi[c].w);
          }
          if (kA) asum[g] += (fabsf(t.x) + fabsf(t.y)) + (fabsf(t.z) + fabsf(t.w));
          word = kF4 ? nibbles4<kOp>(t) : codes4<kOp>(t);
        }
        if (kF4)  // e2m1 codes: cip / 2 bytes per pixel, 64 bytes per 128-channel chunk
          *reinterpret_cast<uint16_t*>(crow + c * 64 + lane * 2) = static_cast<uint16_t>(word);
        else
          *reinterpret_cast<uint32_t*>(crow + c * 128 + lane * 4) = word;
      }
      q = a.pad.next(q, py, px);
    }
    if (kA) {
      // one reduction for the step's pixels; lanes g * kLanesPerPix hold pixel g's sum
      const float total = packdev::warp_sum_multi<kG>(asum, lane);
      const int g = lane / kLanesPerPix;
      if ((lane % kLanesPerPix) == 0 && p0 + g < p_end) a.A[qa] = total / static_cast<float>(ni);
    }
#pragma unroll
    for (int g = 0; g < kG; ++g)
#pragma unroll
      for (int c = 0; c < kC; ++c) v[g][c] = nxt[g][c];
  }
}

// Any channel count: one byte per lane per step (one channel as int8, two as e2m1 nibbles).
template <bool kTerms, bool kA, int kOp, bool kF4>
__global__ void __launch_bounds__(kPackThreads) pack_i8_scalar_kernel(PackI8Args a) {
  wait_prior_grid();
  allow_next_grid();
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kPackThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kPackThreads) >> 5;
  const int ni = a.ni;
  constexpr uint32_t kPos = kF4 ? 0x2u : 0x01u;
  constexpr uint32_t kNeg = kOp == kXnor ? (kF4 ? 0xAu : 0xFFu) : 0x00u;
  constexpr int kPer = kF4 ? 2 : 1;  // channels per lane and step
  for (int64_t p = warp; p < a.npix; p += nwarps) {
    const float* row = a.in + p * ni;
    const int64_t q = a.pad(p);  // the pixel's place in the code buffer (and in A)
    int8_t* crow = a.codes + q * (a.cip / kPer);
    float asum = 0.f;
    for (int f0 = 0; f0 < a.cip; f0 += 32 * kPer) {
      uint32_t byte = 0u;
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const int f = f0 + lane * kPer + u;
        uint32_t code = 0u;
        if (f < ni) {
          float v = __ldcs(row + f);
          if (kTerms) v = fmaf(v, __ldg(a.in_scale + f), __ldg(a.in_bias + f));
          if (kA) asum += fabsf(v);
          code = (v < 0.f) ? kNeg : kPos;
        }
        byte |= code << (4 * u);
      }
      crow[f0 / kPer + lane] = static_cast<int8_t>(byte);
    }
    if (kA) {
      asum = warp_sum(asum);
      if (lane == 0) a.A[q] = asum / static_cast<float>(ni);
    }
  }
}

// ------------------------------------------------------------------------------------
// e2m1 codes through a bulk-copy ring.  The register-fed kernels above keep a few kilobytes in
// flight per warp and spend ~140 instructions per 256-channel pixel; this one has one thread
// stream each CTA's contiguous stretch of pixels into shared memory (kStagedStages stages of
// up to 8 KB: 128 KB in flight per SM) and eight warps convert it, each a whole stage of kSP
// pixels at a time -- lane l takes channels 8 l .. 8 l + 7 of each 256-channel pass, whose
// eight codes are one 32-bit store -- so that a pixel's place in the code grid follows from the
// previous one's and one reduction forms the stage's kSP values of A.
// ------------------------------------------------------------------------------------
constexpr int kStagedStages = 16;  // two per converting warp (one CTA per SM)
constexpr int kStagedBytes = 8192;
constexpr int kStagedWarps = 8;  // converting warps; one more warp feeds the ring
// A stretch of few stages per SM (a small input) runs as two CTAs per SM with half the ring
// each: more copies start at once, and the ramp to full streaming is what such a pack costs.
constexpr int kStagedStagesHalf = 8;
constexpr int kFewStagesPerSm = 32;

struct __align__(8) StagedBars {
  uint64_t full[kStagedStages];
  uint64_t empty[kStagedStages];
  uint32_t abort_flag;
  uint32_t err_word;  // stands in for a missing error word
};

template <bool kTerms, bool kA, int kOp, int kSP, int kStagedStages>
__global__ void __launch_bounds__((kStagedWarps + 1) * 32, 16 / kStagedStages)
    pack_f4_staged_kernel(PackI8Args a, int64_t per_cta) {
  extern __shared__ __align__(128) uint8_t sm[];
  StagedBars* B = reinterpret_cast<StagedBars*>(sm + kStagedStages * kStagedBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ni = a.ni;
  const int64_t p_begin = static_cast<int64_t>(blockIdx.x) * per_cta;
  const int64_t p_end = min(a.npix, p_begin + per_cta);
  const int64_t nst = p_begin < p_end ? (p_end - p_begin + kSP - 1) / kSP : 0;  // stages of this CTA
  uint32_t* err = a.err ? a.err : &B->err_word;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStagedStages; ++i) {
      tcdev::mbar_init(&B->full[i], 1);
      tcdev::mbar_init(&B->empty[i], 1);
    }
    B->abort_flag = 0;
    B->err_word = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (threadIdx.x == 0) BCONV_STAMP(0);
  __syncthreads();
  wait_prior_grid();  // the input and the code buffer belong to the previous kernels until here
  allow_next_grid();
  if (threadIdx.x == 0) BCONV_STAMP(1);
  if (warp == kStagedWarps) {
    if (lane == 0) {
      int64_t issued = 0;
      for (int64_t st = 0; st < nst; ++st) {
        const int slot = static_cast<int>(st % kStagedStages);
        const int64_t use = st / kStagedStages;
        if (use > 0 && !tcdev::mbar_wait(&B->empty[slot], static_cast<uint32_t>((use - 1) & 1), B, err)) break;
        const int64_t p = p_begin + st * kSP;
        const int np = static_cast<int>(min(static_cast<int64_t>(kSP), p_end - p));
        const uint32_t bytes = static_cast<uint32_t>(np) * static_cast<uint32_t>(ni) * 4u;
        tcdev::mbar_expect_tx(&B->full[slot], bytes);
        tcdev::bulk_load(sm + slot * kStagedBytes, a.in + p * ni, bytes, &B->full[slot]);
        issued = st + 1;
      }
      // every copy has landed before the CTA may leave (after an abort too): the last phase
      // of each slot used
      for (int i = 0; i < kStagedStages && i < issued; ++i)
        tcdev::mbar_wait(&B->full[i], static_cast<uint32_t>(((issued - 1 - i) / kStagedStages) & 1), B, err, false);
    }
  } else {
  for (int64_t st = warp; st < nst; st += kStagedWarps) {
    const int slot = static_cast<int>(st % kStagedStages);
    const int64_t use = st / kStagedStages;
    if (!__all_sync(0xffffffffu, tcdev::mbar_wait(&B->full[slot], static_cast<uint32_t>(use & 1), B, err))) break;
    const int64_t p0 = p_begin + st * kSP;
    const int np = static_cast<int>(min(static_cast<int64_t>(kSP), p_end - p0));
    const float* stage = reinterpret_cast<const float*>(sm + slot * kStagedBytes);
    packdev::pack_stage_f4<kSP>(a, stage, p0, np, kTerms, kA, kOp == kXnor ? 0xAu : 0x0u, lane);
    __syncwarp();
    if (lane == 0) tcdev::mbar_arrive(&B->empty[slot]);  // the stage's input has been read
  }
  }
  __syncthreads();
  if (threadIdx.x == 0) BCONV_STAMP(2);
}

template <bool kTerms, bool kA, int kOp, int kStages>
cudaError_t launch_f4_staged_n(const PackI8Args& a, int sp, int ctas_per_sm, cudaStream_t s) {
  const int sms = current_sm_count();
  const int64_t stages = ceil_div(a.npix, sp);
  const int64_t ctas = std::min<int64_t>(static_cast<int64_t>(sms) * ctas_per_sm, stages);
  const int64_t per_cta = ceil_div(stages, ctas) * sp;
  const int grid = static_cast<int>(ceil_div(a.npix, per_cta));
  const int smem = kStages * kStagedBytes + static_cast<int>(sizeof(StagedBars));
  auto kern = sp == 8   ? pack_f4_staged_kernel<kTerms, kA, kOp, 8, kStages>
              : sp == 4 ? pack_f4_staged_kernel<kTerms, kA, kOp, 4, kStages>
              : sp == 2 ? pack_f4_staged_kernel<kTerms, kA, kOp, 2, kStages>
                        : pack_f4_staged_kernel<kTerms, kA, kOp, 1, kStages>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_overlapped(kern, dim3(grid), dim3((kStagedWarps + 1) * 32), smem, s, a, per_cta);
}

template <bool kTerms, bool kA, int kOp>
cudaError_t launch_f4_staged(const PackI8Args& a, cudaStream_t s) {
  const int sp_max = kStagedBytes / (4 * a.ni);  // >= 1 (checked by the caller)
  const int sp = sp_max >= 8 ? 8 : sp_max >= 4 ? 4 : sp_max >= 2 ? 2 : 1;
  const int64_t stages = ceil_div(a.npix, sp);
  if (stages < static_cast<int64_t>(current_sm_count()) * kFewStagesPerSm)
    return launch_f4_staged_n<kTerms, kA, kOp, kStagedStagesHalf>(a, sp, 2, s);
  return launch_f4_staged_n<kTerms, kA, kOp, kStagedStages>(a, sp, 1, s);
}

template <bool kTerms, bool kA, int kOp, bool kF4>
cudaError_t launch_i8_f(const PackI8Args& a, int chunks, dim3 grid, cudaStream_t s) {
  auto kern = chunks == 1   ? pack_i8_vec_kernel<kTerms, kA, kOp, 1, kF4>
              : chunks == 2 ? pack_i8_vec_kernel<kTerms, kA, kOp, 2, kF4>
              : chunks == 4 ? pack_i8_vec_kernel<kTerms, kA, kOp, 4, kF4>
                            : pack_i8_scalar_kernel<kTerms, kA, kOp, kF4>;
  return launch_overlapped(kern, grid, dim3(kPackThreads), 0, s, a);
}

template <bool kTerms, bool kA, int kOp>
cudaError_t launch_i8_t(const PackI8Args& a, int chunks, dim3 grid, cudaStream_t s) {
  return a.f4 ? launch_i8_f<kTerms, kA, kOp, true>(a, chunks, grid, s)
              : launch_i8_f<kTerms, kA, kOp, false>(a, chunks, grid, s);
}

template <bool kTerms, bool kA>
cudaError_t launch_i8_op(const PackI8Args& a, int chunks, dim3 grid, cudaStream_t s) {
  return a.op == kXnor ? launch_i8_t<kTerms, kA, kXnor>(a, chunks, grid, s)
                       : launch_i8_t<kTerms, kA, kAnd>(a, chunks, grid, s);
}

}  // namespace

cudaError_t launch_pack_i8(const PackI8Args& a, cudaStream_t s) {
  if (a.npix == 0) return cudaSuccess;
  const int sms = current_sm_count();
  const bool vec = (a.ni % 4) == 0 && (reinterpret_cast<uintptr_t>(a.in) & 15) == 0 &&
                   (!a.in_scale || ((reinterpret_cast<uintptr_t>(a.in_scale) | reinterpret_cast<uintptr_t>(a.in_bias)) & 15) == 0);
  // e2m1 codes with up to 2048 channels a pixel: the staged (bulk-copy-fed) kernel
  if (vec && a.f4 && a.ni <= kStagedBytes / 4 && a.cip % 256 == 0) {
    if (a.in_scale)
      return a.A ? (a.op == kXnor ? launch_f4_staged<true, true, kXnor>(a, s) : launch_f4_staged<true, true, kAnd>(a, s))
                 : (a.op == kXnor ? launch_f4_staged<true, false, kXnor>(a, s) : launch_f4_staged<true, false, kAnd>(a, s));
    return a.A ? (a.op == kXnor ? launch_f4_staged<false, true, kXnor>(a, s) : launch_f4_staged<false, true, kAnd>(a, s))
               : (a.op == kXnor ? launch_f4_staged<false, false, kXnor>(a, s) : launch_f4_staged<false, false, kAnd>(a, s));
  }
  const int chunks = vec ? a.cip / 128 : 0;  // 1, 2, 4 -> vector kernel; anything else -> scalar
  int64_t blocks = ceil_div(a.npix, kPackThreads / 32);
  const int64_t cap = static_cast<int64_t>(sms) * (chunks ? 2 : 3);  // one wave
  if (blocks > cap) blocks = cap;
  const dim3 grid(static_cast<unsigned>(blocks));
  if (a.in_scale)
    return a.A ? launch_i8_op<true, true>(a, chunks, grid, s) : launch_i8_op<true, false>(a, chunks, grid, s);
  return a.A ? launch_i8_op<false, true>(a, chunks, grid, s) : launch_i8_op<false, false>(a, chunks, grid, s);
}


// ------------------------------------------------------------------------------------
// binaryWeights operand: three exact bf16 parts of x~ per channel.  A warp per pixel; a
// lane takes 2 consecutive channels per step (one 4-byte store per part).
// ------------------------------------------------------------------------------------
namespace {

__device__ __forceinline__ void split3_pair(float x0, float x1, uint32_t (&w)[3]) {
  split3_bf16x2(x0, x1, w[0], w[1], w[2]);
}

template <bool kTerms, bool kA>
__global__ void __launch_bounds__(kPackThreads) pack_bf16x3_kernel(PackBf16x3Args a) {
  wait_prior_grid();
  allow_next_grid();
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kPackThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kPackThreads) >> 5;
  const int ni = a.ni, cip = a.cip;
  for (int64_t p = warp; p < a.npix; p += nwarps) {
    const float* row = a.in + p * ni;
    uint16_t* prow = a.parts + p * 3 * cip;
    float asum = 0.f;
    for (int f0 = 0; f0 < cip; f0 += 64) {
      const int f = f0 + lane * 2;  // channels f, f+1
      float x0 = 0.f, x1 = 0.f;
      if (f < ni) {
        x0 = __ldcs(row + f);
        if (kTerms) x0 = fmaf(x0, __ldg(a.in_scale + f), __ldg(a.in_bias + f));
      }
      if (f + 1 < ni) {
        x1 = __ldcs(row + f + 1);
        if (kTerms) x1 = fmaf(x1, __ldg(a.in_scale + f + 1), __ldg(a.in_bias + f + 1));
      }
      if (kA) asum += fabsf(x0) + fabsf(x1);
      uint32_t w[3];
      split3_pair(x0, x1, w);
#pragma unroll
      for (int part = 0; part < 3; ++part) *reinterpret_cast<uint32_t*>(prow + part * cip + f) = w[part];
    }
    if (kA) {
      asum = warp_sum(asum);
      if (lane == 0) a.A[p] = asum / static_cast<float>(ni);
    }
  }
}

}  // namespace

// Vector path: kC chunks of 64 channels per pixel (compile-time 1, 2, 4 or 8), a group of
// 8 / kC pixels per warp step with all float2 loads issued first; lane l handles channels
// chunk*64 + 2l, 2l+1 and keeps their input terms in registers.
template <bool kTerms, bool kA, int kC>
__global__ void __launch_bounds__(kPackThreads, 3) pack_bf16x3_vec_kernel(PackBf16x3Args a) {
  wait_prior_grid();
  allow_next_grid();
  constexpr int kG = kC >= 8 ? 1 : 8 / kC;
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kPackThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kPackThreads) >> 5;
  const int ni = a.ni, cip = a.cip;
  const float* __restrict__ in = a.in;
  uint16_t* __restrict__ parts = a.parts;
  float2 sc[kC], bi[kC];
  bool live[kC];
#pragma unroll
  for (int c = 0; c < kC; ++c) {
    const int f = c * 64 + lane * 2;
    live[c] = f < ni;
    sc[c] = make_float2(1.f, 1.f);
    bi[c] = make_float2(0.f, 0.f);
    if (kTerms && live[c]) {
      sc[c] = __ldg(reinterpret_cast<const float2*>(a.in_scale + f));
      bi[c] = __ldg(reinterpret_cast<const float2*>(a.in_bias + f));
    }
  }
  for (int64_t p0 = warp * kG; p0 < a.npix; p0 += nwarps * kG) {
    float2 v[kG][kC];
#pragma unroll
    for (int g = 0; g < kG; ++g)
#pragma unroll
      for (int c = 0; c < kC; ++c) {
        const int64_t p = p0 + g;
        v[g][c] = (p < a.npix && live[c]) ? __ldcs(reinterpret_cast<const float2*>(in + p * ni + c * 64 + lane * 2))
                                          : make_float2(0.f, 0.f);
      }
#pragma unroll
    for (int g = 0; g < kG; ++g) {
      const int64_t p = p0 + g;
      if (p >= a.npix) break;  // warp-uniform
      uint16_t* prow = parts + p * 3 * cip;
      float asum = 0.f;
#pragma unroll
      for (int c = 0; c < kC; ++c) {
        float2 t = v[g][c];
        if (kTerms && live[c]) {
          t.x = fmaf(t.x, sc[c].x, bi[c].x);
          t.y = fmaf(t.y, sc[c].y, bi[c].y);
        }
        if (kA) asum += fabsf(t.x) + fabsf(t.y);
        uint32_t w[3];
        split3_pair(t.x, t.y, w);
        const int f = c * 64 + lane * 2;
#pragma unroll
        for (int part = 0; part < 3; ++part) *reinterpret_cast<uint32_t*>(prow + part * cip + f) = w[part];
      }
      if (kA) {
        asum = warp_sum(asum);
        if (lane == 0) a.A[p] = asum / static_cast<float>(ni);
      }
    }
  }
}

template <bool kTerms, bool kA>
cudaError_t launch_bf16x3_vec(const PackBf16x3Args& a, int chunks, dim3 grid, cudaStream_t s) {
  auto kern = chunks == 1   ? pack_bf16x3_vec_kernel<kTerms, kA, 1>
              : chunks == 2 ? pack_bf16x3_vec_kernel<kTerms, kA, 2>
              : chunks == 4 ? pack_bf16x3_vec_kernel<kTerms, kA, 4>
                            : pack_bf16x3_vec_kernel<kTerms, kA, 8>;
  return launch_overlapped(kern, grid, dim3(kPackThreads), 0, s, a);
}

cudaError_t launch_pack_bf16x3(const PackBf16x3Args& a, cudaStream_t s) {
  if (a.npix == 0) return cudaSuccess;
  const int sms = current_sm_count();
  const int chunks = a.cip / 64;
  const bool vec = (a.ni % 2) == 0 && (reinterpret_cast<uintptr_t>(a.in) & 7) == 0 &&
                   (!a.in_scale || ((reinterpret_cast<uintptr_t>(a.in_scale) | reinterpret_cast<uintptr_t>(a.in_bias)) & 7) == 0) &&
                   (chunks == 1 || chunks == 2 || chunks == 4 || chunks == 8);
  int64_t blocks = ceil_div(a.npix, kPackThreads / 32);
  const int64_t cap = static_cast<int64_t>(sms) * (vec ? 3 : 8);
  if (blocks > cap) blocks = cap;
  const dim3 grid(static_cast<unsigned>(blocks));
  if (vec) {
    if (a.in_scale) {
      return a.A ? launch_bf16x3_vec<true, true>(a, chunks, grid, s) : launch_bf16x3_vec<true, false>(a, chunks, grid, s);
    } else {
      return a.A ? launch_bf16x3_vec<false, true>(a, chunks, grid, s)
                 : launch_bf16x3_vec<false, false>(a, chunks, grid, s);
    }
    return cudaGetLastError();
  }
  auto kern = a.in_scale ? (a.A ? pack_bf16x3_kernel<true, true> : pack_bf16x3_kernel<true, false>)
                        : (a.A ? pack_bf16x3_kernel<false, true> : pack_bf16x3_kernel<false, false>);
  return launch_overlapped(kern, grid, dim3(kPackThreads), 0, s, a);
}

}  // namespace bconv

// ------------------------------------------------------------------------------------
// Bit-packed activations (a previous layer's binarized output) into the operand layouts
// of the contractions.  Input: u32 [npix][nw_in], channel c = bit c % 32 of word c / 32,
// nw_in = ceil(ni / 32); bits at or past ni are ignored.
// ------------------------------------------------------------------------------------
namespace bconv {
namespace {

// Four channels' codes from their four bits (bit j -> byte j): the multiply places bit j of n
// at bit 8j (and nowhere else inside the mask); XNOR turns 1 / 0 into 0x01 / 0xFF with no
// carries between bytes, AND keeps 1 / 0; bytes of channels past ni are 0.
template <int kOp>
__device__ __forceinline__ uint32_t codes_of_nibble(uint32_t n, int nvalid) {
  const uint32_t b = (n * 0x00204081u) & 0x01010101u;
  uint32_t c = kOp == kXnor ? ~(b * 0xFEu) : b;
  if (nvalid < 4) c &= nvalid <= 0 ? 0u : ((1u << (8 * nvalid)) - 1u);
  return c;
}

// One thread per 16 channels of a pixel: 16 code bytes as one 16-byte store.  Index math in
// 32 bits (the launcher checks that the chunk count fits).
template <int kOp>
__global__ void __launch_bounds__(256) unpack_bits_i8_kernel(const uint32_t* __restrict__ bits, uint32_t total,
                                                              uint32_t groups, int nw_in, int ni,
                                                              uint4* __restrict__ codes) {
  wait_prior_grid();
  allow_next_grid();
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    const uint32_t p = i / groups;
    const int c0 = static_cast<int>(i - p * groups) * 16;
    uint32_t half = 0;
    if (c0 < ni) half = (__ldg(bits + static_cast<size_t>(p) * nw_in + c0 / 32) >> (c0 & 16)) & 0xFFFFu;
    const int nv = ni - c0;
    codes[i] = make_uint4(codes_of_nibble<kOp>(half & 0xFu, nv), codes_of_nibble<kOp>((half >> 4) & 0xFu, nv - 4),
                          codes_of_nibble<kOp>((half >> 8) & 0xFu, nv - 8), codes_of_nibble<kOp>(half >> 12, nv - 12));
  }
}

// e2m1 codes of 8 channels (bits of `b`, LSB first) as 8 nibbles; nibbles at or past nvalid are 0.
template <int kOp>
__device__ __forceinline__ uint32_t f4_codes_of_byte(uint32_t b, int nvalid) {
  uint32_t x = b & 0xFFu;  // bit i -> bit 4i
  x = (x | (x << 12)) & 0x000F000Fu;
  x = (x | (x << 6)) & 0x03030303u;
  x = (x | (x << 3)) & 0x11111111u;
  uint32_t c = kOp == kXnor ? (0xAAAAAAAAu ^ (x * 8u)) : (x * 2u);  // 1 -> 0x2; 0 -> 0xA or 0
  if (nvalid < 8) c &= nvalid <= 0 ? 0u : ((1u << (4 * nvalid)) - 1u);
  return c;
}

// One thread per 32 channels of a pixel: 32 e2m1 codes (16 bytes) as one 16-byte store.
template <int kOp>
__global__ void __launch_bounds__(256) unpack_bits_f4_kernel(const uint32_t* __restrict__ bits, uint32_t total,
                                                              uint32_t groups, int nw_in, int ni,
                                                              uint4* __restrict__ codes, PadMap pad) {
  wait_prior_grid();
  allow_next_grid();
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    const uint32_t p = i / groups;
    const int g = static_cast<int>(i - p * groups);
    const int64_t o = pad(p) * groups + g;  // this 16-byte group's place in the code buffer
    const int c0 = g * 32;
    uint32_t word = 0;
    if (c0 < ni) word = __ldg(bits + static_cast<size_t>(p) * nw_in + g);
    const int nv = ni - c0;
    codes[o] = make_uint4(f4_codes_of_byte<kOp>(word, nv), f4_codes_of_byte<kOp>(word >> 8, nv - 8),
                          f4_codes_of_byte<kOp>(word >> 16, nv - 16), f4_codes_of_byte<kOp>(word >> 24, nv - 24));
  }
}

// One thread per output word: copy, clear the bits past ni, zero the padding words.
__global__ void __launch_bounds__(256) repack_bits_kernel(const uint32_t* __restrict__ bits, uint32_t total, int nw_in,
                                                           int ni, uint32_t nw_pad, uint32_t* __restrict__ out) {
  const int tail = ni % 32;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    const uint32_t p = i / nw_pad;
    const int w = static_cast<int>(i - p * nw_pad);
    uint32_t v = 0;
    if (w < nw_in) {
      v = __ldg(bits + static_cast<size_t>(p) * nw_in + w);
      if (w == nw_in - 1 && tail != 0) v &= (1u << tail) - 1u;
    }
    out[i] = v;
  }
}

// src [N][h][w] -> dst at the same pixels of a zero-bordered [N][hp][wp] grid.
__global__ void __launch_bounds__(256) pad_copy_kernel(const float* __restrict__ src, int64_t npix, PadMap pad,
                                                        float* __restrict__ dst) {
  wait_prior_grid();
  allow_next_grid();
  for (int64_t p = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; p < npix;
       p += static_cast<int64_t>(gridDim.x) * blockDim.x)
    dst[pad(p)] = __ldg(src + p);
}

unsigned grid_for(int64_t threads) {
  int64_t blocks = ceil_div(threads, 256);
  const int64_t cap = static_cast<int64_t>(current_sm_count()) * 8;
  return static_cast<unsigned>(blocks < cap ? blocks : cap);
}

}  // namespace

cudaError_t launch_unpack_bits_f4(const uint32_t* bits, int64_t npix, int ni, int cip, int op, int8_t* codes,
                                  cudaStream_t s, PadMap pad) {
  if (npix == 0) return cudaSuccess;
  const int64_t total = npix * (cip / 32);
  if (total >= (int64_t{1} << 31)) return cudaErrorInvalidValue;
  const uint32_t t = static_cast<uint32_t>(total), g = static_cast<uint32_t>(cip / 32);
  uint4* out = reinterpret_cast<uint4*>(codes);
  return launch_overlapped(op == kXnor ? unpack_bits_f4_kernel<kXnor> : unpack_bits_f4_kernel<kAnd>,
                           dim3(grid_for(total)), dim3(256), 0, s, bits, t, g, words_for(ni), ni, out, pad);
}

cudaError_t launch_unpack_bits_i8(const uint32_t* bits, int64_t npix, int ni, int cip, int op, int8_t* codes,
                                  cudaStream_t s) {
  if (npix == 0) return cudaSuccess;
  const int64_t total = npix * (cip / 16);
  if (total >= (int64_t{1} << 31)) return cudaErrorInvalidValue;
  const uint32_t t = static_cast<uint32_t>(total), g = static_cast<uint32_t>(cip / 16);
  uint4* out = reinterpret_cast<uint4*>(codes);
  return launch_overlapped(op == kXnor ? unpack_bits_i8_kernel<kXnor> : unpack_bits_i8_kernel<kAnd>,
                           dim3(grid_for(total)), dim3(256), 0, s, bits, t, g, words_for(ni), ni, out);
}

cudaError_t launch_pad_copy(const float* src, int64_t npix, PadMap pad, float* dst, cudaStream_t s) {
  if (npix == 0) return cudaSuccess;
  return launch_overlapped(pad_copy_kernel, dim3(grid_for(npix)), dim3(256), 0, s, src, npix, pad, dst);
}

cudaError_t launch_repack_bits(const uint32_t* bits, int64_t npix, int ni, int nw_pad, uint32_t* out, cudaStream_t s) {
  if (npix == 0) return cudaSuccess;
  const int64_t total = npix * nw_pad;
  if (total >= (int64_t{1} << 31)) return cudaErrorInvalidValue;
  repack_bits_kernel<<<grid_for(total), 256, 0, s>>>(bits, static_cast<uint32_t>(total), words_for(ni), ni,
                                                     static_cast<uint32_t>(nw_pad), out);
  return cudaGetLastError();
}

}  // namespace bconv

BCONV_TIMELINE_READER(bconv_timeline_pack)
