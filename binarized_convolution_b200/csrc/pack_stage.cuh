// The e2m1 pack of one staged run of pixels, shared by the bulk-copy-fed pack kernel and the
// pair convolution kernel that packs its own input; internal to the library.
//
// What it computes (Apple page "MPSCNNBinaryConvolution", Overview: the input terms are applied
// before binarization and before the beta image; bin(x) = x < 0 ? -1 : +1): per pixel and
// channel x~ = fma(x, inScale[c], inBias[c]), its e2m1 code (+1.0 = 0x2; -1.0 = 0xA for XNOR,
// 0 for AND; channels in [ni, cip) 0) and A = (sum_c |x~|) / ni, written at the pixel's place in
// the (possibly zero-bordered) code grid.
#pragma once

#include "common.cuh"
#include "tc_conv.cuh"

namespace bconv {
namespace packdev {

// The sums over the warp of kG values per lane, for kG pixels at once (kG = 1, 2, 4 or 8):
// halving exchanges first (offsets 16, 8, ... while a lane holds more than one value), then
// the plain butterfly.  Each pixel's total is formed by the same pairing tree as a butterfly
// over its own per-lane values, so it is bit-identical to one; lane l returns the total of
// pixel l / (32 / kG).
template <int kG>
__device__ __forceinline__ float warp_sum_multi(float (&v)[kG], int lane) {
  static_assert(kG == 1 || kG == 2 || kG == 4 || kG == 8, "pixels per step");
  constexpr int kLog = kG == 1 ? 0 : kG == 2 ? 1 : kG == 4 ? 2 : 3;
#pragma unroll
  for (int lvl = 0; lvl < kLog; ++lvl) {
    const int off = 16 >> lvl;
    const int n = kG >> (lvl + 1);  // values a lane keeps after this level
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int j = 0; j < n; ++j) {
      const float keep = upper ? v[j + n] : v[j];
      const float send = upper ? v[j] : v[j + n];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  float t = v[0];
#pragma unroll
  for (int off = 16 >> kLog; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
  return t;
}

// Pixels p0 .. p0 + np - 1 (np <= kSP), ni fp32 values each at stage + g * ni (shared memory),
// by one warp: lane l takes channels 8 l .. 8 l + 7 of each 256-channel pass (cip a multiple of
// 256), whose eight codes are one 32-bit store; one division for the first pixel's place in
// the grid, the others follow; one reduction forms the np values of A.  `terms`, `with_a` and
// `neg` (the code of -1) may be compile-time constants of the caller.
template <int kSP>
__device__ __forceinline__ void pack_stage_f4(const PackI8Args& a, const float* stage, int64_t p0, int np, bool terms,
                                              bool with_a, uint32_t neg, int lane) {
  const int ni = a.ni;
  const int npass = a.cip / 256;
  const int64_t pbytes = a.cip / 2;
  int64_t qs[kSP];
  {
    int py = 0, px = 0;
    a.pad.yx(p0, py, px);
    int64_t q = a.pad(p0);
#pragma unroll
    for (int g = 0; g < kSP; ++g) {
      qs[g] = q;
      if (g + 1 < kSP) q = a.pad.next(q, py, px);
    }
  }
  float asum[kSP];
#pragma unroll
  for (int g = 0; g < kSP; ++g) asum[g] = 0.f;
  for (int pass = 0; pass < npass; ++pass) {
    const int f0 = pass * 256 + 8 * lane;  // this lane's first channel
    const bool live0 = f0 < ni, live1 = f0 + 4 < ni;
    float4 sc0 = make_float4(1.f, 1.f, 1.f, 1.f), sc1 = sc0;
    float4 bi0 = make_float4(0.f, 0.f, 0.f, 0.f), bi1 = bi0;
    if (terms) {
      if (live0) {
        sc0 = __ldg(reinterpret_cast<const float4*>(a.in_scale + f0));
        bi0 = __ldg(reinterpret_cast<const float4*>(a.in_bias + f0));
      }
      if (live1) {
        sc1 = __ldg(reinterpret_cast<const float4*>(a.in_scale + f0 + 4));
        bi1 = __ldg(reinterpret_cast<const float4*>(a.in_bias + f0 + 4));
      }
    }
#pragma unroll
    for (int g = 0; g < kSP; ++g) {
      if (g >= np) break;  // warp-uniform
      float t[8];
      {
        const float4 u0 = live0 ? *reinterpret_cast<const float4*>(stage + g * ni + f0) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 u1 = live1 ? *reinterpret_cast<const float4*>(stage + g * ni + f0 + 4) : make_float4(0.f, 0.f, 0.f, 0.f);
        t[0] = u0.x; t[1] = u0.y; t[2] = u0.z; t[3] = u0.w;
        t[4] = u1.x; t[5] = u1.y; t[6] = u1.z; t[7] = u1.w;
      }
      if (terms) {
        t[0] = fmaf(t[0], sc0.x, bi0.x); t[1] = fmaf(t[1], sc0.y, bi0.y);
        t[2] = fmaf(t[2], sc0.z, bi0.z); t[3] = fmaf(t[3], sc0.w, bi0.w);
        t[4] = fmaf(t[4], sc1.x, bi1.x); t[5] = fmaf(t[5], sc1.y, bi1.y);
        t[6] = fmaf(t[6], sc1.z, bi1.z); t[7] = fmaf(t[7], sc1.w, bi1.w);
      }
      uint32_t word = 0u;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const bool ok = j < 4 ? live0 : live1;
        if (with_a && ok) asum[g] += fabsf(t[j]);
        word |= (ok ? ((t[j] < 0.f) ? neg : 0x2u) : 0u) << (4 * j);
      }
      *reinterpret_cast<uint32_t*>(a.codes + qs[g] * pbytes + pass * 128 + lane * 4) = word;
    }
  }
  if (with_a) {
    // lanes g * (32 / kSP) hold pixel g's sum
    const float total = warp_sum_multi<kSP>(asum, lane);
    const int g = lane / (32 / kSP);
    int64_t qa = qs[0];
#pragma unroll
    for (int j = 1; j < kSP; ++j)
      if (g == j) qa = qs[j];
    if ((lane % (32 / kSP)) == 0 && g < np) a.A[qa] = total / static_cast<float>(ni);
  }
}

}  // namespace packdev
}  // namespace bconv
