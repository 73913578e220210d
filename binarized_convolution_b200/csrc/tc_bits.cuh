// Bit-packed epilogue of the tensor-core kernels: the output in the form the next binary
// layer reads (Apple page "MPSCNNBinaryConvolution", Overview: the input terms act before
// binarization and before the beta image; bin(x) = x < 0 ? -1 : 1; A = mean over the
// channels of |x~|).  Internal to the library.
#pragma once

#include "tc_conv.cuh"
#include "tc_device.cuh"

namespace bconv {
namespace tcdev {

// One 32-channel chunk of one pixel: y[j] is the layer output of channel c0 + j and nt[j]
// the next layer's (in_scale, in_bias) for it; channels at or past `nvalid` are not real.
// Returns the sign word (bit j = 1 for x~ >= 0) and adds sum |x~| to `asum`.
__device__ __forceinline__ uint32_t bits_chunk(const float (&y)[32], const float2* nt, int nvalid, float& asum) {
  uint32_t word = 0;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    if (j < nvalid) {
      const float2 t = nt[j];
      const float xt = fmaf(y[j], t.x, t.y);
      word |= (xt < 0.f ? 0u : 1u) << j;
      asum += fabsf(xt);
    }
  }
  return word;
}

// The sign words of one pixel's work item (up to 8 chunks of 32 channels), held in registers.
struct Words8 {
  uint4 lo, hi;
};

__device__ __forceinline__ void words_set(Words8& w, int i, uint32_t v) {
  switch (i) {
    case 0: w.lo.x = v; break;
    case 1: w.lo.y = v; break;
    case 2: w.lo.z = v; break;
    case 3: w.lo.w = v; break;
    case 4: w.hi.x = v; break;
    case 5: w.hi.y = v; break;
    case 6: w.hi.z = v; break;
    default: w.hi.w = v; break;
  }
}

__device__ __forceinline__ uint32_t words_get(const Words8& w, int i) {
  switch (i) {
    case 0: return w.lo.x;
    case 1: return w.lo.y;
    case 2: return w.lo.z;
    case 3: return w.lo.w;
    case 4: return w.hi.x;
    case 5: return w.hi.y;
    case 6: return w.hi.z;
    default: return w.hi.w;
  }
}

// Store the first n (<= 8) words at dst: 16-byte stores when dst is 16-byte aligned and n is
// a multiple of 4 (one 32-byte sector per pixel for a 256-channel item), else word by word.
__device__ __forceinline__ void words_store(uint32_t* dst, const Words8& w, int n) {
  if ((reinterpret_cast<uintptr_t>(dst) & 15u) == 0 && (n & 3) == 0) {
    if (n >= 4) reinterpret_cast<uint4*>(dst)[0] = w.lo;
    if (n == 8) reinterpret_cast<uint4*>(dst)[1] = w.hi;
  } else {
    for (int i = 0; i < n; ++i) dst[i] = words_get(w, i);
  }
}

// Work items (slices of output channels) that cover M tile `mi` of the work list: tiles
// before `full_tiles` are whole, later ones come in `pieces` parts.
__device__ __forceinline__ int bits_slices_of(const TcArgs& a, int mi) {
  const int whole = min(max(a.full_tiles - mi * a.n_tiles, 0), a.n_tiles);
  return whole + (a.n_tiles - whole) * a.pieces;
}

// Called by all 128 epilogue threads after the last chunk of a work item: writes out_a of
// this thread's pixel, directly when the item holds all of the pixel's channels, else
// through the slice partials.  `mi` indexes the work list's M tiles (the pair kernel's
// pair tile), `mrow` the CTA's own M tile (the counter), `slice` = ntile * pieces + piece.
__device__ __forceinline__ void bits_finish_item(const TcArgs& a, int64_t pix, bool valid, float asum, int mi,
                                                 int mrow, int ntile, int slice, uint32_t* flag, int et) {
  const int64_t M = static_cast<int64_t>(a.N) * a.Ho * a.Wo;
  const int target = bits_slices_of(a, mi);
  const float no = static_cast<float>(a.No);
  (void)ntile;
  if (target == 1) {
    if (valid) a.out_a[pix] = asum / no;
    return;
  }
  if (valid) a.a_part[static_cast<int64_t>(slice) * M + pix] = asum;
  __threadfence();
  epi_barrier();
  if (et == 0) {
    const uint32_t old = atomicAdd(a.a_count + mrow, 1u);
    const bool last = old + 1u == static_cast<uint32_t>(target);
    if (last) a.a_count[mrow] = 0u;  // every item of this tile has arrived: ready for the next launch
    *reinterpret_cast<volatile uint32_t*>(flag) = last ? 1u : 0u;
  }
  epi_barrier();
  if (*reinterpret_cast<volatile uint32_t*>(flag)) {
    __threadfence();
    if (valid) {
      float s = 0.f;
      for (int nt = 0; nt < a.n_tiles; ++nt) {
        const bool whole = mi * a.n_tiles + nt < a.full_tiles;
        const int np = whole ? 1 : a.pieces;
        for (int p = 0; p < np; ++p) s += __ldcg(a.a_part + static_cast<int64_t>(nt * a.pieces + p) * M + pix);
      }
      a.out_a[pix] = s / no;
    }
  }
  epi_barrier();  // the flag is read by everyone before the next item may overwrite it
}

}  // namespace tcdev
}  // namespace bconv
