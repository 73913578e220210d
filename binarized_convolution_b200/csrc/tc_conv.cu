// Binary convolution on the 5th-generation tensor cores (tcgen05.mma kind::i8, kind::mxf4 and,
// for binaryWeights, kind::f16).
//
// What it computes (Apple page "MPSCNNBinaryConvolution", Overview, XNOR and AND bullets):
// a product of two binarized values is +-1 (XNOR) or 0/1 (AND), so the window sum
//   S = sum_{valid taps, f} a(x~[f]) * w[f]
// is an exact integer dot product of int8 operands: XNOR codes a = bin(x~) in {-1,+1} and
// w in {-1,+1}; AND codes a, w in {0,1}.  With int32 accumulation the result equals the
// popcount form 32 - 2*popcount(x^y) (resp. popcount(x&y)) summed over the words, bit for
// bit.  Out-of-image taps and padding channels are zero codes, which add exactly 0, so no
// border correction is needed.  The same codes as e2m1 (fp4) values (+1.0, -1.0, 0) with every
// block scale 1.0 (kind::mxf4, kind 2) give the same products exactly, summed in fp32 -- exact
// for sums below 2^24.  The epilogue is out = act(S * scale[c] * beta + bias[c]).
// The fully-connected layer (page "MPSCNNFullyConnected") is the same contraction with one
// tap spanning the flattened image.
//
// Structure: a persistent kernel, one CTA per SM, 6 warps.
//   warp 0      producer: per k-block, one 128-row x 128-byte activation tile by TMA (a box
//               of Bn images x R rows x Cw columns of the int8 NHWC codes, shifted by the tap
//               offset; out-of-image coordinates read zeros; 128-byte swizzled) and one
//               BN x 128-byte weight block by a single bulk copy (laid out already swizzled),
//               into a ring of 4 stages guarded by mbarriers.  binaryWeights (kind::f16): the
//               stage holds the three bf16 parts of x~ for one 64-channel block against one
//               weight block, and the three parts' MMAs go into the same accumulator (2-3
//               stages fit).
//   warp 1      allocates TMEM (two BN-column int32 accumulators) and, from one thread,
//               issues tcgen05.mma M=128 x N=BN x K=32 per 32-byte step; tcgen05.commit frees
//               each stage and publishes each finished accumulator.
//   warps 2-5   epilogue: tcgen05.ld 32 columns at a time (one TMEM lane = one output
//               pixel), apply scale/beta/bias/neuron in fp32, stage through 128-byte
//               swizzled shared memory, and TMA-store the box (clipped at the tensor edges).
//               With a split reduction (the FC layer), the partial sums are instead added
//               into an fp32 workspace by TMA reduce-add (integers below 2^24 add exactly) and
//               a small kernel applies the epilogue.
//   binaryWeights straight from the fp32 input (TcArgs::f32): warp 0 loads each k-block's fp32
//   input as two boxes of 32 channels into the stage's first two part tiles, and the weight
//   block; eight more warps (6-13) read the boxes, form x~ and its three bf16 parts and
//   write them over the boxes (each warp rewrites exactly the rows it read); 3 stages fit.
//   When its tiles outnumber the CTAs, the CTAs take equal contiguous shares of all tiles'
//   k-blocks (ConvWork), and a tile cut between two CTAs is finished by the one holding its
//   first k-blocks, with the other's fp32 partial sums.
// Every mbarrier wait gives up after one second of %globaltimer, sets the error word and
// makes all roles stop; TMEM is released on every exit path.
#include <cuda.h>

#include "common.cuh"
#include "tc_bits.cuh"
#include "tc_conv.cuh"
#include "tc_device.cuh"

namespace bconv {
namespace {

using namespace tcdev;

constexpr int kStages = 4;     // kind 0 (48 KB stages at most)
constexpr int kMaxStages = 6;  // kinds 1 and 2: as many as fit
constexpr int kABytes = 128 * 128;  // 128 rows x 128 bytes
constexpr int kThreadsTc = 192;
constexpr int kEpiThreads = 128;
constexpr int kStageOutBytes = 128 * 128;  // 128 rows x 32 fp32
// binaryWeights from fp32 input: eight converting warps turn three stages' fp32 boxes into parts
constexpr int kConvWarps = 8;
constexpr int kThreadsF32 = kThreadsTc + 32 * kConvWarps;
constexpr int kF32PartStages = 3;

struct __align__(8) Barriers {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t xfull[kMaxStages];  // fp32 input: the stage's fp32 boxes have landed
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t done;
  uint32_t tmem_base;
  uint32_t abort_flag;
  float2 sb[256];  // (scale, bias) of the tile's output channels
};

struct TileCoord {
  int n0, oy0, ox0, ntile, split;
  int noff, bn;  // output channels [ntile*BN + noff, + bn) of this work item
  int mtile;     // M tile index
};

__device__ __forceinline__ TileCoord tile_coord(const TcArgs& a, int w) {
  TileCoord c;
  int t = w;
  c.noff = 0;
  c.bn = a.BN;
  if (w >= a.full_tiles) {  // a piece of a tail tile
    const int i = w - a.full_tiles;
    t = a.full_tiles + i / a.pieces;
    c.bn = a.BN / a.pieces;
    c.noff = (i % a.pieces) * c.bn;
  }
  c.split = t % a.k_splits;
  t /= a.k_splits;
  c.ntile = t % a.n_tiles;
  t /= a.n_tiles;
  c.mtile = t;
  const int tx = t % a.tiles_x;
  t /= a.tiles_x;
  const int ty = t % a.tiles_y;
  t /= a.tiles_y;
  c.n0 = t * a.Bn * a.mt;
  c.oy0 = ty * a.R;
  c.ox0 = tx * a.Cw;
  return c;
}

// A CTA's work list: (tile, k-block range) items.  Without a.sk, tiles blockIdx.x, + gridDim.x,
// ... with their split's k-blocks.  With a.sk (the fp32-input kernel when the tiles outnumber
// the CTAs), a contiguous, equal share of all tiles' k-blocks in tile order: a tile cut between
// CTA c and c + 1 has its first k-blocks as c's last item and the rest as c + 1's first item;
// c + 1 leaves its raw sums in sk_part[c] and raises sk_flag[c], c adds them and finishes the
// tile.  (Each share is at least a tile's k-blocks long, so no tile is cut twice.)
struct ConvWork {
  int64_t u, uend;
  int t, ti;
  __device__ ConvWork(const TcArgs& a, int total_tiles, int kb_total) : ti(0) {
    const int64_t U = static_cast<int64_t>(total_tiles) * kb_total;
    u = a.sk ? U * blockIdx.x / gridDim.x : 0;
    uend = a.sk ? U * (blockIdx.x + 1) / gridDim.x : 0;
    t = blockIdx.x;
  }
  __device__ bool next(const TcArgs& a, int total_tiles, int kb_total, int kb_per_split, int& tile, int& k0, int& k1) {
    if (!a.sk) {
      if (t >= total_tiles) return false;
      tile = t;
      k0 = tile_coord(a, t).split * kb_per_split;
      k1 = min(k0 + kb_per_split, kb_total);
      t += gridDim.x;
    } else {
      if (u >= uend) return false;
      tile = static_cast<int>(u / kb_total);
      k0 = static_cast<int>(u - static_cast<int64_t>(tile) * kb_total);
      k1 = static_cast<int>(min(static_cast<int64_t>(kb_total), k0 + (uend - u)));
      u += k1 - k0;
    }
    ++ti;
    return true;
  }
};

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_u32(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

template <bool kSplit, int kKind, bool kBits, bool kF32 = false>
__global__ void __launch_bounds__(kF32 ? kThreadsF32 : kThreadsTc, 1)
    tc_conv_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmOut,
                   const TcArgs a) {
  static_assert(!kF32 || (kKind == 1 && !kSplit && !kBits), "fp32 input: binaryWeights, fp32 output");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // The swizzled tiles need a 1024-byte aligned base, which the dynamic shared window has
  // when the kernel declares no static shared memory; anything else is refused before any
  // barrier, copy or TMEM allocation happens.
  if ((smem_u32(smem_raw) & 1023u) != 0u) {
    if (threadIdx.x == 0) atomicOr(a.err, kErrLayout);
    return;
  }
  uint8_t* smem = smem_raw;
  const int b_bytes = a.BN * 128;
  const int a_bytes = (kKind == 1 ? 3 : a.mt) * kABytes;  // kind 1: the three parts of x~
  const int stage_bytes = a_bytes + b_bytes;
  // kind 0 always fits kStages (a 48 KB stage at most); kinds 1 and 2 take what fits
  const int stages = kKind == 0 ? kStages : a.stages;
  uint8_t* stage_out = smem + stages * stage_bytes;  // 2 x 16 KB epilogue staging
  Barriers* B = reinterpret_cast<Barriers*>(stage_out + 2 * kStageOutBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total_tiles = a.full_tiles + (a.m_tiles * a.n_tiles * a.k_splits - a.full_tiles) * a.pieces;
  const int kb_total = a.kh * a.kw * a.kb_per_tap;
  const int kb_per_split = (kb_total + a.k_splits - 1) / a.k_splits;
  const uint32_t tmem_cols = a.tmem_cols;

  if (threadIdx.x == 0) {
    BCONV_STAMP(0);
    for (int s = 0; s < stages; ++s) {
      // fp32 input: the weights' copy and the eight converting warps complete a stage
      mbar_init(&B->full[s], kF32 ? 1 + kConvWarps : 1);
      mbar_init(&B->empty[s], 1);
      mbar_init(&B->xfull[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&B->tmem_full[b], 1);
      mbar_init(&B->tmem_empty[b], kEpiThreads / 32);
    }
    mbar_init(&B->done, 1);
    B->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&B->tmem_base)),
                 "r"(tmem_cols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = B->tmem_base;
  // kind 2: the block scale factors live in TMEM after the two accumulators, 16 columns for A
  // and 16 for B; every factor is 1.0 (ue8m0 0x7F), so the epilogue warps fill all 32 columns
  // of their lanes once and every MMA reads them in whatever arrangement it uses
  const uint32_t sf_col = static_cast<uint32_t>(2 * a.BN);
  if constexpr (kKind == 2) {
    if (warp >= 2) tc_fill_32x32(tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16) + sf_col, 0x7F7F7F7Fu);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  if (threadIdx.x == 0) {
    prefetch_tensor_map(&tmA);
    if (!kBits) prefetch_tensor_map(&tmOut);  // a bit-packed output never uses (or encodes) it
  }
  wait_prior_grid();  // the codes, A and the output buffer are the previous kernels' business until here
  if (threadIdx.x == 0) BCONV_STAMP(1);

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      ConvWork wk(a, total_tiles, kb_total);
      int t, kb0, kb1;
      while (ok && wk.next(a, total_tiles, kb_total, kb_per_split, t, kb0, kb1)) {
        const TileCoord tc = tile_coord(a, t);
        for (int kb = kb0; kb < kb1; ++kb) {
          if constexpr (kF32) {
            // the fp32 input of the k-block as two boxes of 32 channels (128-byte rows, 128-byte
            // swizzle) over the stage's hi and mid tiles, for the converting warps; the weights
            if (!mbar_wait(&B->empty[stage], phase ^ 1u, B, a.err)) {
              ok = false;
              break;
            }
            if (wk.ti == 1 && kb - kb0 < 8) BCONV_STAMP(56 + kb - kb0);
            uint8_t* sa = smem + stage * stage_bytes;
            mbar_expect_tx(&B->xfull[stage], static_cast<uint32_t>(2 * kABytes));
            const int tap = kb / a.kb_per_tap, cb = kb - tap * a.kb_per_tap;
            const int ky = tap / a.kw, kx = tap - ky * a.kw;
            for (int h = 0; h < 2; ++h)
              tma_load_4d(sa + h * kABytes, &tmA, &B->xfull[stage], cb * 64 + h * 32, tc.ox0 * a.sx + kx - a.kw / 2,
                          tc.oy0 * a.sy + ky - a.kh / 2, tc.n0);
            mbar_expect_tx(&B->full[stage], static_cast<uint32_t>(tc.bn * 128));
            bulk_load(smem + stage * stage_bytes + a_bytes,
                      a.b_tiles + ((static_cast<int64_t>(tc.ntile) * kb_total + kb) * a.BN + tc.noff) * 128,
                      static_cast<uint32_t>(tc.bn * 128), &B->full[stage]);
            if (++stage == stages) {
              stage = 0;
              phase ^= 1u;
            }
            continue;
          }
          if (!mbar_wait(&B->empty[stage], phase ^ 1u, B, a.err)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * stage_bytes;
          uint8_t* sb = sa + a_bytes;
          mbar_expect_tx(&B->full[stage], static_cast<uint32_t>(a_bytes + tc.bn * 128));
          const int tap = kb / a.kb_per_tap, cb = kb - tap * a.kb_per_tap;
          const int ky = tap / a.kw, kx = tap - ky * a.kw;
          if constexpr (kKind == 1) {
            for (int part = 0; part < 3; ++part)
              tma_load_4d(sa + part * kABytes, &tmA, &B->full[stage], act_x(cb, part, a.kb_px, a.px_bytes, a.part_bytes),
                          tc.ox0 * a.sx + kx - a.kw / 2, tc.oy0 * a.sy + ky - a.kh / 2, tc.n0);
          } else {
            for (int h = 0; h < a.mt; ++h)  // kind 0: k-blocks are consecutive 128-byte blocks
              tma_load_4d(sa + h * kABytes, &tmA, &B->full[stage], cb * 128, tc.ox0 * a.sx + kx - a.kw / 2,
                          tc.oy0 * a.sy + ky - a.kh / 2, tc.n0 + h * a.Bn);
          }
          // the weight stage is one contiguous, already swizzled block of bn rows
          bulk_load(sb, a.b_tiles + ((static_cast<int64_t>(tc.ntile) * kb_total + kb) * a.BN + tc.noff) * 128,
                    static_cast<uint32_t>(tc.bn * 128), &B->full[stage]);
          if (++stage == stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      ConvWork wk(a, total_tiles, kb_total);
      int t, kb0, kb1;
      while (ok && wk.next(a, total_tiles, kb_total, kb_per_split, t, kb0, kb1)) {
        const TileCoord tc = tile_coord(a, t);
        const uint32_t idesc = idesc_for(kKind, 128, tc.bn);
        if (!mbar_wait(&B->tmem_empty[acc], acc_phase ^ 1u, B, a.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * a.mt * a.BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&B->full[stage], phase, B, a.err)) {
            ok = false;
            break;
          }
          if (wk.ti == 1 && kb - kb0 < 18) BCONV_STAMP(12 + kb - kb0);
          tc_fence_after();
          uint8_t* sa = smem + stage * stage_bytes;
          const uint64_t db = smem_desc_sw128(sa + a_bytes);
          if constexpr (kKind == 1) {
            // the three parts of x~ against the same weight block, into one accumulator (fully
            // unrolled: the issuing thread must do nothing between MMAs but step descriptors)
            const uint64_t da0 = smem_desc_sw128(sa);
            const uint32_t acc0 = kb > kb0 ? 1u : 0u;
#pragma unroll
            for (int part = 0; part < 3; ++part) {
              const uint64_t da = da0 + static_cast<uint64_t>(part) * (kABytes >> 4);
#pragma unroll
              for (int j = 0; j < 4; ++j)  // four 32-byte K steps across the 128-byte row
                tc_mma_bf16(d_tmem, da + 2u * j, db + 2u * j, idesc, (part > 0 || j > 0) ? 1u : acc0);
            }
          } else if constexpr (kKind == 2) {
            const uint64_t da = smem_desc_sw128(sa);
#pragma unroll
            for (int j = 0; j < 4; ++j) {  // four 32-byte (64-code) K steps across the 128-byte row
              const uint32_t accum = (kb > kb0 || j > 0) ? 1u : 0u;
              tc_mma_f4(d_tmem, da + 2u * j, db + 2u * j, idesc, accum, tmem_base + sf_col, tmem_base + sf_col + 16u);
            }
          } else {
            for (int h = 0; h < a.mt; ++h) {
              const uint64_t da = smem_desc_sw128(sa + h * kABytes);
#pragma unroll
              for (int j = 0; j < 4; ++j) {  // four 32-byte K steps across the 128-byte row
                const uint32_t accum = (kb > kb0 || j > 0) ? 1u : 0u;
                tc_mma_i8(d_tmem + static_cast<uint32_t>(h * a.BN), da + 2u * j, db + 2u * j, idesc, accum);
              }
            }
          }
          tc_commit(&B->empty[stage]);
          if (++stage == stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&B->tmem_full[acc]);
        if (wk.ti <= 4) BCONV_STAMP(1 + wk.ti);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      // all MMAs issued by this thread have completed once `done` fires (waited even after an
      // abort, so that TMEM is never released under a running MMA)
      tc_commit(&B->done);
      mbar_wait(&B->done, 0, B, a.err, false, true);
    }
  } else if (kF32 && warp >= 6) {
    // ---------------- converting warps (fp32 input) ----------------
    // Warp 6 + w takes tile rows (pixels) 16 w .. 16 w + 15: lane l row 16 w + l % 16 and the
    // k-block's channels 32 (l / 16) .. + 31, i.e. row r of fp32 box l / 16, which lies in the
    // hi (box 0) or mid (box 1) tile of the stage.  A lane reads its 32 values, forms x~ =
    // fma(x, in_scale, in_bias) (0 for a tap outside the image or a channel >= Ni) and the three
    // bf16 parts, and once the whole warp has its values writes them into the part tiles in the
    // 128-byte-swizzled layout the MMAs read (8-channel piece m of row r at m ^ (r % 8)).  The
    // bytes a warp overwrites in the hi and mid tiles are exactly the rows it read from the
    // two boxes, so no other warp's reads are in the way.
    const int cw_ = warp - 6;
    const int r = cw_ * 16 + (lane & 15), half = lane >> 4;
    const int rc = a.R * a.Cw;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    ConvWork wk(a, total_tiles, kb_total);
    int t, kb0, kb1;
    while (ok && wk.next(a, total_tiles, kb_total, kb_per_split, t, kb0, kb1)) {
      const TileCoord tc = tile_coord(a, t);
      const int n = tc.n0 + r / rc, oy = tc.oy0 + (r / a.Cw) % a.R, ox = tc.ox0 + r % a.Cw;
      const bool row_ok = n < a.N && oy < a.Ho && ox < a.Wo;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_wait(&B->xfull[stage], phase, B, a.err))) {
          ok = false;
          break;
        }
        if (warp == 6 && lane == 0 && wk.ti == 1 && kb - kb0 < 8) BCONV_STAMP(30 + kb - kb0);
        uint8_t* sa = smem + stage * stage_bytes;
        float4 u[8];  // 16-byte chunk j of the row holds channels 4 j .. 4 j + 3 of this half
        {
          const uint8_t* fb = sa + half * kABytes + r * 128;
#pragma unroll
          for (int j = 0; j < 8; ++j) u[j] = *reinterpret_cast<const float4*>(fb + ((j ^ (r & 7)) * 16));
        }
        const int tap = kb / a.kb_per_tap, cb = kb - tap * a.kb_per_tap;
        const int ky = tap / a.kw, kx = tap - ky * a.kw;
        const int iy = oy * a.sy + ky - a.kh / 2, ix = ox * a.sx + kx - a.kw / 2;
        const bool in_img = row_ok && iy >= 0 && iy < a.H && ix >= 0 && ix < a.W;
        uint32_t hi[4][4], mid[4][4], lo[4][4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {  // channels 8 q .. 8 q + 7 of this half
          const int c = cb * 64 + half * 32 + 8 * q;
          float v[8] = {u[2 * q].x, u[2 * q].y, u[2 * q].z, u[2 * q].w,
                        u[2 * q + 1].x, u[2 * q + 1].y, u[2 * q + 1].z, u[2 * q + 1].w};
          const bool live0 = in_img && c < a.Ni, live1 = in_img && c + 4 < a.Ni;
          if (a.in_scale) {
            if (live0) {
              const float4 s4 = __ldg(reinterpret_cast<const float4*>(a.in_scale + c));
              const float4 b4 = __ldg(reinterpret_cast<const float4*>(a.in_bias + c));
              v[0] = fmaf(v[0], s4.x, b4.x); v[1] = fmaf(v[1], s4.y, b4.y);
              v[2] = fmaf(v[2], s4.z, b4.z); v[3] = fmaf(v[3], s4.w, b4.w);
            }
            if (live1) {
              const float4 s4 = __ldg(reinterpret_cast<const float4*>(a.in_scale + c + 4));
              const float4 b4 = __ldg(reinterpret_cast<const float4*>(a.in_bias + c + 4));
              v[4] = fmaf(v[4], s4.x, b4.x); v[5] = fmaf(v[5], s4.y, b4.y);
              v[6] = fmaf(v[6], s4.z, b4.z); v[7] = fmaf(v[7], s4.w, b4.w);
            }
          }
          // out-of-image taps and channels >= Ni read zeros from the box (a row past the output
          // reads some other pixel, whose sums are never stored), but the terms would turn
          // them into in_bias
          if (a.in_scale) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              if (!(j < 4 ? live0 : live1)) v[j] = 0.f;
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) split3_bf16x2(v[2 * j], v[2 * j + 1], hi[q][j], mid[q][j], lo[q][j]);
        }
        __syncwarp();  // every lane has read its values before any lane overwrites the boxes
        uint8_t* db = sa + r * 128;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int pos = ((half * 4 + q) ^ (r & 7)) * 16;
          *reinterpret_cast<uint4*>(db + pos) = make_uint4(hi[q][0], hi[q][1], hi[q][2], hi[q][3]);
          *reinterpret_cast<uint4*>(db + kABytes + pos) = make_uint4(mid[q][0], mid[q][1], mid[q][2], mid[q][3]);
          *reinterpret_cast<uint4*>(db + 2 * kABytes + pos) = make_uint4(lo[q][0], lo[q][1], lo[q][2], lo[q][3]);
        }
        fence_proxy_async();  // the parts (generic stores) before the MMAs read them (async proxy)
        __syncwarp();
        if (lane == 0) mbar_arrive(&B->full[stage]);
        if (warp == 6 && lane == 0 && wk.ti == 1 && kb - kb0 < 8) BCONV_STAMP(38 + kb - kb0);
        if (++stage == stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;
    const int et = threadIdx.x - 64;  // 0..127 within the epilogue group
    int acc = 0;
    uint32_t acc_phase = 0;
    int chunk_count = 0;
    int loaded_ntile = -1;
    const int rc = a.R * a.Cw;
    // bit-packed output: the next layer's terms and a flag live in the unused staging area
    constexpr bool bits_out = kBits && !kSplit;
    float2* next_t = reinterpret_cast<float2*>(stage_out);
    uint32_t* bits_flag = reinterpret_cast<uint32_t*>(stage_out + kStageOutBytes);
    ConvWork wk(a, total_tiles, kb_total);
    int t, ek0, ek1;
    while (wk.next(a, total_tiles, kb_total, kb_per_split, t, ek0, ek1)) {
      const TileCoord tc = tile_coord(a, t);
      if (kF32 && a.sk && ek0 > 0) {
        // the later k-blocks of a tile that CTA blockIdx.x - 1 finishes: leave the raw sums
        if (!epi_all(mbar_wait(&B->tmem_full[acc], acc_phase, B, a.err, true, true))) break;
        tc_fence_after();
        uint32_t* part = a.sk_part + static_cast<size_t>(blockIdx.x - 1) * a.BN * 128;
        const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * a.BN);
        for (int ch = 0; ch < tc.bn / 32; ++ch) {
          uint32_t v[32];
          tc_ld_32x32(tb + static_cast<uint32_t>(ch * 32), v);
          if (ch == tc.bn / 32 - 1) {
            tc_fence_before();
            if (lane == 0) mbar_arrive(&B->tmem_empty[acc]);
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) part[(ch * 32 + j) * 128 + row] = v[j];  // lanes write 128-byte rows
        }
        __threadfence();
        epi_barrier();
        if (et == 0) st_release_u32(a.sk_flag + blockIdx.x - 1, 1u);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
        continue;
      }
      const bool sk_owner = kF32 && a.sk && ek1 < kb_total;  // CTA blockIdx.x + 1 has the rest
      if (!kSplit && tc.ntile != loaded_ntile) {  // this tile's (scale, bias) into shared memory
        epi_barrier();
        for (int j = et; j < a.BN; j += kEpiThreads) {
          const int c = tc.ntile * a.BN + j;
          B->sb[j] = c < a.No ? make_float2(__ldg(a.scale + c), __ldg(a.bias + c)) : make_float2(0.f, 0.f);
          if (bits_out)
            next_t[j] = c < a.No ? make_float2(__ldg(a.next_scale + c), __ldg(a.next_bias + c)) : make_float2(0.f, 0.f);
        }
        epi_barrier();
        loaded_ntile = tc.ntile;
      }
      // beta of this thread's row in each sub-tile, formed before the accumulator is ready
      const bool has_beta = a.A != nullptr || a.beta != nullptr;
      float beta_h[2] = {1.f, 1.f};
      for (int h = 0; h < a.mt; ++h) {
        const int n = tc.n0 + h * a.Bn + row / rc, oy = tc.oy0 + (row / a.Cw) % a.R, ox = tc.ox0 + row % a.Cw;
        const bool valid = n < a.N && oy < a.Ho && ox < a.Wo;
        if (kSplit || !valid) continue;
        if (a.A) {
          // beta = sum of A over the in-image window / (kh*kw), in the order of the beta kernel
          const float* An = a.A + static_cast<int64_t>(n) * a.H * a.W;
          float s = 0.f;
          for (int dy = -(a.kh / 2); dy <= (a.kh - 1) / 2; ++dy) {
            const int y = oy * a.sy + dy;  // window centred on input (oy*sy, ox*sx)
            if (y < 0 || y >= a.H) continue;
            for (int dx = -(a.kw / 2); dx <= (a.kw - 1) / 2; ++dx) {
              const int x = ox * a.sx + dx;
              if (x < 0 || x >= a.W) continue;
              s += __ldg(An + static_cast<int64_t>(y) * a.W + x);
            }
          }
          beta_h[h] = s / static_cast<float>(a.kh * a.kw);
        } else if (a.beta) {
          beta_h[h] = __ldg(a.beta + (static_cast<int64_t>(n) * a.Ho + oy) * a.Wo + ox);
        }
      }
      const uint32_t* part = nullptr;
      if (sk_owner) {  // wait (bounded) for the raw sums of this tile's later k-blocks
        bool ready = true;
        if (et == 0) {
          const uint32_t* flag = a.sk_flag + blockIdx.x;
          const uint64_t t0 = globaltimer();
          while (ld_acquire_u32(flag) == 0u) {
            if (*reinterpret_cast<volatile uint32_t*>(&B->abort_flag) || globaltimer() - t0 > kTimeoutNs) {
              atomicOr(a.err, kErrTimeout);
              atomicExch(&B->abort_flag, 1u);
              ready = false;
              break;
            }
          }
        }
        if (!epi_all(ready)) break;
        __threadfence();
        part = a.sk_part + static_cast<size_t>(blockIdx.x) * a.BN * 128;
      }
      if (!epi_all(mbar_wait(&B->tmem_full[acc], acc_phase, B, a.err, true, true))) break;
      const int eti = wk.ti - 1;
      if (et == 0 && eti < 4) BCONV_STAMP(52 + eti);
      tc_fence_after();
      float bits_asum = 0.f;
      Words8 bits_w{};
      const int bits_n = tc.n0 + row / rc, bits_oy = tc.oy0 + (row / a.Cw) % a.R, bits_ox = tc.ox0 + row % a.Cw;
      const bool bits_valid = bits_n < a.N && bits_oy < a.Ho && bits_ox < a.Wo;
      const int64_t bits_pix = (static_cast<int64_t>(bits_n) * a.Ho + bits_oy) * a.Wo + bits_ox;
      for (int h = 0; h < a.mt; ++h) {
        const float beta = beta_h[h];
        const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                               static_cast<uint32_t>((acc * a.mt + h) * a.BN);
        for (int ch = 0; ch < tc.bn / 32; ++ch) {
          uint32_t v[32];
          tc_ld_32x32(tbase + static_cast<uint32_t>(ch * 32), v);
          if (h == a.mt - 1 && ch == tc.bn / 32 - 1) {  // accumulator fully read: hand it back
            tc_fence_before();
            if (lane == 0) mbar_arrive(&B->tmem_empty[acc]);
          }
          if (kF32 && part) {  // + the later k-blocks' sums, in this fixed order
#pragma unroll
            for (int j = 0; j < 32; ++j)
              v[j] = __float_as_uint(__uint_as_float(v[j]) + __uint_as_float(__ldcg(part + (ch * 32 + j) * 128 + row)));
          }
          const int buf = chunk_count & 1;
          ++chunk_count;
          uint8_t* so = stage_out + buf * kStageOutBytes;
          if (!bits_out) epi_barrier();  // the store that last read `so` has finished (waited below by et 0)
          const int c0 = tc.ntile * a.BN + tc.noff + ch * 32;
          float y[32];
          if (kSplit) {
#pragma unroll
            for (int j = 0; j < 32; ++j) y[j] = acc_value(kKind, v[j]);
          } else {
            const float4* sb4 = reinterpret_cast<const float4*>(&B->sb[tc.noff + ch * 32]);
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const float4 p = sb4[j / 2];  // (scale, bias) of channels j, j+1 (same for all lanes)
              const float s0 = acc_value(kKind, v[j]);
              const float s1 = acc_value(kKind, v[j + 1]);
              float r0 = has_beta ? fmaf(s0 * p.x, beta, p.y) : fmaf(s0, p.x, p.y);
              float r1 = has_beta ? fmaf(s1 * p.z, beta, p.w) : fmaf(s1, p.z, p.w);
              if (a.relu) {
                r0 = fmaxf(r0, 0.f);
                r1 = fmaxf(r1, 0.f);
              }
              y[j] = r0;
              y[j + 1] = r1;
            }
          }
          if (bits_out) {
            words_set(bits_w, ch, bits_chunk(y, next_t + tc.noff + ch * 32, min(32, a.No - c0), bits_asum));
            continue;
          }
          // 128-byte swizzled row: 16-byte chunk k of row r lives at chunk k ^ (r % 8)
          float4* orow = reinterpret_cast<float4*>(so + row * 128);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            orow[k ^ (row & 7)] = make_float4(y[4 * k], y[4 * k + 1], y[4 * k + 2], y[4 * k + 3]);
          fence_proxy_async();
          epi_barrier();
          if (et == 0) {
            if (c0 < a.No) {  // a box past the last channel would write nothing; skip it
              if (kSplit)
                tma_reduce_add_4d(&tmOut, so, c0, tc.ox0, tc.oy0, tc.n0 + h * a.Bn);
              else
                tma_store_4d(&tmOut, so, c0, tc.ox0, tc.oy0, tc.n0 + h * a.Bn);
            }
            bulk_commit();  // one group per chunk (possibly empty) keeps the buffer accounting
            bulk_wait_read_1();
          }
        }
      }
      if (bits_out) {
        const int w0 = (tc.ntile * a.BN + tc.noff) / 32;  // first word of this item
        if (bits_valid) words_store(a.out_bits + bits_pix * a.nwo + w0, bits_w, min(tc.bn / 32, a.nwo - w0));
        bits_finish_item(a, bits_pix, bits_valid, bits_asum, tc.mtile, tc.mtile, tc.ntile,
                         tc.ntile * a.pieces + tc.noff / tc.bn, bits_flag, et);
      }
      if (sk_owner) {  // every thread has read the partial sums: the slot is free for the next launch
        epi_barrier();
        if (et == 0) a.sk_flag[blockIdx.x] = 0u;
      }
      if (et == 0 && eti < 4) BCONV_STAMP(48 + eti);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (et == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  // only now may the next kernel's blocks be scheduled: launched at the start they would sit
  // beside this kernel's CTAs for its whole run, waiting for it, and take issue slots from it
  allow_next_grid();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(tmem_cols));
  }
}

// y = act(S * scale[c] * beta[n] + bias[c]) from the fp32 partial-sum workspace [N][No]; a block
// per 256 x 4 channels of one row n.  With beta, each block first forms beta[n] = sum over the
// image of A / (H*W) (the FC's window is the whole image; the same reduction as
// beta_image_mean_kernel, so every block of a row gets the same value).  Every workspace entry
// is zeroed once read, so the next forward's reduce-add starts from zero.
constexpr int kFinThreads = 256;
__global__ void __launch_bounds__(kFinThreads) tc_finalize_kernel(float4* __restrict__ ws, float4* __restrict__ out,
                                                                 const float* __restrict__ scale,
                                                                 const float* __restrict__ bias,
                                                                 const float* __restrict__ A, int hw, int no4,
                                                                 int relu) {
  wait_prior_grid();
  allow_next_grid();
  __shared__ float part[kFinThreads / 32];
  __shared__ float beta_s;
  const int chunks = (no4 + kFinThreads - 1) / kFinThreads;
  const int r = blockIdx.x / chunks, i0 = (blockIdx.x - r * chunks) * kFinThreads;
  float b = 1.f;
  if (A) {
    const float* Ar = A + static_cast<int64_t>(r) * hw;
    float acc = 0.f;
    for (int p = threadIdx.x; p < hw; p += kFinThreads) acc += __ldg(Ar + p);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x < 32) {
      acc = threadIdx.x < kFinThreads / 32 ? part[threadIdx.x] : 0.f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (threadIdx.x == 0) beta_s = acc / static_cast<float>(hw);
    }
    __syncthreads();
    b = beta_s;
  }
  const int i = i0 + threadIdx.x;
  if (i < no4) {
    const int64_t k = static_cast<int64_t>(r) * no4 + i;
    const float4 sv = ws[k];
    ws[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    const int c = i * 4;
    const float4 sc = __ldg(reinterpret_cast<const float4*>(scale + c));
    const float4 bi = __ldg(reinterpret_cast<const float4*>(bias + c));
    float4 y;
    if (A) {
      y = make_float4(fmaf(sv.x * sc.x, b, bi.x), fmaf(sv.y * sc.y, b, bi.y), fmaf(sv.z * sc.z, b, bi.z),
                      fmaf(sv.w * sc.w, b, bi.w));
    } else {
      y = make_float4(fmaf(sv.x, sc.x, bi.x), fmaf(sv.y, sc.y, bi.y), fmaf(sv.z, sc.z, bi.z),
                      fmaf(sv.w, sc.w, bi.w));
    }
    if (relu) y = make_float4(fmaxf(y.x, 0.f), fmaxf(y.y, 0.f), fmaxf(y.z, 0.f), fmaxf(y.w, 0.f));
    out[k] = y;
  }
}

}  // namespace

BCONV_TIMELINE_READER(bconv_timeline_tc)

constexpr int kSmemMax = 227 * 1024;  // dynamic shared memory one CTA may opt in to

int tc_stages(int kind, int bn, int mt) {
  const int stage = (kind == 1 ? 3 : mt) * kABytes + bn * 128;
  const int s = (kSmemMax - 2 * kStageOutBytes - static_cast<int>(sizeof(Barriers))) / stage;
  const int cap = kind == 0 ? kStages : kMaxStages;
  return s < cap ? s : cap;
}

int tc_smem_bytes(const TcArgs& a) {
  return a.stages * ((a.kind == 1 ? 3 : a.mt) * kABytes + a.BN * 128) + 2 * kStageOutBytes +
         static_cast<int>(sizeof(Barriers));
}

int tc_f32_stages(int bn) {
  const int stage = 3 * kABytes + bn * 128;
  const int fixed = 2 * kStageOutBytes + static_cast<int>(sizeof(Barriers));
  return bn <= 128 && fixed + kF32PartStages * stage <= kSmemMax ? kF32PartStages : 0;
}

int tc_plan(TcArgs& a, int sm_count) {
  const int tiles = a.m_tiles * a.n_tiles * a.k_splits;
  int grid = sm_count < tiles ? sm_count : tiles;
  a.full_tiles = tiles;
  a.pieces = 1;
  const int tail = grid > 0 ? tiles % grid : 0;
  if (a.k_splits == 1 && tiles > grid && tail > 0) {
    // cut each tail tile into the most 32-channel-multiple pieces that still fit one wave
    for (int p = a.BN / 32; p > 1; --p) {
      if ((a.BN / 32) % p == 0 && tail * p <= grid) {
        a.pieces = p;
        break;
      }
    }
    if (a.pieces > 1) a.full_tiles = tiles - tail;
  }
  return grid;
}

cudaError_t launch_tc_conv(const CUtensorMap* tmA, const CUtensorMap* tmOut, const TcArgs& a, cudaStream_t s) {
  if (a.stages < 2 || a.stages > (a.kind == 0 ? kStages : kMaxStages) || (a.kind != 0 && a.mt != 1) ||
      (a.kind == 0 && a.stages != kStages) || (a.kind == 2 && 2 * a.BN + 32 > static_cast<int>(a.tmem_cols)))
    return cudaErrorInvalidValue;
  if (a.f32 && (a.kind != 1 || a.k_splits != 1 || a.out_bits || a.stages != kF32PartStages || a.BN > 128 ||
                a.Ni % 4 != 0 || (a.in_scale && !a.in_bias)))
    return cudaErrorInvalidValue;
  // the balanced work list: the fp32-input kernel only, whole tiles (no pieces), a grid of
  // grid_ctas CTAs, all resident at once (one per SM), each with at least a tile's k-blocks
  if (a.sk && (!a.f32 || !a.sk_part || !a.sk_flag || a.pieces != 1 || a.grid_ctas < 1 ||
               a.grid_ctas > current_sm_count() || a.m_tiles * a.n_tiles < a.grid_ctas))
    return cudaErrorInvalidValue;
  const int smem = tc_smem_bytes(a);
  const int tiles = a.m_tiles * a.n_tiles * a.k_splits;
  if (tiles == 0) return cudaSuccess;
  int grid = current_sm_count();
  if (grid > tiles) grid = tiles;
  if (a.sk) grid = a.grid_ctas;  // the shares and the exchange slots were cut for this grid
  if ((a.out_bits && a.k_splits > 1) || !a.b_tiles) return cudaErrorInvalidValue;
  auto pick = [](auto k0, auto k1, auto k2, int kind) { return kind == 2 ? k2 : kind == 1 ? k1 : k0; };
  auto kern = a.k_splits > 1 ? pick(tc_conv_kernel<true, 0, false>, tc_conv_kernel<true, 1, false>,
                                    tc_conv_kernel<true, 2, false>, a.kind)
              : a.out_bits   ? pick(tc_conv_kernel<false, 0, true>, tc_conv_kernel<false, 1, true>,
                                    tc_conv_kernel<false, 2, true>, a.kind)
                             : pick(tc_conv_kernel<false, 0, false>, tc_conv_kernel<false, 1, false>,
                                    tc_conv_kernel<false, 2, false>, a.kind);
  if (a.f32) kern = tc_conv_kernel<false, 1, false, true>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_overlapped(kern, dim3(grid), dim3(a.f32 ? kThreadsF32 : kThreadsTc), smem, s, *tmA, *tmOut, a);
}

cudaError_t launch_tc_finalize(float* ws, float* out, const float* scale, const float* bias, const float* A, int hw,
                               int rows, int no, int relu, cudaStream_t s) {
  if (rows == 0 || no == 0) return cudaSuccess;
  const int chunks = (no / 4 + kFinThreads - 1) / kFinThreads;
  return launch_overlapped(tc_finalize_kernel, dim3(rows * chunks), dim3(kFinThreads), 0, s, reinterpret_cast<float4*>(ws),
                           reinterpret_cast<float4*>(out), scale, bias, A, hw, no / 4, relu);
}

}  // namespace bconv
