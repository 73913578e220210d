// Binary convolution on the tensor cores with the activation window held in shared memory:
// one load of a tile's input rows serves every tap of the window.
//
// What it computes is the same as tc_conv_kernel (Apple page "MPSCNNBinaryConvolution",
// Overview, XNOR and AND bullets): with e2m1 codes +1.0 / -1.0 (XNOR) or 1.0 / 0 (AND), every
// block scale 1.0 (tcgen05.mma kind::mxf4), each product is the operator's +-1 / 0 / 1 and
// the fp32 accumulator adds integers below 2^24 exactly, so the window sum S equals the
// per-word popcount forms bit for bit; out = act(S * scale[c] * beta + bias[c]).  Taps
// outside the image read zero codes and add 0.
//
// Layout.  The codes sit in a zero-bordered image: pixel (n, y, x) at padded position
// (n, y + kh/2, x + kw/2) of an [N][Hp][Wp] grid, Hp = H + kh - 1, Wp = W + kw - 1, each
// pixel a row of kb_per_tap 128-byte k-blocks.  Outputs are enumerated over the same grid
// (slot s = (n * Hp + oy) * Wp + ox; slots with oy >= H or ox >= W are junk), and output slot s,
// tap (ty, tx) reads padded pixel s + ty * Wp + tx.  A tile is 128 consecutive slots (junk
// slots are computed and never stored); per k-block the producer loads the tile's halo -- the
// 128 + (kh - 1) * Wp + kw - 1 rows starting at its first slot -- with one 2-D TMA box
// (128-byte swizzle), and the MMA of tap (ty, tx) reads the 128 rows starting ty * Wp + tx rows
// into it: the operand descriptor just starts further in (the swizzle follows the
// shared-memory address, which the copy used too).  A (the channel means of x~) lies in the
// same zero-bordered grid, so a slot's beta is the sum of the same shifted positions.

// Structure: a persistent kernel, one CTA per SM, 6 warps; each CTA works on one N tile of
// BN output channels.
//   warp 0      producer: the CTA's weights, once, when they fit ("resident": every
//               (tap, k-block) block of BN rows x 128 bytes, laid out already swizzled, issued
//               before the wait for the previous kernel since they do not depend on it);
//               then per tile and k-block one halo box into a 2-stage ring, and, when the
//               weights are streamed, one weight block per tap into a ring.
//   warp 1      allocates TMEM (two BN-column fp32 accumulators + the unit scale factors)
//               and, from one thread, issues kh * kw * kb_per_tap groups of four
//               tcgen05.mma.kind::mxf4 (M = 128, N = BN, K = 64 each) per tile.
//   warps 2-5   epilogue: tcgen05.ld 32 columns at a time, scale / bias / neuron in fp32;
//               each warp stages its 32 rows in its own 4 KB of shared memory (128-byte
//               swizzle) and reads them back so that each store instruction writes 4 output
//               rows x 128 contiguous bytes; junk rows are skipped.  No TMA store, and a chunk
//               never waits for another warp's stores.  Beta is formed ahead for a batch of
//               tiles at a time (the first batch while the first tile's MMAs run) from their
//               strips of A, staged through the same buffers.
// Every mbarrier wait gives up after one second of %globaltimer, sets the error word and
// makes all roles stop; TMEM is released on every exit path.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "tc_conv.cuh"
#include "tc_device.cuh"

namespace bconv {
namespace {

using namespace tcdev;

constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr int kHaloStages = 2;
constexpr int kMaxWStages = 8;
constexpr int kWarpStageBytes = 32 * 128;           // one epilogue warp's 32 rows x 32 fp32
constexpr int kAStrip = 1024;                        // longest halo (and strip of A) a tile reads
constexpr int kStripFloats = 4 * kWarpStageBytes / 4;  // strips of A staged in the epilogue's buffers
constexpr int kMaxTiles = 6;                         // tiles whose betas are formed in one batch
constexpr int kMinResidentBN = 128;                  // narrowest tile the plan narrows to

struct __align__(16) HaloBars {
  uint64_t hfull[kHaloStages];
  uint64_t hempty[kHaloStages];
  uint64_t wfull[kMaxWStages];
  uint64_t wempty[kMaxWStages];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t done;
  uint32_t tmem_base;
  uint32_t abort_flag;
  float2 sb[128];                // (scale, bias) of the CTA's output channels (BN <= 128)
  float betas[kMaxTiles * 128];  // beta of each row of the current batch of tiles
};

__global__ void __launch_bounds__(kThreads, 1)
    tc_halo_kernel(const __grid_constant__ CUtensorMap tmA, const HaloArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0u) {
    if (threadIdx.x == 0) atomicOr(a.err, kErrLayout);
    return;
  }
  const int taps = a.kh * a.kw;
  const int kb_total = taps * a.kb_per_tap;
  const int wblock = a.BN * 128;  // bytes of one (tap, k-block) weight block
  uint8_t* halo = smem_raw;
  uint8_t* wsm = halo + kHaloStages * a.halo_bytes;
  uint8_t* stage_out = wsm + (a.resident ? kb_total : a.wstages) * wblock;
  HaloBars* B = reinterpret_cast<HaloBars*>(stage_out + 4 * kWarpStageBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntile = static_cast<int>(blockIdx.x) % a.n_tiles;
  const int slot0 = static_cast<int>(blockIdx.x) / a.n_tiles;
  const int slots = static_cast<int>(gridDim.x) / a.n_tiles;
  const int8_t* wsrc = a.b_tiles + static_cast<int64_t>(ntile) * kb_total * wblock;

  if (threadIdx.x == 0) {
    BCONV_STAMP(0);
    for (int s = 0; s < kHaloStages; ++s) {
      mbar_init(&B->hfull[s], 1);
      mbar_init(&B->hempty[s], 1);
    }
    for (int s = 0; s < kMaxWStages; ++s) {
      mbar_init(&B->wfull[s], 1);
      mbar_init(&B->wempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&B->tmem_full[b], 1);
      mbar_init(&B->tmem_empty[b], kEpiThreads / 32);
    }
    mbar_init(&B->done, 1);
    B->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tensor_map(&tmA);
    if (a.resident && slot0 < a.m_tiles) {
      // the weights do not depend on the previous kernel: fetch them while it finishes
      mbar_expect_tx(&B->wfull[0], static_cast<uint32_t>(kb_total * wblock));
      for (int kb = 0; kb < kb_total; ++kb)
        bulk_load(wsm + kb * wblock, wsrc + static_cast<int64_t>(kb) * wblock, static_cast<uint32_t>(wblock),
                  &B->wfull[0]);
    }
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&B->tmem_base)),
                 "r"(a.tmem_cols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (warp >= 2) {  // this CTA's (scale, bias), static like the weights
    for (int j = threadIdx.x - 64; j < a.BN; j += kEpiThreads) {
      const int c = ntile * a.BN + j;
      B->sb[j] = c < a.No ? make_float2(__ldg(a.scale + c), __ldg(a.bias + c)) : make_float2(0.f, 0.f);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = B->tmem_base;
  // unit block scale factors (ue8m0 0x7F) in the 32 columns after the two accumulators
  const uint32_t sf_col = static_cast<uint32_t>(2 * a.BN);
  if (warp >= 2) tc_fill_32x32(tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16) + sf_col, 0x7F7F7F7Fu);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  wait_prior_grid();  // the codes, A and the output buffer belong to the previous kernels until here
  if (threadIdx.x == 0) BCONV_STAMP(1);

  const int rows_per_img = a.Hp * a.Wp;
  const int total_slots = a.N * rows_per_img;
  if (warp == 0) {
    // ---------------- producer ----------------
    if (lane == 0) {
      int hs = 0, ws = 0;
      uint32_t hphase = 0, wphase = 0;
      bool ok = true;
      for (int m = slot0; m < a.m_tiles && ok; m += slots) {
        const int row0 = m * 128;  // the tile's first slot
        for (int kb = 0; kb < a.kb_per_tap && ok; ++kb) {
          if (!mbar_wait(&B->hempty[hs], hphase ^ 1u, B, a.err)) {
            ok = false;
            break;
          }
          uint8_t* h = halo + hs * a.halo_bytes;
          mbar_expect_tx(&B->hfull[hs], static_cast<uint32_t>(a.halo_boxes * a.halo_rows * 128));
          for (int b = 0; b < a.halo_boxes; ++b)
            tma_load_2d(h + b * a.halo_rows * 128, &tmA, &B->hfull[hs], kb * 128, row0 + b * a.halo_rows);
          if (++hs == kHaloStages) {
            hs = 0;
            hphase ^= 1u;
          }
          if (!a.resident) {
            for (int tap = 0; tap < taps; ++tap) {
              if (!mbar_wait(&B->wempty[ws], wphase ^ 1u, B, a.err)) {
                ok = false;
                break;
              }
              mbar_expect_tx(&B->wfull[ws], static_cast<uint32_t>(wblock));
              bulk_load(wsm + ws * wblock, wsrc + static_cast<int64_t>(tap * a.kb_per_tap + kb) * wblock,
                        static_cast<uint32_t>(wblock), &B->wfull[ws]);
              if (++ws == a.wstages) {
                ws = 0;
                wphase ^= 1u;
              }
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int hs = 0, ws = 0, acc = 0, ti = 0;
      uint32_t hphase = 0, wphase = 0, acc_phase = 0;
      bool ok = slot0 >= a.m_tiles || !a.resident || mbar_wait(&B->wfull[0], 0, B, a.err);
      BCONV_STAMP(2);
      const uint32_t idesc = idesc_for(2, 128, a.BN);
      // descriptor start-address units are 16 bytes: a tap moves the A operand by whole 128-byte
      // rows (tx within a row, then Wp - kw + 1 rows on to the next window row) and the resident
      // B operand by one weight block per tap
      const uint64_t row_step = 128 >> 4, wrap_step = static_cast<uint64_t>(a.Wp - a.kw + 1) * (128 >> 4);
      const uint64_t wb_step = static_cast<uint64_t>(a.kb_per_tap) * wblock >> 4;
      // streamed weights: stage s's descriptor is the first one plus s blocks
      const uint64_t wdesc0 = smem_desc_sw128(wsm), wstage_step = static_cast<uint64_t>(wblock) >> 4;
      const uint32_t sfa = tmem_base + sf_col, sfb = tmem_base + sf_col + 16u;
      const int kw = a.kw;
      for (int m = slot0; m < a.m_tiles && ok; m += slots, ++ti) {
        if (!mbar_wait(&B->tmem_empty[acc], acc_phase ^ 1u, B, a.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * a.BN);
        for (int kb = 0; kb < a.kb_per_tap && ok; ++kb) {
          if (!mbar_wait(&B->hfull[hs], hphase, B, a.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (kb == 0 && ti < 8) BCONV_STAMP(3 + 2 * ti);
          // The issuing loops are kept free of anything but the MMAs and their descriptors: the
          // tensor pipe runs dry when the single issuing thread spends more than a few cycles
          // between MMAs (a branch holding an mbarrier wait in this loop, even never taken,
          // cost about half the pipe's rate).
          uint64_t da = smem_desc_sw128(halo + hs * a.halo_bytes);
          const uint32_t acc0 = kb > 0 ? 1u : 0u;
          if (a.resident) {
            uint64_t db = smem_desc_sw128(wsm + kb * wblock);
            int tx = 0;
            for (int tap = 0; tap < taps; ++tap) {
              tc_mma_f4(d_tmem, da, db, idesc, tap > 0 ? 1u : acc0, sfa, sfb);
              tc_mma_f4(d_tmem, da + 2u, db + 2u, idesc, 1u, sfa, sfb);
              tc_mma_f4(d_tmem, da + 4u, db + 4u, idesc, 1u, sfa, sfb);
              tc_mma_f4(d_tmem, da + 6u, db + 6u, idesc, 1u, sfa, sfb);
              db += wb_step;
              if (++tx == kw) {
                tx = 0;
                da += wrap_step;
              } else {
                da += row_step;
              }
            }
          } else {
            int tx = 0;
            for (int tap = 0; tap < taps; ++tap) {
              if (!mbar_wait(&B->wfull[ws], wphase, B, a.err)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint64_t db = wdesc0 + static_cast<uint64_t>(ws) * wstage_step;
              tc_mma_f4(d_tmem, da, db, idesc, tap > 0 ? 1u : acc0, sfa, sfb);
              tc_mma_f4(d_tmem, da + 2u, db + 2u, idesc, 1u, sfa, sfb);
              tc_mma_f4(d_tmem, da + 4u, db + 4u, idesc, 1u, sfa, sfb);
              tc_mma_f4(d_tmem, da + 6u, db + 6u, idesc, 1u, sfa, sfb);
              tc_commit(&B->wempty[ws]);
              if (++ws == a.wstages) {
                ws = 0;
                wphase ^= 1u;
              }
              if (++tx == kw) {
                tx = 0;
                da += wrap_step;
              } else {
                da += row_step;
              }
            }
          }
          if (!ok) break;
          tc_commit(&B->hempty[hs]);
          if (++hs == kHaloStages) {
            hs = 0;
            hphase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&B->tmem_full[acc]);
        if (ti < 8) BCONV_STAMP(4 + 2 * ti);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      // all MMAs issued by this thread have completed once `done` fires (waited even after an
      // abort, so that TMEM is never released under a running MMA)
      tc_commit(&B->done);
      mbar_wait(&B->done, 0, B, a.err, false, true);
      BCONV_STAMP(20);
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    // Each warp turns its 32 TMEM lanes (tile rows) into output rows 32 channels at a time:
    // raw rows into its own 4 KB of shared memory (16-byte chunk k of row r at k ^ (r % 8)),
    // then read back, with the terms applied, so that each store instruction writes 4 rows x
    // 128 contiguous bytes.
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;
    uint8_t* wst = stage_out + q * kWarpStageBytes;
    int acc = 0;
    uint32_t acc_phase = 0;
    const int et = threadIdx.x - 64;
    // betas are formed for a batch of tiles at a time, the first batch while the first tile's
    // MMAs run, through the (then idle) staging buffers
    const int batch = min(kMaxTiles, kStripFloats / a.halo_len);
    // Each warp moves on to the next tile as soon as its own stores are issued (no barrier
    // across the epilogue warps but tile_betas' own); after an abort a warp keeps walking the
    // tile list without waiting or storing, so that it still meets the others in tile_betas.
    bool ok = true;
    int ti = 0;
    for (int m = slot0; m < a.m_tiles; m += slots, ++ti) {
      const int s0 = m * 128;
      if (a.A && ti % batch == 0)
        tile_betas(a.A, total_slots, m, slots, min(batch, (a.m_tiles - m + slots - 1) / slots), a.halo_len,
                   a.kh, a.kw, a.Wp, reinterpret_cast<float*>(stage_out), B->betas, row, true, et, kEpiThreads);
      // the output rows this lane stores: rows 4i + lane / 8 of the warp's 32 (i = 0..7), and
      // their betas
      int64_t dst[8];
      float rb[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int sl = s0 + q * 32 + 4 * i + (lane >> 3);
        const int n = sl / rows_per_img, rem = sl - n * rows_per_img;
        const int oy = rem / a.Wp, ox = rem - oy * a.Wp;
        const bool ok = sl < total_slots && oy < a.H && ox < a.W;
        dst[i] = ok ? ((static_cast<int64_t>(n) * a.H + oy) * a.W + ox) * a.No : -1;
        rb[i] = a.A ? B->betas[(ti % batch) * 128 + q * 32 + 4 * i + (lane >> 3)] : 1.f;
      }
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&B->tmem_full[acc], acc_phase, B, a.err, true, true));
      if (!ok) {
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
        continue;
      }
      tc_fence_after();
      if (et == 0 && ti < 8) BCONV_STAMP(21 + 2 * ti);
      const uint32_t tbase =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * a.BN);
      for (int ch = 0; ch < a.BN / 32; ++ch) {
        uint32_t v[32];
        tc_ld_32x32(tbase + static_cast<uint32_t>(ch * 32), v);
        if (ch == a.BN / 32 - 1) {  // accumulator fully read: hand it back
          tc_fence_before();
          if (lane == 0) mbar_arrive(&B->tmem_empty[acc]);
        }
        // raw sums through the staging buffer; the terms are applied as they are read back,
        // where a lane holds 4 channels of 8 rows (two float4 loads of (scale, bias) per chunk)
        uint4* orow = reinterpret_cast<uint4*>(wst + lane * 128);
#pragma unroll
        for (int k = 0; k < 8; ++k) orow[k ^ (lane & 7)] = make_uint4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
        __syncwarp();
        const int cl = ch * 32 + 4 * (lane & 7);  // this lane's first channel in the tile
        const int c = ntile * a.BN + cl;
        if (c < a.No) {  // No % 4 == 0: a float4 of channels is all real or all padding
          const float4 p01 = *reinterpret_cast<const float4*>(&B->sb[cl]);      // (s0, b0, s1, b1)
          const float4 p23 = *reinterpret_cast<const float4*>(&B->sb[cl + 2]);  // (s2, b2, s3, b3)
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int r = 4 * i + (lane >> 3);
            const float4 sv = reinterpret_cast<const float4*>(wst + r * 128)[(lane & 7) ^ (r & 7)];
            const float beta = rb[i];
            float4 y;
            y.x = a.A ? fmaf(sv.x * p01.x, beta, p01.y) : fmaf(sv.x, p01.x, p01.y);
            y.y = a.A ? fmaf(sv.y * p01.z, beta, p01.w) : fmaf(sv.y, p01.z, p01.w);
            y.z = a.A ? fmaf(sv.z * p23.x, beta, p23.y) : fmaf(sv.z, p23.x, p23.y);
            y.w = a.A ? fmaf(sv.w * p23.z, beta, p23.w) : fmaf(sv.w, p23.z, p23.w);
            if (a.relu) {
              y.x = fmaxf(y.x, 0.f);
              y.y = fmaxf(y.y, 0.f);
              y.z = fmaxf(y.z, 0.f);
              y.w = fmaxf(y.w, 0.f);
            }
            if (dst[i] >= 0) *reinterpret_cast<float4*>(a.out + dst[i] + c) = y;
          }
        }
        __syncwarp();  // the rows are read before the next chunk overwrites them
      }
      if (et == 0 && ti < 8) BCONV_STAMP(22 + 2 * ti);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (et == 0) BCONV_STAMP(37);
  }

  tc_fence_before();
  __syncthreads();
  allow_next_grid();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(a.tmem_cols));
  }
}

}  // namespace

constexpr int kHaloSmemMax = 227 * 1024;

int tc_halo_smem_bytes(const HaloArgs& a) {
  const int taps = a.kh * a.kw;
  const int wbytes = (a.resident ? taps * a.kb_per_tap : a.wstages) * a.BN * 128;
  return kHaloStages * a.halo_bytes + wbytes + 4 * kWarpStageBytes + static_cast<int>(sizeof(HaloBars));
}

bool tc_halo_plan(HaloArgs& a, int sm_count) {
  if (a.BN < 32 || a.BN > 128 || a.BN % 32 != 0) return false;
  if (static_cast<int64_t>(a.N) * a.Hp * a.Wp + 1024 >= (int64_t{1} << 31)) return false;  // int32 slot indices
  // every row any tile's MMAs read: the 128 slots plus the window's reach
  a.halo_len = 128 + (a.kh - 1) * a.Wp + (a.kw - 1);
  if (a.halo_len > kAStrip) return false;  // at least four tiles' strips of A fit the staging
  a.m_tiles = static_cast<int>((static_cast<int64_t>(a.N) * a.Hp * a.Wp + 127) / 128);
  a.halo_boxes = (a.halo_len + 255) / 256;
  a.halo_rows = round_up((a.halo_len + a.halo_boxes - 1) / a.halo_boxes, 8);
  a.halo_bytes = round_up(a.halo_boxes * a.halo_rows * 128, 1024);
  const int taps = a.kh * a.kw;
  const int fixed = kHaloStages * a.halo_bytes + 4 * kWarpStageBytes + static_cast<int>(sizeof(HaloBars));
  // Resident weights are read from L2 once per CTA instead of once per tile: take the widest
  // tile, down to kMinResidentBN channels, whose weights fit beside the halos, else stream the
  // weights at the given width.  (Narrower MMAs cost about as much each as 128-channel ones --
  // the tensor core's time goes with reading the 128-row operand -- so narrowing below 128
  // channels loses more than it saves.)
  const int bn0 = a.BN;
  a.resident = 0;
  for (int bn = bn0; bn >= 32 && bn % 32 == 0 && (bn == bn0 || bn >= kMinResidentBN); bn /= 2) {
    if (fixed + taps * a.kb_per_tap * bn * 128 <= kHaloSmemMax) {
      a.BN = bn;
      a.resident = 1;
      break;
    }
  }
  if (!a.resident) a.BN = bn0;
  a.n_tiles = (a.No + a.BN - 1) / a.BN;
  const int wblock = a.BN * 128;
  a.wstages = a.resident ? 0 : std::min(kMaxWStages, (kHaloSmemMax - fixed) / wblock);
  if (!a.resident && a.wstages < 2) return false;
  uint32_t cols = 32;  // two accumulators and the 32 scale-factor columns, a power of two
  while (cols < static_cast<uint32_t>(2 * a.BN + 32)) cols <<= 1;
  a.tmem_cols = cols;
  // CTAs: a multiple of the N tiles (each CTA keeps one N tile), at most one per SM, and no
  // more per N tile than there are M tiles
  const int per_n = std::max(1, std::min(sm_count / a.n_tiles, a.m_tiles));
  a.grid_ctas = per_n * a.n_tiles;
  return true;
}

cudaError_t launch_tc_halo(const CUtensorMap* tmA, const HaloArgs& a, cudaStream_t s) {
  if (a.m_tiles == 0) return cudaSuccess;
  if (!a.b_tiles || !a.out || a.grid_ctas % a.n_tiles != 0 || (reinterpret_cast<uintptr_t>(a.out) & 15u) != 0)
    return cudaErrorInvalidValue;
  const int smem = tc_halo_smem_bytes(a);
  cudaError_t e = cudaFuncSetAttribute(tc_halo_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_overlapped(tc_halo_kernel, dim3(a.grid_ctas), dim3(kThreads), smem, s, *tmA, a);
}

}  // namespace bconv

BCONV_TIMELINE_READER(bconv_timeline_halo)
