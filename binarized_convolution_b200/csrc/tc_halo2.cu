// Rows-staged binary convolution on SM pairs: tcgen05.mma.cta_group::2 kind::mxf4, M = 256 across
// two SMs, N = 256 output channels.
//
// What it computes is what tc_halo_kernel computes (Apple page "MPSCNNBinaryConvolution",
// Overview, XNOR and AND bullets; e2m1 codes +-1 / 0 with unit block scales, exact fp32 sums
// below 2^24; out = act(S * scale[c] * beta + bias[c])), with the same zero-bordered grid of
// codes and A, the same 128-slot tiles and the same halo: one load of a tile's rows serves every
// tap, whose MMA operand just starts ty * Wp + tx rows further into it.
//
// Why pairs: the tensor core's time per MMA goes with reading its 128-row A operand from shared
// memory, so it keeps pace only with 256 output channels per SM.  A cluster of two CTAs does
// that without doubling the weights each SM holds: each CTA keeps its own 128-slot tile's halo
// and half (128 rows) of the pair's 256-channel weight tile, the leader CTA's single thread
// issues M256 N256 K64 MMAs that read both CTAs' shared memory, and each CTA's TMEM receives its
// own 128 rows x 256 channels.  The weights stay resident in each CTA when its half fits
// (batch 16, 56x56, 256 -> 256, 3x3: 9 taps x 16 KB), else they stream through a ring.
//
// Roles (10 warps per CTA): warp 0 of each CTA loads its halos (and streamed weights) with TMA,
// completing on the leader's barriers (cta_group::2 copies); warp 1 of the leader issues the
// MMAs and releases halo stages, weight stages and the accumulator with commits multicast to
// both CTAs; warps 2-9 of each CTA (two per TMEM lane quarter, 128 columns each) read the
// accumulator into registers at once and hand it back -- there is room in TMEM for one 256-column
// accumulator and the scale factors only -- then apply beta, scale, bias and the neuron and
// store 32 channels x 16 rows at a time through 2 KB of shared memory per warp, so that every
// store instruction writes whole 128-byte lines (the SMs' write requests, not bytes, bound
// this epilogue).  Beta is formed ahead for a batch of tiles from their strips of A, staged
// through the same buffers while the first tile's MMAs run.  TMEM is allocated with
// cta_group::2 in both CTAs; the pair synchronises (cluster barrier) after set-up and before
// exit.  Every mbarrier wait gives up after one second of %globaltimer, sets the error word and
// makes all roles stop; TMEM is released on every exit path.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "tc_conv.cuh"
#include "tc_device.cuh"

namespace bconv {
namespace {

using namespace tcdev;

constexpr int kThreads = 320;
constexpr int kEpiThreads = 256;
constexpr int kHaloStages = 2;
constexpr int kMaxWStages = 10;
constexpr int kBN = 256;                       // output channels per pair item
constexpr int kHalfRows = kBN / 2;             // weight rows each CTA holds
constexpr int kWBlock = kHalfRows * 128;       // one (tap, k-block) weight block of one CTA: 16 KB
constexpr int kOutCols = 32;                   // output channels per epilogue chunk: 128-byte row pieces
constexpr int kStageRows = 16;                 // rows staged at a time (half a warp's 32)
constexpr int kWarpStage = kStageRows * kOutCols * 4;  // 2 KB per epilogue warp
constexpr int kAStrip = 1024;                  // longest halo (and strip of A) a tile reads
constexpr int kStripFloats = 8 * kWarpStage / 4;  // strips of A staged in the epilogue's buffers
constexpr int kMaxTiles = 4;                   // tiles whose betas are formed in one batch
constexpr uint32_t kTmemCols = 512;            // the accumulator (256) and 64 scale-factor columns

struct __align__(16) PairHaloBars {
  uint64_t hfull[kHaloStages];   // leader: both CTAs' halo copies
  uint64_t hempty[kHaloStages];  // both CTAs (multicast commit)
  uint64_t wfull[kMaxWStages];   // leader: both CTAs' weight copies (resident weights: [0])
  uint64_t wempty[kMaxWStages];  // both CTAs (multicast commit)
  uint64_t tmem_full;            // both CTAs (multicast commit)
  uint64_t tmem_empty;           // leader: 8 epilogue warps x 2 CTAs
  uint64_t done;                 // both CTAs: every MMA of the pair has completed
  uint32_t tmem_base;
  uint32_t abort_flag;
  float2 sb[kBN];                // (scale, bias) of the pair's 256 output channels
  float betas[kMaxTiles * 128];  // beta of each row of the current batch of this CTA's tiles
};

__global__ void __launch_bounds__(kThreads, 1)
    tc_halo2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const HaloArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0u) {  // same in both CTAs: both leave before any set-up
    if (threadIdx.x == 0) atomicOr(a.err, kErrLayout);
    return;
  }
  const int taps = a.kh * a.kw;
  const int kb_total = taps * a.kb_per_tap;
  // the same layout in both CTAs: the leader's descriptors address both
  uint8_t* halo = smem_raw;
  uint8_t* wsm = halo + kHaloStages * a.halo_bytes;
  uint8_t* stage_out = wsm + (a.resident ? kb_total : a.wstages) * kWBlock;
  PairHaloBars* B = reinterpret_cast<PairHaloBars*>(stage_out + 8 * kWarpStage);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = static_cast<int>(blockIdx.x) >> 1, npairs = static_cast<int>(gridDim.x) >> 1;
  const int ntile = pair % a.n_tiles;          // each pair keeps one N tile
  const int pslot0 = pair / a.n_tiles, pslots = npairs / a.n_tiles;
  const int pair_tiles = (a.m_tiles + 1) / 2;  // a pair tile = this CTA's M tile 2 p + rank

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
    mbar_init(&B->tmem_full, 1);
    mbar_init(&B->tmem_empty, 2 * kEpiThreads / 32);
    mbar_init(&B->done, 1);
    B->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tensor_map(&tmA);
    prefetch_tensor_map(&tmB);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&B->tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  if (warp >= 2) {
    for (int j = threadIdx.x - 64; j < kBN; j += kEpiThreads) {
      const int c = ntile * kBN + j;
      B->sb[j] = c < a.No ? make_float2(__ldg(a.scale + c), __ldg(a.bias + c)) : make_float2(0.f, 0.f);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = B->tmem_base;
  const uint32_t sf_col = static_cast<uint32_t>(kBN);  // 64 columns of unit scale factors (ue8m0 0x7F)
  if (warp >= 2) {
    const uint32_t lanes = static_cast<uint32_t>((warp & 3) * 32) << 16;
    tc_fill_32x32(tmem_base + lanes + sf_col + static_cast<uint32_t>(((warp - 2) >> 2) * 32), 0x7F7F7F7Fu);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers and scale factors exist before any copy, MMA or commit crosses
  tc_fence_after();
  if (threadIdx.x == 0 && a.resident && pslot0 < pair_tiles) {
    // the weights do not depend on the previous kernel: fetch them while it finishes
    if (leader) mbar_expect_tx(&B->wfull[0], static_cast<uint32_t>(2 * kb_total * kWBlock));
    const uint32_t wfull_leader = mapa(&B->wfull[0], 0);
    for (int kb = 0; kb < kb_total; ++kb)
      tma_load_2d_pair(wsm + kb * kWBlock, &tmB, wfull_leader, kb * 128,
                       ntile * kBN + static_cast<int>(rank) * kHalfRows);
  }
  wait_prior_grid();  // the codes, A and the output buffer belong to the previous kernels until here
  if (threadIdx.x == 0) BCONV_STAMP(1);

  const int rows_per_img = a.Hp * a.Wp;
  const int total_slots = a.N * rows_per_img;
  if (warp == 0) {
    // ---------------- producer (both CTAs) ----------------
    if (lane == 0) {
      int hs = 0, ws = 0;
      uint32_t hphase = 0, wphase = 0;
      bool ok = true;
      for (int pt = pslot0; pt < pair_tiles && ok; pt += pslots) {
        const int row0 = (2 * pt + static_cast<int>(rank)) * 128;  // past the end: zero rows, not stored
        for (int kb = 0; kb < a.kb_per_tap && ok; ++kb) {
          if (!mbar_wait(&B->hempty[hs], hphase ^ 1u, B, a.err)) {
            ok = false;
            break;
          }
          if (leader) mbar_expect_tx(&B->hfull[hs], static_cast<uint32_t>(2 * a.halo_boxes * a.halo_rows * 128));
          const uint32_t hfull_leader = mapa(&B->hfull[hs], 0);
          uint8_t* h = halo + hs * a.halo_bytes;
          for (int b = 0; b < a.halo_boxes; ++b)
            tma_load_2d_pair(h + b * a.halo_rows * 128, &tmA, hfull_leader, kb * 128, row0 + b * a.halo_rows);
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
              if (leader) mbar_expect_tx(&B->wfull[ws], static_cast<uint32_t>(2 * kWBlock));
              tma_load_2d_pair(wsm + ws * kWBlock, &tmB, mapa(&B->wfull[ws], 0), (tap * a.kb_per_tap + kb) * 128,
                               ntile * kBN + static_cast<int>(rank) * kHalfRows);
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
    // ---------------- MMA issuer (leader only) ----------------
    if (leader && lane == 0) {
      int hs = 0, ws = 0, ti = 0;
      uint32_t hphase = 0, wphase = 0;
      bool ok = pslot0 >= pair_tiles || !a.resident || mbar_wait(&B->wfull[0], 0, B, a.err);
      BCONV_STAMP(2);
      const uint32_t idesc = idesc_for(2, 256, kBN);
      // descriptor start-address units are 16 bytes: a tap moves the A operand by whole rows
      const uint64_t row_step = 128 >> 4, wrap_step = static_cast<uint64_t>(a.Wp - a.kw + 1) * (128 >> 4);
      const uint64_t wb_step = static_cast<uint64_t>(a.kb_per_tap) * kWBlock >> 4;
      const uint64_t wdesc0 = smem_desc_sw128(wsm);  // streamed weights: stage s is s blocks on
      const uint32_t sfa = tmem_base + sf_col, sfb = tmem_base + sf_col + 32u;
      const int kw = a.kw;
      for (int pt = pslot0; pt < pair_tiles && ok; pt += pslots, ++ti) {
        // the single accumulator: wait until both CTAs' epilogues have read the previous tile
        if (!mbar_wait(&B->tmem_empty, (ti & 1) ^ 1u, B, a.err)) break;
        tc_fence_after();
        for (int kb = 0; kb < a.kb_per_tap && ok; ++kb) {
          if (!mbar_wait(&B->hfull[hs], hphase, B, a.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (kb == 0 && ti < 8) BCONV_STAMP(3 + 2 * ti);
          // The issuing loops hold nothing but the MMAs and their descriptors: the tensor pipes
          // run dry when the single issuing thread spends more than a few cycles between MMAs.
          uint64_t da = smem_desc_sw128(halo + hs * a.halo_bytes);
          const uint32_t acc0 = kb > 0 ? 1u : 0u;
          if (a.resident) {
            uint64_t db = smem_desc_sw128(wsm + kb * kWBlock);
            int tx = 0;
            for (int tap = 0; tap < taps; ++tap) {
              tc_mma_f4_pair(tmem_base, da, db, idesc, tap > 0 ? 1u : acc0, sfa, sfb);
              tc_mma_f4_pair(tmem_base, da + 2u, db + 2u, idesc, 1u, sfa, sfb);
              tc_mma_f4_pair(tmem_base, da + 4u, db + 4u, idesc, 1u, sfa, sfb);
              tc_mma_f4_pair(tmem_base, da + 6u, db + 6u, idesc, 1u, sfa, sfb);
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
              const uint64_t db = wdesc0 + static_cast<uint64_t>(ws) * (kWBlock >> 4);
              tc_mma_f4_pair(tmem_base, da, db, idesc, tap > 0 ? 1u : acc0, sfa, sfb);
              tc_mma_f4_pair(tmem_base, da + 2u, db + 2u, idesc, 1u, sfa, sfb);
              tc_mma_f4_pair(tmem_base, da + 4u, db + 4u, idesc, 1u, sfa, sfb);
              tc_mma_f4_pair(tmem_base, da + 6u, db + 6u, idesc, 1u, sfa, sfb);
              tc_commit_pair(&B->wempty[ws]);
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
          tc_commit_pair(&B->hempty[hs]);
          if (++hs == kHaloStages) {
            hs = 0;
            hphase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair(&B->tmem_full);
        if (ti < 8) BCONV_STAMP(4 + 2 * ti);
      }
      tc_commit_pair(&B->done);  // fires in both CTAs once every MMA above has completed
    }
    if (lane == 0) mbar_wait(&B->done, 0, B, a.err, false, true);
    if (leader && lane == 0) BCONV_STAMP(20);
  } else {
    // ---------------- epilogue (warps 2..9, both CTAs) ----------------
    const int q = warp & 3;                   // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;         // columns [128 half, 128 half + 128)
    const int row = q * 32 + lane;            // TMEM lane = tile row
    const int et = threadIdx.x - 64;          // 0..255
    uint8_t* wst = stage_out + (warp - 2) * kWarpStage;
    const uint32_t empty_leader = mapa(&B->tmem_empty, 0);
    // betas are formed for a batch of tiles at a time, the first batch while the first tile's
    // MMAs run, through the (then idle) staging buffers
    const int batch = min(kMaxTiles, kStripFloats / a.halo_len);
    // Each warp moves on to the next tile as soon as its own stores are issued (no barrier
    // across the epilogue warps but tile_betas' own); after an abort a warp keeps walking the
    // tile list without waiting or storing, so that it still meets the others in tile_betas.
    bool ok = true;
    int ti = 0;
    for (int pt = pslot0; pt < pair_tiles; pt += pslots, ++ti) {
      const int s0 = (2 * pt + static_cast<int>(rank)) * 128;
      if (a.A && ti % batch == 0)
        tile_betas(a.A, total_slots, 2 * pt + static_cast<int>(rank), 2 * pslots,
                   min(batch, (pair_tiles - pt + pslots - 1) / pslots), a.halo_len, a.kh, a.kw, a.Wp,
                   reinterpret_cast<float*>(stage_out), B->betas, row, half == 0, et, kEpiThreads);
      // this lane's store rows: 4 i + lane / 8 of the warp's 32 (i = 0..7), 16 bytes each of 128;
      // their output pixels (N * H * W < 2^31), or -1 for junk slots
      int dst[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int sl = s0 + q * 32 + 4 * i + (lane >> 3);
        const int n = sl / rows_per_img, rem = sl - n * rows_per_img;
        const int oy = rem / a.Wp, ox = rem - oy * a.Wp;
        const bool ok = sl < total_slots && oy < a.H && ox < a.W;
        dst[i] = ok ? (n * a.H + oy) * a.W + ox : -1;
      }
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&B->tmem_full, ti & 1, B, a.err, true, true));
      if (!ok) continue;
      tc_fence_after();
      if (et == 0 && ti < 8) BCONV_STAMP(21 + 2 * ti);
      // the whole 128-column half of this warp's lanes into registers, then the accumulator back
      uint32_t v[128];
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(half * 128);
      tc_ld_32x32_nowait(tb, v);
      tc_ld_32x32_nowait(tb + 32u, v + 32);
      tc_ld_32x32_nowait(tb + 64u, v + 64);
      tc_ld_32x32_nowait(tb + 96u, v + 96);
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(empty_leader);
      // Raw sums go through the staging buffer; the terms are applied as they are read back,
      // where a lane holds 4 channels of 4 rows: its (scale, bias) pairs are two float4 loads
      // per chunk.
      const float* tb_beta = B->betas + (ti % batch) * 128 + q * 32 + (lane >> 3);
#pragma unroll
      for (int ch = 0; ch < 128 / kOutCols; ++ch) {
        const int cl = half * 128 + ch * kOutCols + 4 * (lane & 7);  // this lane's first channel in the tile
        const float4 p01 = *reinterpret_cast<const float4*>(&B->sb[cl]);      // (s0, b0, s1, b1)
        const float4 p23 = *reinterpret_cast<const float4*>(&B->sb[cl + 2]);  // (s2, b2, s3, b3)
        const int c = ntile * kBN + cl;
        // 16 rows at a time through the warp's 2 KB (16-byte piece k of row r at k ^ (r % 8)):
        // each store instruction then writes 4 rows x 128 contiguous bytes
#pragma unroll
        for (int h = 0; h < 32 / kStageRows; ++h) {
          if ((lane >> 4) == h) {
            uint4* orow = reinterpret_cast<uint4*>(wst + (lane & 15) * 128);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              orow[k ^ (lane & 7)] = make_uint4(v[ch * kOutCols + 4 * k], v[ch * kOutCols + 4 * k + 1],
                                                v[ch * kOutCols + 4 * k + 2], v[ch * kOutCols + 4 * k + 3]);
          }
          __syncwarp();
          if (c < a.No) {  // No % 4 == 0: a float4 of channels is all real or all padding
#pragma unroll
            for (int i = 0; i < kStageRows / 4; ++i) {
              const int r = 4 * i + (lane >> 3);
              const float4 sv = reinterpret_cast<const float4*>(wst + r * 128)[(lane & 7) ^ (r & 7)];
              const float beta = a.A ? tb_beta[4 * (h * (kStageRows / 4) + i)] : 1.f;
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
              const int d = dst[h * (kStageRows / 4) + i];
              if (d >= 0) *reinterpret_cast<float4*>(a.out + static_cast<int64_t>(d) * a.No + c) = y;
            }
          }
          __syncwarp();  // the rows are read before the next ones overwrite them
        }
      }
      if (et == 0 && ti < 8) BCONV_STAMP(22 + 2 * ti);
    }
    if (et == 0) BCONV_STAMP(37);
  }

  tc_fence_before();
  __syncthreads();
  allow_next_grid();
  cluster_sync();  // the peer is done with this CTA's barriers, shared memory and TMEM
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols));
  }
}

}  // namespace

constexpr int kPairSmemMax = 227 * 1024;

int tc_halo2_smem_bytes(const HaloArgs& a) {
  const int taps = a.kh * a.kw;
  return kHaloStages * a.halo_bytes + (a.resident ? taps * a.kb_per_tap : a.wstages) * kWBlock + 8 * kWarpStage +
         static_cast<int>(sizeof(PairHaloBars));
}

int tc_halo2_max_pairs(const HaloArgs& a) {
  const int smem = tc_halo2_smem_bytes(a);
  if (cudaFuncSetAttribute(tc_halo2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, tc_halo2_kernel, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

bool tc_halo2_plan(HaloArgs& a, int max_pairs) {
  if (a.No <= 128) return false;  // one SM's 128-channel tile covers the layer
  if (static_cast<int64_t>(a.N) * a.Hp * a.Wp + 1024 >= (int64_t{1} << 31)) return false;
  a.BN = kBN;
  a.n_tiles = (a.No + kBN - 1) / kBN;
  a.halo_len = 128 + (a.kh - 1) * a.Wp + (a.kw - 1);
  if (a.halo_len > kAStrip) return false;
  a.m_tiles = static_cast<int>((static_cast<int64_t>(a.N) * a.Hp * a.Wp + 127) / 128);
  a.halo_boxes = (a.halo_len + 255) / 256;
  a.halo_rows = round_up((a.halo_len + a.halo_boxes - 1) / a.halo_boxes, 8);
  a.halo_bytes = round_up(a.halo_boxes * a.halo_rows * 128, 1024);
  const int taps = a.kh * a.kw;
  const int fixed = kHaloStages * a.halo_bytes + 8 * kWarpStage + static_cast<int>(sizeof(PairHaloBars));
  a.resident = fixed + taps * a.kb_per_tap * kWBlock <= kPairSmemMax ? 1 : 0;
  a.wstages = a.resident ? 0 : std::min(kMaxWStages, (kPairSmemMax - fixed) / kWBlock);
  if (!a.resident && a.wstages < 2) return false;
  a.tmem_cols = kTmemCols;
  if (max_pairs <= 0) max_pairs = tc_halo2_max_pairs(a);
  const int pair_tiles = (a.m_tiles + 1) / 2;
  const int per_n = std::min(max_pairs / a.n_tiles, pair_tiles);  // each pair keeps one N tile
  if (per_n < 1) return false;
  a.grid_ctas = 2 * per_n * a.n_tiles;
  return true;
}

cudaError_t launch_tc_halo2(const CUtensorMap* tmA, const CUtensorMap* tmB, const HaloArgs& a, cudaStream_t s) {
  if (a.m_tiles == 0) return cudaSuccess;
  const int npairs = a.grid_ctas / 2;
  if (!a.out || npairs <= 0 || npairs % a.n_tiles != 0 || (reinterpret_cast<uintptr_t>(a.out) & 15u) != 0)
    return cudaErrorInvalidValue;
  const int smem = tc_halo2_smem_bytes(a);
  cudaError_t e = cudaFuncSetAttribute(tc_halo2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * npairs));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // may overlap the pack's tail
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, tc_halo2_kernel, *tmA, *tmB, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace bconv

BCONV_TIMELINE_READER(bconv_timeline_halo2)
