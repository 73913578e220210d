// The binary fully-connected layer on the tensor cores, 256 output channels per item.
//
// What it computes (page "MPSCNNFullyConnected", Overview and Note: the kernel is the whole
// source image and the result is the flattened (y, x, f) input vector times the weight matrix;
// the operator, terms, beta and neuron of page "MPSCNNBinaryConvolution", Overview): with e2m1
// codes +1.0 / -1.0 (XNOR) or 1.0 / 0 (AND) and unit block scales (tcgen05.mma kind::mxf4),
// every product is the operator's +-1 / 0 / 1 and the fp32 accumulators add integers below
// 2^24 exactly, so S equals the per-word popcount forms bit for bit; y = act(S * scale[c] *
// beta_n + bias[c]) with beta_n the mean of A over the image.
//
// Work: an item is 128 images x 256 output channels x a share of the k-blocks (the reduction is
// split so that the items fill the SMs once); one item per CTA, one 256-column fp32 accumulator
// in TMEM.  Per k-block a 128 x 128-byte box of activation codes and a 256 x 128-byte box of
// weight codes (both 128-byte swizzled) feed four M128 N256 K64 MMAs: the activations are read
// once per 256 channels, the weights once per 128 images.
//
// The epilogue stages the item's whole 128 x 256 tile in the idle stage memory and moves it by
// TMA.  A split item adds its exact partial sums into an fp32 workspace by TMA reduce-add
// (integers below 2^24 add exactly in any order); the last item of a tile to finish (an atomic
// count per tile, after proxy and memory fences) loads the tile's sums back, applies the
// epilogue with the betas the epilogue warps formed during the main loop, stores the output,
// zeroes the workspace and resets the count -- no separate finalize launch.  An unsplit item
// stores y itself.
//
// Roles (6 warps): warp 0 TMA producer (4-stage ring); warp 1 TMEM allocation and, from one
// thread, the MMAs; warps 2-5 the epilogue.  Every mbarrier wait gives up after one second of
// %globaltimer, sets the error word and makes all roles stop; TMEM is released on every exit
// path.
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
constexpr int kStages = 4;
constexpr int kBN = 256;               // output channels per item
constexpr int kABytes = 128 * 128;     // 128 images x one k-block of codes
constexpr int kBBytes = kBN * 128;     // 256 channels x one k-block of codes
constexpr int kStageBytes = kABytes + kBBytes;
constexpr uint32_t kTmemCols = 512;    // the accumulator (256) and 64 scale-factor columns

struct __align__(16) FcBars {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tmem_full;
  uint64_t done;
  uint32_t tmem_base;
  uint32_t abort_flag;
  uint64_t fin_full;  // the finishing CTA's load of the tile's sums
  uint32_t last;      // this CTA finishes its tile
  float2 sb[kBN];
  float beta[128];
};

__global__ void __launch_bounds__(kThreads, 1)
    tc_fc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmWs, const __grid_constant__ CUtensorMap tmOut, const FcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0u) {
    if (threadIdx.x == 0) atomicOr(a.err, kErrLayout);
    return;
  }
  // stage s: [A codes 16 KB][B codes 32 KB]; the epilogue reuses the first stage
  uint8_t* smem = smem_raw;
  FcBars* B = reinterpret_cast<FcBars*>(smem + kStages * kStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // item -> (split, N tile, M tile)
  int t = blockIdx.x;
  const int split = t % a.k_splits;
  t /= a.k_splits;
  const int ntile = t % a.n_tiles;
  const int mtile = t / a.n_tiles;
  const int kb0 = split * a.kb_per_split;
  const int kb1 = min(kb0 + a.kb_per_split, a.kb_total);
  const int m0 = mtile * 128, c0 = ntile * kBN;

  if (threadIdx.x == 0) {
    BCONV_STAMP(0);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&B->full[s], 1);
      mbar_init(&B->empty[s], 1);
    }
    mbar_init(&B->tmem_full, 1);
    mbar_init(&B->done, 1);
    mbar_init(&B->fin_full, 1);
    B->abort_flag = 0;
    B->last = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tensor_map(&tmA);
    prefetch_tensor_map(&tmB);
    prefetch_tensor_map(&tmOut);
    if (a.k_splits > 1) prefetch_tensor_map(&tmWs);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&B->tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (warp >= 2) {
    for (int j = threadIdx.x - 64; j < kBN; j += kEpiThreads) {
      const int c = c0 + j;
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
    tc_fill_32x32(tmem_base + lanes + sf_col, 0x7F7F7F7Fu);
    tc_fill_32x32(tmem_base + lanes + sf_col + 32u, 0x7F7F7F7Fu);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  wait_prior_grid();  // the codes and A come from the previous kernel
  if (threadIdx.x == 0) BCONV_STAMP(1);

  if (warp == 0) {
    // ---------------- producer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&B->empty[stage], phase ^ 1u, B, a.err)) break;
        uint8_t* st = smem + stage * kStageBytes;
        mbar_expect_tx(&B->full[stage], static_cast<uint32_t>(kABytes + kBBytes));
        tma_load_2d(st, &tmA, &B->full[stage], kb * 128, m0);
        tma_load_2d(st + kABytes, &tmB, &B->full[stage], kb * 128, c0);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      const uint32_t idesc = idesc_for(2, 128, kBN);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&B->full[stage], phase, B, a.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (kb == kb0) BCONV_STAMP(2);
        uint8_t* st = smem + stage * kStageBytes;
        const uint64_t da = smem_desc_sw128(st), db = smem_desc_sw128(st + kABytes);
#pragma unroll
        for (int j = 0; j < 4; ++j)  // four 32-byte (64-code) K steps across the 128-byte rows
          tc_mma_f4(tmem_base, da + 2u * j, db + 2u * j, idesc, (kb > kb0 || j > 0) ? 1u : 0u, tmem_base + sf_col,
                    tmem_base + sf_col + 32u);
        tc_commit(&B->empty[stage]);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      BCONV_STAMP(3);
      if (ok) tc_commit(&B->tmem_full);
      tc_commit(&B->done);
      mbar_wait(&B->done, 0, B, a.err, false, true);
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    // The whole 128 x 256 tile is staged in the (by then idle) stage memory as 8 chunks of
    // 128 rows x 32 fp32 (16 KB each; 16-byte chunk k of row r at k ^ (r % 8)) and moved by TMA:
    // reduce-add into the workspace (split) or store into the output (unsplit).  The finishing
    // item of a split tile loads the tile's sums back by TMA, applies the epilogue in shared
    // memory, stores the output and zeroes the workspace, again by TMA.
    const int et = threadIdx.x - 64;  // 0..127
    const int q = warp & 3;
    const int row = q * 32 + lane;    // TMEM lane = image m0 + row
    // betas of the tile's images, while the MMAs run: beta_n = mean of A over the image
    {
      float b = 1.f;
      if (a.A && m0 + et < a.N) {
        const float* An = a.A + static_cast<int64_t>(m0 + et) * a.hw;
        float s = 0.f;
#pragma unroll 8
        for (int p = 0; p < a.hw; ++p) s += __ldg(An + p);
        b = s / static_cast<float>(a.hw);
      }
      B->beta[et] = b;
    }
    auto epilogue_row = [&](float (&y)[32], int ch, float beta) {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float2 p = B->sb[ch * 32 + j];
        const float r = a.A ? fmaf(y[j] * p.x, beta, p.y) : fmaf(y[j], p.x, p.y);
        y[j] = a.relu ? fmaxf(r, 0.f) : r;
      }
    };
    if (epi_all(mbar_wait(&B->tmem_full, 0, B, a.err, true, true))) {
      tc_fence_after();
      if (et == 0) BCONV_STAMP(4);
      const float beta = B->beta[row];
      for (int ch = 0; ch < kBN / 32; ++ch) {
        uint32_t v[32];
        tc_ld_32x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(ch * 32), v);
        float y[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) y[j] = __uint_as_float(v[j]);
        if (a.k_splits == 1) epilogue_row(y, ch, beta);
        float4* orow = reinterpret_cast<float4*>(smem + ch * 16384 + row * 128);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          orow[k ^ (row & 7)] = make_float4(y[4 * k], y[4 * k + 1], y[4 * k + 2], y[4 * k + 3]);
      }
      fence_proxy_async();
      epi_barrier();
      if (et == 0) {
        for (int ch = 0; ch < kBN / 32; ++ch) {
          if (c0 + ch * 32 >= a.No) break;
          if (a.k_splits > 1)
            tma_reduce_add_2d(&tmWs, smem + ch * 16384, c0 + ch * 32, m0);  // integers below 2^24: exact
          else
            tma_store_2d(&tmOut, smem + ch * 16384, c0 + ch * 32, m0);
        }
        bulk_commit();
        bulk_wait_all();
        BCONV_STAMP(5);
        if (a.k_splits > 1) {
          // this item's partial sums are in the workspace: count it in; the last item finishes the tile
          asm volatile("fence.proxy.async.global;" ::: "memory");
          __threadfence();
          const uint32_t old = atomicAdd(a.count + mtile * a.n_tiles + ntile, 1u);
          B->last = (old == static_cast<uint32_t>(a.k_splits - 1)) ? 1u : 0u;
        }
      }
      epi_barrier();
      if (a.k_splits > 1 && B->last) {
        int nch = 0;
        if (et == 0) {
          __threadfence();
          asm volatile("fence.proxy.async.global;" ::: "memory");
          for (int ch = 0; ch < kBN / 32 && c0 + ch * 32 < a.No; ++ch) ++nch;
          mbar_expect_tx(&B->fin_full, static_cast<uint32_t>(nch * 16384));
          for (int ch = 0; ch < nch; ++ch)
            tma_load_2d(smem + ch * 16384, &tmWs, &B->fin_full, c0 + ch * 32, m0);
        }
        if (epi_all(mbar_wait(&B->fin_full, 0, B, a.err, true, true))) {
          for (int ch = 0; ch < kBN / 32; ++ch) {
            float4* orow = reinterpret_cast<float4*>(smem + ch * 16384 + row * 128);
            float y[32];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const float4 t4 = orow[k ^ (row & 7)];
              y[4 * k] = t4.x;
              y[4 * k + 1] = t4.y;
              y[4 * k + 2] = t4.z;
              y[4 * k + 3] = t4.w;
            }
            epilogue_row(y, ch, beta);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              orow[k ^ (row & 7)] = make_float4(y[4 * k], y[4 * k + 1], y[4 * k + 2], y[4 * k + 3]);
          }
          fence_proxy_async();
          epi_barrier();
          if (et == 0) {
            for (int ch = 0; ch < kBN / 32 && c0 + ch * 32 < a.No; ++ch)
              tma_store_2d(&tmOut, smem + ch * 16384, c0 + ch * 32, m0);
            bulk_commit();
            bulk_wait_read_0();
          }
          epi_barrier();
          // zero the workspace tile for the next forward: a zero chunk stored over every chunk
          float4* z = reinterpret_cast<float4*>(smem);
          for (int i = et; i < 16384 / 16; i += kEpiThreads) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
          fence_proxy_async();
          epi_barrier();
          if (et == 0) {
            for (int ch = 0; ch < kBN / 32 && c0 + ch * 32 < a.No; ++ch)
              tma_store_2d(&tmWs, smem, c0 + ch * 32, m0);
            bulk_commit();
            bulk_wait_all();
            a.count[mtile * a.n_tiles + ntile] = 0u;
            BCONV_STAMP(6);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  allow_next_grid();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols));
  }
}

}  // namespace

int tc_fc_smem_bytes() { return kStages * kStageBytes + static_cast<int>(sizeof(FcBars)); }

void tc_fc_plan(FcArgs& a, int sm_count) {
  a.m_tiles = (a.N + 127) / 128;
  a.n_tiles = (a.No + kBN - 1) / kBN;
  const int tiles = a.m_tiles * a.n_tiles;
  // the most splits that keep every item on its own SM, each with at least 4 k-blocks
  int ks = std::max(1, sm_count / std::max(tiles, 1));
  ks = std::min(ks, std::max(1, a.kb_total / 4));
  a.kb_per_split = (a.kb_total + ks - 1) / ks;
  a.k_splits = (a.kb_total + a.kb_per_split - 1) / a.kb_per_split;
}

cudaError_t launch_tc_fc(const CUtensorMap* tmA, const CUtensorMap* tmB, const CUtensorMap* tmWs,
                         const CUtensorMap* tmOut, const FcArgs& a, cudaStream_t s) {
  const int items = a.m_tiles * a.n_tiles * a.k_splits;
  if (items == 0) return cudaSuccess;
  if (!a.out || (reinterpret_cast<uintptr_t>(a.out) & 15u) != 0 || (a.k_splits > 1 && (!a.ws || !a.count)))
    return cudaErrorInvalidValue;
  const int smem = tc_fc_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(tc_fc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_overlapped(tc_fc_kernel, dim3(items), dim3(kThreads), smem, s, *tmA, *tmB, *tmWs, *tmOut, a);
}

}  // namespace bconv

BCONV_TIMELINE_READER(bconv_timeline_fc)
