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
// The k_splits items of a tile form one cluster.  After its MMAs each CTA writes its exact
// partial sums (a 128 x 256 fp32 tile, 16-byte pieces XOR-swizzled within each row) into its
// own shared memory; after a cluster barrier each CTA finishes 128 / k_splits rows: it reads the
// rows of every CTA's partial tile through distributed shared memory, adds them in rank order
// (integers below 2^24: exact in fp32 in any order), applies beta (formed by the epilogue warps
// while the MMAs run), scale, bias and the neuron, and writes each output row with coalesced
// stores.  A second cluster barrier keeps every CTA's shared memory alive until all have read it.
// No workspace and no second launch.
//
// Roles (6 warps): warp 0 TMA producer (4-stage ring); warp 1 TMEM allocation and, from one
// thread, the MMAs; warps 2-5 the epilogue.  Every mbarrier wait gives up after one second of
// %globaltimer, sets the error word and makes all roles stop; TMEM is released on every exit
// path; the cluster barriers are reached on every path.
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
  float2 sb[kBN];
  float beta[128];
};

// Offset, within a CTA's partial tile (128 rows x 1 KB), of float4 `k` (0..63) of row `r`: the
// low three bits of the float4 index are XORed with the row's, so that 32 consecutive rows
// writing the same float4 index hit different banks.
__device__ __forceinline__ uint32_t part_off(int r, int k) {
  return static_cast<uint32_t>(r * 1024 + (((k & ~7) | ((k & 7) ^ (r & 7))) * 16));
}

__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}

// Rows [split * 128 / KS, (split + 1) * 128 / KS) of the tile from the KS partial tiles of the
// cluster: warp q of the epilogue takes every fourth row, lane l channels 8 l .. 8 l + 7.  All
// KS x 2 distributed-shared-memory loads of a row (two rows when KS <= 4) are issued before any
// is used, so that a row costs one remote latency rather than KS of them.
template <int KS>
__device__ __forceinline__ void finish_rows(const FcArgs& a, const FcBars* B, const uint8_t* smem, int split, int m0,
                                            int c0, int q, int lane) {
  constexpr int kRowsPer = 128 / KS;
  constexpr int kUnroll = KS <= 4 ? 2 : 1;  // rows in flight per warp
  uint32_t base[KS];
#pragma unroll
  for (int p = 0; p < KS; ++p) base[p] = mapa(smem, static_cast<uint32_t>(p));
  for (int r0 = split * kRowsPer + q; r0 < (split + 1) * kRowsPer; r0 += 4 * kUnroll) {
    float4 u[kUnroll][KS][2];
#pragma unroll
    for (int h = 0; h < kUnroll; ++h)
#pragma unroll
      for (int p = 0; p < KS; ++p) {
        const int r = r0 + 4 * h;
        u[h][p][0] = ld_cluster_f4(base[p] + part_off(r, 2 * lane));
        u[h][p][1] = ld_cluster_f4(base[p] + part_off(r, 2 * lane + 1));
      }
#pragma unroll
    for (int h = 0; h < kUnroll; ++h) {
      const int r = r0 + 4 * h;
      const int nn = m0 + r;
      if (nn >= a.N) continue;
      float y[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int p = 0; p < KS; ++p) {  // rank order
        y[0] += u[h][p][0].x; y[1] += u[h][p][0].y; y[2] += u[h][p][0].z; y[3] += u[h][p][0].w;
        y[4] += u[h][p][1].x; y[5] += u[h][p][1].y; y[6] += u[h][p][1].z; y[7] += u[h][p][1].w;
      }
      const float bb = B->beta[r];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float2 p = B->sb[8 * lane + j];
        const float v = a.A ? fmaf(y[j] * p.x, bb, p.y) : fmaf(y[j], p.x, p.y);
        y[j] = a.relu ? fmaxf(v, 0.f) : v;
      }
      const int c = c0 + 8 * lane;
      float* o = a.out + static_cast<int64_t>(nn) * a.No + c;
      if (c < a.No) *reinterpret_cast<float4*>(o) = make_float4(y[0], y[1], y[2], y[3]);
      if (c + 4 < a.No) *reinterpret_cast<float4*>(o + 4) = make_float4(y[4], y[5], y[6], y[7]);
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    tc_fc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const FcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0u) {
    if (threadIdx.x == 0) atomicOr(a.err, kErrLayout);
    return;
  }
  // stage s: [A codes 16 KB][B codes 32 KB]; the epilogue reuses the first stage
  uint8_t* smem = smem_raw;
  FcBars* B = reinterpret_cast<FcBars*>(smem + kStages * kStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // item -> (split = the CTA's rank in its cluster, N tile, M tile)
  int t = blockIdx.x;
  const int split = static_cast<int>(cluster_rank());
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
    B->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tensor_map(&tmA);
    prefetch_tensor_map(&tmB);
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
    bool ok = epi_all(mbar_wait(&B->tmem_full, 0, B, a.err, true, true));
    if (ok) {
      tc_fence_after();
      if (et == 0) BCONV_STAMP(4);
      // this CTA's partial tile into its (now idle) stage memory; a split past the last k-block
      // (k_splits * kb_per_split may exceed kb_total by up to a share) issued no MMA and adds 0
      const bool no_kb = kb1 <= kb0;
      for (int ch = 0; ch < kBN / 32; ++ch) {
        uint32_t v[32];
        if (no_kb) {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0u;
        } else {
          tc_ld_32x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(ch * 32), v);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k)
          *reinterpret_cast<float4*>(smem + part_off(row, ch * 8 + k)) =
              make_float4(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]), __uint_as_float(v[4 * k + 2]),
                          __uint_as_float(v[4 * k + 3]));
      }
      if (et == 0) BCONV_STAMP(5);
    }
  }

  // every CTA of the cluster reaches both barriers, whatever happened above
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // every partial tile of the cluster is written
  if (warp >= 2 && !*reinterpret_cast<volatile uint32_t*>(&B->abort_flag)) {
    switch (a.k_splits) {
      case 1: finish_rows<1>(a, B, smem, split, m0, c0, warp & 3, lane); break;
      case 2: finish_rows<2>(a, B, smem, split, m0, c0, warp & 3, lane); break;
      case 4: finish_rows<4>(a, B, smem, split, m0, c0, warp & 3, lane); break;
      default: finish_rows<8>(a, B, smem, split, m0, c0, warp & 3, lane); break;
    }
    if (warp == 2 && lane == 0) BCONV_STAMP(6);
  }
  cluster_sync();  // no CTA leaves while another may still read its partial tile
  allow_next_grid();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols));
  }
}

}  // namespace

int tc_fc_smem_bytes() { return kStages * kStageBytes + static_cast<int>(sizeof(FcBars)); }

namespace {
// Clusters of `ks` CTAs of the FC kernel that can be resident at once (0 if unknown).
int fc_max_clusters(int ks) {
  const int smem = tc_fc_smem_bytes();
  if (cudaFuncSetAttribute(tc_fc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ks));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(ks);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, tc_fc_kernel, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}
}  // namespace

void tc_fc_plan(FcArgs& a, int sm_count) {
  a.m_tiles = (a.N + 127) / 128;
  a.n_tiles = (a.No + kBN - 1) / kBN;
  const int tiles = a.m_tiles * a.n_tiles;
  // the most splits (a cluster of at most 8 CTAs per tile) that keep every item on its own SM
  // in one wave of resident clusters, each with at least 4 k-blocks and an even share of the
  // tile's 128 rows
  int ks = std::max(1, sm_count / std::max(tiles, 1));
  ks = std::min({ks, 8, std::max(1, a.kb_total / 4)});
  while (ks > 1 && (128 % ks != 0 || fc_max_clusters(ks) < tiles)) --ks;
  a.kb_per_split = (a.kb_total + ks - 1) / ks;
  a.k_splits = ks;
}

cudaError_t launch_tc_fc(const CUtensorMap* tmA, const CUtensorMap* tmB, const FcArgs& a, cudaStream_t s) {
  const int items = a.m_tiles * a.n_tiles * a.k_splits;
  if (items == 0) return cudaSuccess;
  if (!a.out || (reinterpret_cast<uintptr_t>(a.out) & 15u) != 0 || a.k_splits < 1 || a.k_splits > 8 ||
      128 % a.k_splits != 0)
    return cudaErrorInvalidValue;
  const int smem = tc_fc_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(tc_fc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess && a.k_splits > 1)
    e = cudaFuncSetAttribute(tc_fc_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(items));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;  // the k splits of a tile
  attr[0].val.clusterDim.x = static_cast<unsigned>(a.k_splits);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // may overlap the pack's tail
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, tc_fc_kernel, *tmA, *tmB, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace bconv

BCONV_TIMELINE_READER(bconv_timeline_fc)
