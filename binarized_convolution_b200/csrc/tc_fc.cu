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
// in TMEM.  Per k-block a 128 x 128-byte box of activation codes (TMA, 128-byte swizzled) and a
// 256 x 128-byte block of weight codes (one 32 KB bulk copy of a block the layer laid out
// contiguously, already swizzled: contiguous reads stream from HBM faster than 256 rows of 128
// bytes) feed four M128 N256 K64 MMAs: the activations are read once per 256 channels, the
// weights once per 128 images.  The first stages' weights are requested before the wait for
// the previous kernel: they do not depend on it.
//
// The k_splits items of a tile form one cluster, and each CTA finishes 128 / k_splits rows of
// the tile.  Once every CTA of the cluster has completed its MMAs (a cluster barrier), their
// stage memory is idle and becomes receive buffers (k_splits slots x the owner's rows x 256
// int16): each CTA reads its accumulator and sends every row's exact partial sums, as int16
// (|partial| <= 256 x k-blocks per split <= 32512), to the row's owner -- st.async into the
// peers, completing on the owner's mbarrier, and plain stores for its own rows.  The owner
// adds the slots in rank order (int32, exact), applies beta (formed by the epilogue warps
// while the MMAs run), scale, bias and the neuron and writes each output row with coalesced
// stores.  (The barrier costs nothing on the critical path: an owner needs every split's
// partial sums, so it waits for the slowest CTA of its cluster anyway.)  A second cluster
// barrier keeps every CTA alive until the pushes into it are done.  No workspace, no second
// launch.
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
constexpr int kRowBytes = kBN * 2;     // one row of int16 partial sums
constexpr int kRecvBytes = 128 * kRowBytes;  // k_splits slots x (128 / k_splits) rows, in stage memory
constexpr int kMaxKbPerSplit = 127;    // 256 codes per k-block: |partial| <= 32512 fits int16

struct __align__(16) FcBars {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tmem_full;
  uint64_t done;
  uint64_t recv;  // this CTA's rows of every split's partial sums have arrived
  uint32_t tmem_base;
  uint32_t abort_flag;
  float2 sb[kBN];
  float beta[128];
};

static_assert(kRecvBytes <= kStages * kStageBytes, "the receive buffers live in the stage memory");
static_assert(kStages * kStageBytes + sizeof(FcBars) <= 227 * 1024, "shared memory of one CTA");

// Byte offset, in a receive buffer, of 16-byte piece k (0..31: columns 8 k .. 8 k + 7) of slot
// row sr: the piece index is XORed with the row's low five bits, so that 32 consecutive rows
// writing (or a row's 32 pieces read) hit distinct banks.
__device__ __forceinline__ uint32_t recv_off(int sr, int k) {
  return static_cast<uint32_t>(sr * kRowBytes + ((k ^ (sr & 31)) * 16));
}

// 16 bytes into another CTA's shared memory (cluster address), completing `bytes` on its mbarrier.
__device__ __forceinline__ void st_async_v4(uint32_t addr, uint32_t x, uint32_t y, uint32_t z, uint32_t w,
                                            uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                   addr),
               "r"(x), "r"(y), "r"(z), "r"(w), "r"(bar)
               : "memory");
}

// Two integer-valued fp32 sums (|v| < 2^15) as int16 halves of one word.
__device__ __forceinline__ uint32_t pack_i16x2(uint32_t lo_f, uint32_t hi_f) {
  const int lo = __float2int_rn(__uint_as_float(lo_f)), hi = __float2int_rn(__uint_as_float(hi_f));
  return (static_cast<uint32_t>(lo) & 0xFFFFu) | (static_cast<uint32_t>(hi) << 16);
}

__global__ void __launch_bounds__(kThreads, 1)
    tc_fc_kernel(const __grid_constant__ CUtensorMap tmA, const FcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0u) {
    if (threadIdx.x == 0) atomicOr(a.err, kErrLayout);
    return;
  }
  // stage s: [A codes 16 KB][B codes 32 KB]; once the cluster's MMAs are done the first 64 KB
  // receive the partial sums
  uint8_t* smem = smem_raw;
  uint8_t* recv = smem;
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
    mbar_init(&B->recv, 1);
    B->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    // the one arrival, before any byte can land: the other splits' slots of this CTA's rows
    mbar_expect_tx(&B->recv, static_cast<uint32_t>((a.k_splits - 1) * (128 / a.k_splits) * kRowBytes));
    prefetch_tensor_map(&tmA);
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
  const uint8_t* wblocks = a.b_blocks + static_cast<int64_t>(ntile) * a.kb_total * kBBytes;
  const int pre = min(kStages, max(kb1 - kb0, 0));  // stages whose weights are requested early
  if (threadIdx.x == 0) {  // (the producer thread) the weights do not depend on the previous kernel
    for (int i = 0; i < pre; ++i) {
      uint8_t* st = smem + i * kStageBytes;
      mbar_expect_tx(&B->full[i], static_cast<uint32_t>(kABytes + kBBytes));
      bulk_load(st + kABytes, wblocks + static_cast<int64_t>(kb0 + i) * kBBytes, kBBytes, &B->full[i]);
    }
  }
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
        if (kb - kb0 >= pre) {  // (the first stages' weights are on their way)
          mbar_expect_tx(&B->full[stage], static_cast<uint32_t>(kABytes + kBBytes));
          bulk_load(st + kABytes, wblocks + static_cast<int64_t>(kb) * kBBytes, kBBytes, &B->full[stage]);
        }
        tma_load_2d(st, &tmA, &B->full[stage], kb * 128, m0);
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
    if (__all_sync(0xffffffffu, mbar_wait(&B->tmem_full, 0, B, a.err, true, true))) {
      tc_fence_after();
      if (et == 0) BCONV_STAMP(4);
    }
  }

  // every CTA of the cluster reaches both barriers, whatever happened above
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // every MMA of the cluster has completed: all stage memory is idle
  if (warp >= 2 && !*reinterpret_cast<volatile uint32_t*>(&B->abort_flag)) {
    tc_fence_after();
    const int et = threadIdx.x - 64;
    const int q = warp & 3;
    const int row = q * 32 + lane;  // TMEM lane = image m0 + row
    const int rows_per = 128 / a.k_splits;
    // this row's partial sums to its owner: slot row split * rows_per + (row % rows_per) of CTA
    // row / rows_per; a split past the last k-block (k_splits * kb_per_split may exceed
    // kb_total by up to a share) issued no MMA and sends zeros
    const int owner = row / rows_per;
    const int sr = split * rows_per + (row - owner * rows_per);
    const bool local = owner == split;
    const uint32_t dst = mapa(recv, static_cast<uint32_t>(owner));
    const uint32_t bar = mapa(&B->recv, static_cast<uint32_t>(owner));
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
      for (int i = 0; i < 4; ++i) {  // piece 4 ch + i: columns 32 ch + 8 i .. + 7
        const uint32_t w0 = pack_i16x2(v[8 * i], v[8 * i + 1]), w1 = pack_i16x2(v[8 * i + 2], v[8 * i + 3]);
        const uint32_t w2 = pack_i16x2(v[8 * i + 4], v[8 * i + 5]), w3 = pack_i16x2(v[8 * i + 6], v[8 * i + 7]);
        if (local)
          *reinterpret_cast<uint4*>(recv + recv_off(sr, 4 * ch + i)) = make_uint4(w0, w1, w2, w3);
        else
          st_async_v4(dst + recv_off(sr, 4 * ch + i), w0, w1, w2, w3, bar);
      }
    }
    if (et == 0) BCONV_STAMP(5);
    // this CTA's rows: every split's partial sums, added in rank order
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&B->recv, 0, B, a.err, true, true));
    epi_barrier();  // (the local slots, written by the other epilogue warps)
    if (ok) {
      for (int r = q; r < rows_per; r += 4) {
        const int tr = split * rows_per + r;  // row of the tile
        const int nn = m0 + tr;
        if (nn >= a.N) break;
        int acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (int p = 0; p < a.k_splits; ++p) {
          const int psr = p * rows_per + r;
          const uint4 w = *reinterpret_cast<const uint4*>(recv + recv_off(psr, lane));
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            acc[2 * j] += static_cast<int>(static_cast<int16_t>(ww[j] & 0xFFFFu));
            acc[2 * j + 1] += static_cast<int>(ww[j]) >> 16;
          }
        }
        const float bb = B->beta[tr];
        float y[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float2 p = B->sb[8 * lane + j];
          const float sv = static_cast<float>(acc[j]);  // |S| < 2^24: exact
          const float v = a.A ? fmaf(sv * p.x, bb, p.y) : fmaf(sv, p.x, p.y);
          y[j] = a.relu ? fmaxf(v, 0.f) : v;
        }
        const int c = c0 + 8 * lane;
        float* o = a.out + static_cast<int64_t>(nn) * a.No + c;
        if (c < a.No) *reinterpret_cast<float4*>(o) = make_float4(y[0], y[1], y[2], y[3]);
        if (c + 4 < a.No) *reinterpret_cast<float4*>(o + 4) = make_float4(y[4], y[5], y[6], y[7]);
      }
      if (et == 0) BCONV_STAMP(6);
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA leaves while a peer may still push into its receive buffer
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

bool tc_fc_plan(FcArgs& a, int sm_count) {
  a.m_tiles = (a.N + 127) / 128;
  a.n_tiles = (a.No + kBN - 1) / kBN;
  const int tiles = a.m_tiles * a.n_tiles;
  // the most splits (a cluster of at most 8 CTAs per tile) that keep every item on its own SM
  // in one wave of resident clusters, each with at least 4 k-blocks and an even share of the
  // tile's 128 rows
  int ks = std::max(1, sm_count / std::max(tiles, 1));
  ks = std::min({ks, 8, std::max(1, a.kb_total / 4)});
  while (ks > 1 && (128 % ks != 0 || fc_max_clusters(ks) < tiles)) --ks;
  // each split's partial sums travel as int16: at most kMaxKbPerSplit k-blocks per split
  while ((a.kb_total + ks - 1) / ks > kMaxKbPerSplit && ks < 8) ks *= 2;
  if ((a.kb_total + ks - 1) / ks > kMaxKbPerSplit || fc_max_clusters(ks) < 1) return false;
  a.kb_per_split = (a.kb_total + ks - 1) / ks;
  a.k_splits = ks;
  return true;
}

cudaError_t launch_tc_fc(const CUtensorMap* tmA, const FcArgs& a, cudaStream_t s) {
  const int items = a.m_tiles * a.n_tiles * a.k_splits;
  if (items == 0) return cudaSuccess;
  if (!a.out || (reinterpret_cast<uintptr_t>(a.out) & 15u) != 0 || !a.b_blocks ||
      (reinterpret_cast<uintptr_t>(a.b_blocks) & 15u) != 0 || a.k_splits < 1 || a.k_splits > 8 ||
      128 % a.k_splits != 0 || a.kb_per_split > kMaxKbPerSplit)
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
  e = cudaLaunchKernelEx(&cfg, tc_fc_kernel, *tmA, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace bconv

BCONV_TIMELINE_READER(bconv_timeline_fc)
