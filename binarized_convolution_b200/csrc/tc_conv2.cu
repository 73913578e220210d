// Binary convolution on SM pairs: tcgen05.mma.cta_group::2 kind::i8 (M = 256 across two SMs).
//
// Same arithmetic as tc_conv.cu (exact int8 +-1 / {0,1} dot products accumulated in int32;
// Apple page "MPSCNNBinaryConvolution", XNOR and AND bullets), with the operand traffic per SM
// cut by a third: a cluster of two CTAs computes a 256 x BN output tile, each CTA holding its
// own 128 output pixels of A and half (BN/2 rows) of the weight tile B.  The pair's MMA is
// issued by one thread of the even CTA (the leader) and reads both CTAs' shared memory; each
// CTA's TMEM receives its own 128 x BN accumulator rows.
//
// Per CTA: warp 0 loads its A box and its half of B with TMA into a 6-stage ring (binaryWeights:
// three A boxes, the parts of x~, per stage against one half weight block; 3 stages); both CTAs'
// copies complete on the leader's `full` barrier, whose expected byte count covers the pair.
// The leader's warp 1 issues the MMAs and releases each stage and each finished accumulator
// with tcgen05.commit multicast to both CTAs.  Warps 2-5 of each CTA run the epilogue of its
// 128 rows (as in tc_conv.cu) and release the accumulator on the leader's barrier.  TMEM is
// allocated and freed with cta_group::2 in both CTAs; the pair synchronises (cluster barrier)
// after set-up and before exit, so no copy or commit ever targets a CTA that has left.
// Every mbarrier wait is bounded by one second of %globaltimer.
#include <cuda.h>

#include "common.cuh"
#include "tc_bits.cuh"
#include "tc_conv.cuh"
#include "tc_device.cuh"

namespace bconv {
namespace {

using namespace tcdev;

constexpr int kStages2 = 6;
constexpr int kABytes2 = 128 * 128;
constexpr int kThreads2 = 192;
constexpr int kEpi2 = 128;
constexpr int kOutBytes2 = 128 * 128;

struct __align__(8) Barriers2 {
  uint64_t full[kStages2];   // used in the leader only
  uint64_t empty[kStages2];  // both CTAs (multicast commit)
  uint64_t tmem_full[2];     // both CTAs (multicast commit)
  uint64_t tmem_empty[2];    // leader only: 4 epilogue warps x 2 CTAs
  uint64_t done;             // both CTAs: every MMA of the pair has completed
  uint32_t tmem_base;
  uint32_t abort_flag;
  float2 sb[256];
};

__device__ __forceinline__ void tma_load_4d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                                 int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, "
      "%5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

__device__ __forceinline__ void tc_mma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tc_mma_i8_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

struct PairCoord {
  int n0, oy0, ox0, ntile;
  int noff, bn;  // channels [ntile*BN + noff, + bn)
  bool dummy;    // this CTA's M tile lies past the end (odd tile count): compute, do not store
  int ptile;     // the pair's M tile (index into the work list)
  int mtile;     // this CTA's M tile
};

// Work item w of the pair -> this CTA's M tile (2*pair + rank) and the N range.
__device__ __forceinline__ PairCoord pair_coord(const TcArgs& a, int w, int rank) {
  PairCoord c;
  int t = w;
  c.noff = 0;
  c.bn = a.BN;
  if (w >= a.full_tiles) {
    const int i = w - a.full_tiles;
    t = a.full_tiles + i / a.pieces;
    c.bn = a.BN / a.pieces;
    c.noff = (i % a.pieces) * c.bn;
  }
  c.ntile = t % a.n_tiles;
  c.ptile = t / a.n_tiles;
  int m = c.ptile * 2 + rank;
  c.dummy = m >= a.m_tiles;
  if (c.dummy) m = a.m_tiles - 1;
  c.mtile = m;
  const int tx = m % a.tiles_x;
  m /= a.tiles_x;
  const int ty = m % a.tiles_y;
  m /= a.tiles_y;
  c.n0 = m * a.Bn;
  c.oy0 = ty * a.R;
  c.ox0 = tx * a.Cw;
  return c;
}

// A pair's work: the items w = pair, pair + npairs, ... with all k-blocks, or (kSk) the
// contiguous share [U*pair/npairs, U*(pair+1)/npairs) of the U = items x kb_total
// reduction units, as segments (item, k0, k1).
template <bool kSk>
struct PairWork {
  int64_t u, uend;
  int w, ks;
  __device__ PairWork(int pair, int npairs, int items, int kb_total, int k_splits = 1) {
    const int64_t U = static_cast<int64_t>(items) * kb_total;
    u = kSk ? U * pair / npairs : 0;
    uend = kSk ? U * (pair + 1) / npairs : 0;
    w = pair;
    ks = k_splits;
  }
  // items are (tile, split) pairs, split fastest; a tile's split s covers k-blocks
  // [s * ceil(kb_total / ks), ...) -- ks = 1 without a split reduction
  __device__ bool next(int npairs, int items, int kb_total, int& item, int& k0, int& k1) {
    if (!kSk) {
      if (w >= items) return false;
      item = w / ks;
      const int per = (kb_total + ks - 1) / ks;
      k0 = (w - item * ks) * per;
      k1 = min(k0 + per, kb_total);
      w += npairs;
      return true;
    }
    if (u >= uend) return false;
    item = static_cast<int>(u / kb_total);
    k0 = static_cast<int>(u - static_cast<int64_t>(item) * kb_total);
    k1 = static_cast<int>(min(static_cast<int64_t>(kb_total), k0 + (uend - u)));
    u += k1 - k0;
    return true;
  }
};

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

template <int kKind, bool kBits, bool kSk, bool kSplit>
__global__ void __launch_bounds__(kThreads2, 1)
    tc_conv2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmBp, const __grid_constant__ CUtensorMap tmOut,
                    const TcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0u) {  // same in both CTAs: both leave before any set-up
    if (threadIdx.x == 0) atomicOr(a.err, kErrLayout);
    return;
  }
  const int half_b = a.BN / 2;  // weight rows this CTA holds
  constexpr int kParts = kKind == 1 ? 3 : 1;  // kind 1: the three parts of x~ per stage
  const int stage_bytes = kParts * kABytes2 + half_b * 128;
  // kind 0 always fits kStages2 (a 32 KB stage at most); kind 1 stages are larger
  const int stages = kKind == 1 ? a.stages : kStages2;
  uint8_t* stage_out = smem + stages * stage_bytes;
  Barriers2* B = reinterpret_cast<Barriers2*>(stage_out + 2 * kOutBytes2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  // work items: pair tiles (x k splits for a split reduction, with its partial sums added into
  // an fp32 workspace by TMA reduce-add; a separate kernel applies the epilogue)
  const int pair_tiles = (a.m_tiles + 1) / 2 * a.n_tiles * a.k_splits;
  const int total = a.full_tiles + (pair_tiles - a.full_tiles) * a.pieces;
  const int kb_total = a.kh * a.kw * a.kb_per_tap;
  const uint32_t tmem_cols = a.tmem_cols;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&B->full[s], 1);
      mbar_init(&B->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&B->tmem_full[b], 1);
      mbar_init(&B->tmem_empty[b], 2 * kEpi2 / 32);
    }
    mbar_init(&B->done, 1);
    B->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&B->tmem_base)),
                 "r"(tmem_cols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any copy or commit crosses over
  tc_fence_after();
  const uint32_t tmem_base = B->tmem_base;
  if (threadIdx.x == 0) {
    prefetch_tensor_map(&tmA);
    prefetch_tensor_map(&tmB);
    prefetch_tensor_map(&tmBp);
    if (!kBits) prefetch_tensor_map(&tmOut);  // a bit-packed output never uses (or encodes) it
  }
  wait_prior_grid();  // the codes, A and the output buffer are the previous kernels' business until here

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      PairWork<kSk> work(pair, npairs, total, kb_total, a.k_splits);
      int w, k0, k1;
      while (ok && work.next(npairs, total, kb_total, w, k0, k1)) {
        const PairCoord pc = pair_coord(a, w, rank);
        const uint32_t tx = static_cast<uint32_t>(2 * (kParts * kABytes2 + (pc.bn / 2) * 128));  // both CTAs' bytes
        for (int kb = k0; kb < k1; ++kb) {
          if (!mbar_wait(&B->empty[stage], phase ^ 1u, B, a.err)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * stage_bytes;
          uint8_t* sb = sa + kParts * kABytes2;
          const uint32_t full_leader = mapa(&B->full[stage], 0);
          if (leader) mbar_expect_tx(&B->full[stage], tx);
          const int tap = kb / a.kb_per_tap, cb = kb - tap * a.kb_per_tap;
          const int ky = tap / a.kw, kx = tap - ky * a.kw;
          for (int part = 0; part < kParts; ++part)  // kind 0: k-blocks are consecutive 128-byte blocks
            tma_load_4d_pair(sa + part * kABytes2, &tmA, full_leader,
                             kKind == 1 ? act_x(cb, part, a.kb_px, a.px_bytes, a.part_bytes) : cb * 128,
                             pc.ox0 * a.sx + kx - a.kw / 2, pc.oy0 * a.sy + ky - a.kh / 2, pc.n0);
          const int brow = pc.ntile * a.BN + pc.noff + static_cast<int>(rank) * (pc.bn / 2);
          if (pc.bn == a.BN)
            tma_load_2d_pair(sb, &tmB, full_leader, kb * 128, brow);
          else
            tma_load_2d_pair(sb, &tmBp, full_leader, kb * 128, brow);
          if (++stage == stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader only) ----------------
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      PairWork<kSk> work(pair, npairs, total, kb_total, a.k_splits);
      int w, k0, k1;
      while (ok && work.next(npairs, total, kb_total, w, k0, k1)) {
        const PairCoord pc = pair_coord(a, w, 0);
        const uint32_t idesc = idesc_for(kKind, 256, pc.bn);
        if (!mbar_wait(&B->tmem_empty[acc], acc_phase ^ 1u, B, a.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * a.BN);
        for (int kb = k0; kb < k1; ++kb) {
          if (!mbar_wait(&B->full[stage], phase, B, a.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint8_t* sa = smem + stage * stage_bytes;
          const uint64_t db = smem_desc_sw128(sa + kParts * kABytes2);
          for (int part = 0; part < kParts; ++part) {  // kind 1: the parts against one weight block
            const uint64_t da = smem_desc_sw128(sa + part * kABytes2);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t accum = (kb > k0 || part > 0 || j > 0) ? 1u : 0u;
              if constexpr (kKind == 1)
                tc_mma_bf16_pair(d_tmem, da + 2u * j, db + 2u * j, idesc, accum);
              else
                tc_mma_i8_pair(d_tmem, da + 2u * j, db + 2u * j, idesc, accum);
            }
          }
          tc_commit_pair(&B->empty[stage]);
          if (++stage == stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair(&B->tmem_full[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      tc_commit_pair(&B->done);  // fires in both CTAs once every MMA above has completed
    }
    if (lane == 0) mbar_wait(&B->done, 0, B, a.err, false, true);
  } else {
    // ---------------- epilogue (both CTAs, warps 2..5) ----------------
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int et = threadIdx.x - 64;
    int acc = 0;
    uint32_t acc_phase = 0;
    int chunk_count = 0;
    int loaded_ntile = -1;
    const int rc = a.R * a.Cw;
    const uint32_t empty_leader0 = mapa(&B->tmem_empty[0], 0), empty_leader1 = mapa(&B->tmem_empty[1], 0);
    // bit-packed output: the next layer's terms and a flag live in the unused staging area
    constexpr bool bits_out = kBits;
    float2* next_t = reinterpret_cast<float2*>(stage_out);
    uint32_t* bits_flag = reinterpret_cast<uint32_t*>(stage_out + kOutBytes2);
    PairWork<kSk> work(pair, npairs, total, kb_total, a.k_splits);
    int w, k0, k1;
    while (work.next(npairs, total, kb_total, w, k0, k1)) {
      const PairCoord pc = pair_coord(a, w, rank);
      if (kSk && k0 > 0) {
        // the later k-blocks of an item that pair - 1 finishes: leave the raw sums for it
        if (!epi_all(mbar_wait(&B->tmem_full[acc], acc_phase, B, a.err, true, true))) break;
        tc_fence_after();
        uint32_t* part = a.sk_part + static_cast<size_t>((pair - 1) * 2 + static_cast<int>(rank)) * a.BN * 128;
        const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * a.BN);
        for (int ch = 0; ch < pc.bn / 32; ++ch) {
          uint32_t v[32];
          tc_ld_32x32(tb + static_cast<uint32_t>(ch * 32), v);
          if (ch == pc.bn / 32 - 1) {
            tc_fence_before();
            if (lane == 0) mbar_arrive_remote(acc == 0 ? empty_leader0 : empty_leader1);
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) part[(ch * 32 + j) * 128 + row] = v[j];  // lanes write 128 B rows
        }
        __threadfence();
        epi_barrier();
        if (et == 0) st_release(a.sk_flag + (pair - 1) * 2 + rank, 1u);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
        continue;
      }
      const bool owner = kSk && k1 < kb_total;  // pair + 1 computes this item's remaining k-blocks
      if (pc.ntile != loaded_ntile) {
        epi_barrier();
        for (int j = et; j < a.BN; j += kEpi2) {
          const int c = pc.ntile * a.BN + j;
          B->sb[j] = c < a.No ? make_float2(__ldg(a.scale + c), __ldg(a.bias + c)) : make_float2(0.f, 0.f);
          if (bits_out)
            next_t[j] = c < a.No ? make_float2(__ldg(a.next_scale + c), __ldg(a.next_bias + c)) : make_float2(0.f, 0.f);
        }
        epi_barrier();
        loaded_ntile = pc.ntile;
      }
      const int n = pc.n0 + row / rc, oy = pc.oy0 + (row / a.Cw) % a.R, ox = pc.ox0 + row % a.Cw;
      const bool valid = !pc.dummy && n < a.N && oy < a.Ho && ox < a.Wo;
      const bool has_beta = a.A != nullptr || a.beta != nullptr;
      float beta = 1.f;
      if (valid && a.A) {
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
        beta = s / static_cast<float>(a.kh * a.kw);
      } else if (valid && a.beta) {
        beta = __ldg(a.beta + (static_cast<int64_t>(n) * a.Ho + oy) * a.Wo + ox);
      }
      const uint32_t* part = nullptr;
      uint32_t pnext[32];  // the other pair's sums for the next chunk, loaded a chunk ahead
      if (owner) {  // wait (bounded) for the partial sums of this item's remaining k-blocks
        bool ready = true;
        if (et == 0) {
          const uint32_t* flag = a.sk_flag + pair * 2 + rank;
          const uint64_t t0 = globaltimer();
          while (ld_acquire(flag) == 0u) {
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
        part = a.sk_part + static_cast<size_t>(pair * 2 + static_cast<int>(rank)) * a.BN * 128;
#pragma unroll
        for (int j = 0; j < 32; ++j) pnext[j] = __ldcg(part + j * 128 + row);  // while the MMAs finish
      }
      if (!epi_all(mbar_wait(&B->tmem_full[acc], acc_phase, B, a.err, true, true))) break;
      tc_fence_after();
      float bits_asum = 0.f;
      Words8 bits_w{};
      const int64_t pix = (static_cast<int64_t>(n) * a.Ho + oy) * a.Wo + ox;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * a.BN);
      for (int ch = 0; ch < pc.bn / 32; ++ch) {
        uint32_t v[32];
        tc_ld_32x32(tbase + static_cast<uint32_t>(ch * 32), v);
        if (ch == pc.bn / 32 - 1) {  // this CTA's rows are read: release them on the leader
          tc_fence_before();
          if (lane == 0) mbar_arrive_remote(acc == 0 ? empty_leader0 : empty_leader1);
        }
        if (part) {  // + the other pair's sums: int32 exactly, fp32 in this fixed order
          uint32_t o[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = pnext[j];
          if (ch + 1 < pc.bn / 32) {
#pragma unroll
            for (int j = 0; j < 32; ++j) pnext[j] = __ldcg(part + ((ch + 1) * 32 + j) * 128 + row);
          }
#pragma unroll
          for (int j = 0; j < 32; ++j)
            v[j] = kKind == 1 ? __float_as_uint(__uint_as_float(v[j]) + __uint_as_float(o[j]))
                              : static_cast<uint32_t>(static_cast<int32_t>(v[j]) + static_cast<int32_t>(o[j]));
        }
        const int buf = chunk_count & 1;
        ++chunk_count;
        uint8_t* so = stage_out + buf * kOutBytes2;
        if (!bits_out) epi_barrier();
        const int c0 = pc.ntile * a.BN + pc.noff + ch * 32;
        const float4* sb4 = reinterpret_cast<const float4*>(&B->sb[pc.noff + ch * 32]);
        float y[32];
        if (kSplit) {  // raw partial sums for the workspace (integers below 2^24 add exactly)
#pragma unroll
          for (int j = 0; j < 32; ++j) y[j] = acc_value(kKind, v[j]);
        } else {
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float4 p = sb4[j / 2];
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
          words_set(bits_w, ch, bits_chunk(y, next_t + pc.noff + ch * 32, min(32, a.No - c0), bits_asum));
          continue;
        }
        float4* orow = reinterpret_cast<float4*>(so + row * 128);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          orow[k ^ (row & 7)] = make_float4(y[4 * k], y[4 * k + 1], y[4 * k + 2], y[4 * k + 3]);
        fence_proxy_async();
        epi_barrier();
        if (et == 0) {
          if (c0 < a.No && !pc.dummy) {
            if (kSplit)
              tma_reduce_add_4d(&tmOut, so, c0, pc.ox0, pc.oy0, pc.n0);
            else
              tma_store_4d(&tmOut, so, c0, pc.ox0, pc.oy0, pc.n0);
          }
          bulk_commit();
          bulk_wait_read_1();
        }
      }
      if (owner) {  // every thread has read the partial sums: the slot is free for the next launch
        epi_barrier();
        if (et == 0) a.sk_flag[pair * 2 + rank] = 0u;
      }
      if (bits_out && !pc.dummy) {
        const int w0 = (pc.ntile * a.BN + pc.noff) / 32;  // first word of this item
        if (valid) words_store(a.out_bits + pix * a.nwo + w0, bits_w, min(pc.bn / 32, a.nwo - w0));
        bits_finish_item(a, pix, valid, bits_asum, pc.ptile, pc.mtile, pc.ntile, pc.ntile * a.pieces + pc.noff / pc.bn,
                         bits_flag, et);
      }
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
  cluster_sync();  // the peer is done with this CTA's barriers and shared memory
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(tmem_cols));
  }
}

}  // namespace

constexpr int kSmemMax2 = 227 * 1024;  // dynamic shared memory one CTA may opt in to

int tc2_stages(int kind, int bn) {
  const int stage = (kind == 1 ? 3 : 1) * kABytes2 + (bn / 2) * 128;
  const int s = (kSmemMax2 - 2 * kOutBytes2 - static_cast<int>(sizeof(Barriers2))) / stage;
  return s < kStages2 ? s : kStages2;
}

int tc2_smem_bytes(int kind, int bn, int stages) {
  return stages * ((kind == 1 ? 3 : 1) * kABytes2 + (bn / 2) * 128) + 2 * kOutBytes2 +
         static_cast<int>(sizeof(Barriers2));
}

int tc2_max_pairs(int kind, int bn) {
  const int stages = tc2_stages(kind, bn);
  if (stages < 2) return 0;
  const int smem = tc2_smem_bytes(kind, bn, stages);
  const void* kerns[] = {
      reinterpret_cast<const void*>(tc_conv2_kernel<0, false, false, false>),
      reinterpret_cast<const void*>(tc_conv2_kernel<1, false, false, false>),
      reinterpret_cast<const void*>(tc_conv2_kernel<0, true, false, false>),
      reinterpret_cast<const void*>(tc_conv2_kernel<1, true, false, false>),
      reinterpret_cast<const void*>(tc_conv2_kernel<0, false, true, false>),
      reinterpret_cast<const void*>(tc_conv2_kernel<1, false, true, false>),
      reinterpret_cast<const void*>(tc_conv2_kernel<0, true, true, false>),
      reinterpret_cast<const void*>(tc_conv2_kernel<1, true, true, false>),
      reinterpret_cast<const void*>(tc_conv2_kernel<0, false, false, true>),
      reinterpret_cast<const void*>(tc_conv2_kernel<1, false, false, true>)};
  bool attr_ok = true;
  for (const void* k : kerns)
    attr_ok = attr_ok && cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess;
  if (!attr_ok) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(kThreads2);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, tc_conv2_kernel<0, false, false, false>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

int tc2_plan(TcArgs& a, int pairs) {
  const int pair_tiles = (a.m_tiles + 1) / 2 * a.n_tiles * a.k_splits;
  const int npairs = pairs;
  a.full_tiles = pair_tiles;
  a.pieces = 1;
  a.sk = 0;
  const int grid_pairs = npairs < pair_tiles ? npairs : pair_tiles;
  const int tail = grid_pairs > 0 ? pair_tiles % grid_pairs : 0;
  // More items than pairs and a last wave so ragged that whole-item waves would keep more
  // than a fifth of the pairs idle on average: give every pair an equal share of the
  // items x k-blocks instead (each share then spans at least one whole item, so an item is
  // cut between two pairs at most).  Measured: 98 items on 74 pairs (waves 66 % full) go from
  // 53.2 to 46.3 us; 196 items (88 % full) run slower split than whole (36.5 -> 49.9 us).
  if (a.k_splits == 1 && pair_tiles > grid_pairs && tail > 0) {
    const int waves = (pair_tiles + grid_pairs - 1) / grid_pairs;
    if (static_cast<double>(pair_tiles) / (static_cast<double>(waves) * grid_pairs) < 0.8) a.sk = 1;
  }
  a.grid_ctas = 2 * grid_pairs;
  return a.grid_ctas;
}

cudaError_t launch_tc_conv2(const CUtensorMap* tmA, const CUtensorMap* tmB, const CUtensorMap* tmBp,
                            const CUtensorMap* tmOut, const TcArgs& a, cudaStream_t s) {
  const int pair_tiles = (a.m_tiles + 1) / 2 * a.n_tiles * a.k_splits;
  if (pair_tiles == 0) return cudaSuccess;
  if (a.stages < 2 || a.stages > kStages2) return cudaErrorInvalidValue;
  const int smem = tc2_smem_bytes(a.kind, a.BN, a.stages);
  const int npairs = a.grid_ctas / 2;
  if (npairs <= 0) return cudaErrorInvalidConfiguration;
  if (a.k_splits > 1 && (a.out_bits || a.sk)) return cudaErrorInvalidValue;
  auto kern =
      a.k_splits > 1 ? (a.kind ? tc_conv2_kernel<1, false, false, true> : tc_conv2_kernel<0, false, false, true>)
      : a.sk ? (a.out_bits ? (a.kind ? tc_conv2_kernel<1, true, true, false> : tc_conv2_kernel<0, true, true, false>)
                           : (a.kind ? tc_conv2_kernel<1, false, true, false> : tc_conv2_kernel<0, false, true, false>))
             : (a.out_bits ? (a.kind ? tc_conv2_kernel<1, true, false, false> : tc_conv2_kernel<0, true, false, false>)
                           : (a.kind ? tc_conv2_kernel<1, false, false, false> : tc_conv2_kernel<0, false, false, false>));
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * npairs));
  cfg.blockDim = dim3(kThreads2);
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
  e = cudaLaunchKernelEx(&cfg, kern, *tmA, *tmB, *tmBp, *tmOut, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace bconv
