// Inline-PTX wrappers shared by the tensor-core kernels (mbarriers, TMA, tcgen05); internal.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "common.cuh"

namespace bconv {
namespace tcdev {

constexpr uint64_t kTimeoutNs = 1000000000ull;  // one second per wait

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait that may suspend the thread (up to `hint_ns`) until the phase completes, so that a
// waiting warp takes no issue slots from the warps that share its scheduler.
__device__ __forceinline__ bool mbar_try_suspend(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete; false after the time limit or, when
// `follow_abort`, as soon as another role has given up (the caller then stops).  `idle`
// waits (the epilogue's wait for an accumulator, the final drain) suspend between checks.
// The polling loop is out of line: inlined into an MMA-issuing loop, even untaken, it slowed
// the issue enough to starve the tensor pipe; the inlined part is one try_wait.
static __device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, uint32_t* abort_flag,
                                                   uint32_t* err, bool follow_abort, bool idle, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer();
  while (true) {
    if (idle ? mbar_try_suspend(bar, parity, 20000u) : mbar_try(bar, parity)) return true;
    if (follow_abort && *reinterpret_cast<volatile uint32_t*>(abort_flag)) return false;
    if (globaltimer() - t0 > limit_ns) {
      atomicOr(err, kErrTimeout);
      atomicExch(abort_flag, 1u);
      return false;
    }
  }
}

template <class Bars>
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, Bars* B, uint32_t* err,
                                          bool follow_abort = true, bool idle = false,
                                          uint64_t limit_ns = kTimeoutNs) {
  if (mbar_try(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, &B->abort_flag, err, follow_abort, idle, limit_ns);
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2,
                                            int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// One contiguous global -> shared copy (addresses 16-byte aligned, bytes a multiple of 16)
// that completes `bytes` of the transaction count of `bar`, like a tensor-map load.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, const void* src, int c0, int c1, int c2, int c3) {
  asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}

__device__ __forceinline__ void tma_reduce_add_4d(const CUtensorMap* map, const void* src, int c0, int c1, int c2,
                                                  int c3) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.4d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1)
               : "memory");
}

__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, const void* src, int c0, int c1) {
  asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1)
               : "memory");
}

// Bring a tensor map (a kernel parameter) into the TMA unit's descriptor cache ahead of use.
__device__ __forceinline__ void prefetch_tensor_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void epi_barrier() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Named barrier 1 over the 128 epilogue threads that also ANDs a predicate across them, so
// that they take every break decision together.
__device__ __forceinline__ bool epi_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, 1, 128, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, M = 128, N and K=32 from the descriptors.
__device__ __forceinline__ void tc_mma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A * B^T with bf16 operands and an fp32 accumulator (kind::f16, K = 16).
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor for M = m, N = n, K-major operands: kind 0 = signed int8 with an s32
// accumulator, kind 1 = bf16 with an f32 accumulator.
__host__ __device__ constexpr uint32_t idesc_for(int kind, int m, int n) {
  // kind 2, kind::mxf4 with block scales: A and B e2m1 (format 1 at bits 7 and 10), K-major,
  // scale factors ue8m0 (bit 23), scale-factor ids 0 (bits 4-5, 29-30), K = 64 (bit 31 = 0);
  // no accumulator-format field (always fp32).
  return (kind == 2   ? ((1u << 7) | (1u << 10) | (1u << 23))
          : kind == 0 ? ((2u << 4) | (1u << 7) | (1u << 10))
                      : ((1u << 4) | (1u << 7) | (1u << 10))) |
         (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(m >> 4) << 24);
}

// D[tmem] (+)= A * B^T with e2m1 operands, every 32 elements scaled by the ue8m0 factors at
// TMEM addresses sfa / sfb (kind::mxf4, K = 64, fp32 accumulator).  With codes +-1 / 0 and
// unit scales every product is exact and so is the fp32 sum of up to 2^24 of them.
__device__ __forceinline__ void tc_mma_f4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate, uint32_t sfa, uint32_t sfb) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// 32 consecutive 32-bit TMEM columns of this warp's 32 lanes set to `value`.
__device__ __forceinline__ void tc_fill_32x32(uint32_t taddr, uint32_t value) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, "
      "%1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1};" ::"r"(taddr),
      "r"(value)
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Byte offset, within a pixel row of the activation map, of part `part` of k-block `cb` of a
// tap (kind 0 has one part).
__device__ __forceinline__ int act_x(int cb, int part, int kb_px, int px_bytes, int part_bytes) {
  if (cb < kb_px) return part * part_bytes + cb * 128;  // a convolution tap: one pixel
  return (cb / kb_px) * px_bytes + part * part_bytes + (cb % kb_px) * 128;
}

// Accumulator word -> fp32 value of the window sum (kind 0: int32; kinds 1 and 2: fp32).
__device__ __forceinline__ float acc_value(int kind, uint32_t v) {
  return kind ? __uint_as_float(v) : static_cast<float>(static_cast<int32_t>(v));
}

// 32 consecutive 32-bit columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tc_ld_32x32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
        "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// The same load without the wait: the caller issues several and then one tcgen05.wait::ld.
__device__ __forceinline__ void tc_ld_32x32_nowait(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
        "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}

// Shared-memory matrix descriptor: K-major operand, rows of 128 bytes with the 128-byte
// swizzle, 8-row groups 1024 bytes apart (tile base 1024-byte aligned).
__device__ __forceinline__ uint64_t smem_desc_sw128(const void* p) {
  const uint32_t a = smem_u32(p);
  uint64_t d = static_cast<uint64_t>((a & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(1) << 16;          // leading byte offset (unused for this layout)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;  // stride byte offset: 8 rows x 128 bytes
  d |= static_cast<uint64_t>(1) << 46;          // descriptor version
  d |= static_cast<uint64_t>(2) << 61;          // 128-byte swizzle
  return d;
}



// ---- SM pairs (clusters of two CTAs, tcgen05 cta_group::2) ----

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// shared::cluster address of a local shared variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}

// (Release semantics at CTA scope, the default: what the arrival hands over -- TMEM columns
// read with tcgen05.ld and waited for -- is ordered by the tcgen05 fences, not by this fence; a
// cluster-scope release waited for this thread's earlier global stores, about a microsecond.)
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                                 int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}

// Arrive on the barrier at this offset in both CTAs of the pair when the MMAs issued so far
// by this thread have completed.
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
}

// D[tmem] (+)= A * B^T over the pair (M = 256: each CTA's A rows and half of B's rows), e2m1
// operands with the ue8m0 block scales at TMEM addresses sfa / sfb (kind::mxf4, K = 64).
__device__ __forceinline__ void tc_mma_f4_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate, uint32_t sfa, uint32_t sfb) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// Named barrier 1 over `n` threads (a multiple of 32), and the same with an AND of a predicate.
__device__ __forceinline__ void named_barrier(uint32_t n) { asm volatile("bar.sync 1, %0;" ::"r"(n) : "memory"); }
__device__ __forceinline__ bool named_all(bool v, uint32_t n) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, 1, %2, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(n)
      : "memory");
  return r != 0;
}

// XNOR-Net beta of the rows-staged kernels' output slots, for `count` tiles of 128 consecutive
// slots (tile t starts at slot (first + t * step) * 128): beta = (sum of A over the kh x kw
// window) / (kh * kw), A being the channel means in the zero-bordered [N][Hp][Wp] grid
// (`total` slots), so the window of slot s is s + ty * wp + tx.  The `nthreads` threads of
// named barrier 1 (index et) first stage the tiles' strips of A -- len = 128 + (kh - 1) * wp +
// kw - 1 floats each, count * len <= the floats `strip` holds -- with eight independent loads
// in flight per thread; then each thread forms the betas of its row (`writer` picks one thread
// per row) into betas[t * 128 + row].  Barriers before (the strip's other users are done with
// it), between, and after (the strip is free again and every beta is visible).
__device__ __forceinline__ void tile_betas(const float* __restrict__ A, int total, int first, int step, int count,
                                           int len, int kh, int kw, int wp, float* strip, float* betas, int row,
                                           bool writer, int et, int nthreads) {
  named_barrier(static_cast<uint32_t>(nthreads));
  const int n = count * len;
  for (int base = 0; base < n; base += 8 * nthreads) {
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int f = base + j * nthreads + et;
      v[j] = 0.f;
      if (f < n) {
        const int t = f / len;
        const int s = (first + t * step) * 128 + (f - t * len);
        if (s < total) v[j] = __ldg(A + s);
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int f = base + j * nthreads + et;
      if (f < n) strip[f] = v[j];
    }
  }
  named_barrier(static_cast<uint32_t>(nthreads));
  if (writer) {
    for (int t = 0; t < count; ++t) {
      const float* w = strip + t * len + row;
      float sum = 0.f;
      for (int ty = 0; ty < kh; ++ty)
        for (int tx = 0; tx < kw; ++tx) sum += w[ty * wp + tx];
      betas[t * 128 + row] = sum / static_cast<float>(kh * kw);
    }
  }
  named_barrier(static_cast<uint32_t>(nthreads));
}

}  // namespace tcdev
}  // namespace bconv
