// Instruction-throughput probes: the measured ceilings the contraction kernels are held to.
//
//   kind 0: XOR + POPC + IADD, the inner-loop mix of the POPC contraction; reported as
//           bit operations per second (32 per POPC).
//   kind 1: LOP3 alone; reported as bit operations per second (32 per instruction).
//   kind 2: b1 tensor MMA, mma.sync m16n8k256 .xor.popc; reported as bit
//           multiply-accumulates per second (16*8*256 per instruction).
//   kind 3: tcgen05.mma.cta_group::1.kind::i8, M=128 N=256 K=32, operands in shared memory,
//           accumulator in TMEM; multiply-accumulates per second.
//   kind 4: tcgen05.mma.cta_group::1.kind::f16 (bf16 operands), M=128 N=256 K=16.
//   kinds 5, 6: kinds 3 and 4 on pseudo-random +-1 operands instead of zeros.
//
// Every thread runs independent dependency chains so that issue rate, not latency, is the
// limit.  Results are stored so the work cannot be removed.  The grid fills every SM with
// four 256-thread CTAs.
#include "common.cuh"
#include "tc_device.cuh"

namespace bconv {
namespace {

constexpr int kProbeThreads = 256;
constexpr int kChains = 16;

__global__ void __launch_bounds__(kProbeThreads) popc_probe(int iters, uint32_t* out, long long* cycles) {
  const uint32_t tid = blockIdx.x * blockDim.x + threadIdx.x;
  uint32_t x[kChains], acc[kChains];
#pragma unroll
  for (int j = 0; j < kChains; ++j) {
    x[j] = tid * 2654435761u + j * 40503u;
    acc[j] = 0;
  }
  const long long t0 = clock64();
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int j = 0; j < kChains; ++j) acc[j] += __popc(x[j] ^ static_cast<uint32_t>(it));
  }
  const long long t1 = clock64();
  uint32_t s = 0;
#pragma unroll
  for (int j = 0; j < kChains; ++j) s += acc[j];
  out[tid] = s;
  if ((threadIdx.x & 31) == 0) atomicMax(reinterpret_cast<unsigned long long*>(cycles), static_cast<unsigned long long>(t1 - t0));
}

__global__ void __launch_bounds__(kProbeThreads) lop3_probe(int iters, uint32_t* out, long long* cycles) {
  const uint32_t tid = blockIdx.x * blockDim.x + threadIdx.x;
  uint32_t x[kChains];
#pragma unroll
  for (int j = 0; j < kChains; ++j) x[j] = tid * 2654435761u + j * 40503u;
  const long long t0 = clock64();
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int j = 0; j < kChains; ++j) {
      uint32_t r;
      // (x & it) ^ ~x, one LOP3 with a loop-varying operand
      asm volatile("lop3.b32 %0, %1, %2, %3, 0x4B;\n" : "=r"(r) : "r"(x[j]), "r"(static_cast<uint32_t>(it)), "r"(x[j]));
      x[j] = r;
    }
  }
  const long long t1 = clock64();
  uint32_t s = 0;
#pragma unroll
  for (int j = 0; j < kChains; ++j) s ^= x[j];
  out[tid] = s;
  if ((threadIdx.x & 31) == 0) atomicMax(reinterpret_cast<unsigned long long*>(cycles), static_cast<unsigned long long>(t1 - t0));
}

constexpr int kMmaChains = 4;

__global__ void __launch_bounds__(kProbeThreads) b1mma_probe(int iters, uint32_t* out, long long* cycles) {
  const uint32_t tid = blockIdx.x * blockDim.x + threadIdx.x;
  uint32_t a[4], b[2];
#pragma unroll
  for (int j = 0; j < 4; ++j) a[j] = tid * 2654435761u + j * 97u;
  b[0] = tid * 40503u + 7u;
  b[1] = tid * 69069u + 3u;
  int32_t d[kMmaChains][4];
#pragma unroll
  for (int c = 0; c < kMmaChains; ++c)
#pragma unroll
    for (int j = 0; j < 4; ++j) d[c][j] = 0;
  const long long t0 = clock64();
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int c = 0; c < kMmaChains; ++c) {
      asm volatile(
          "mma.sync.aligned.m16n8k256.row.col.s32.b1.b1.s32.xor.popc "
          "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
          : "+r"(d[c][0]), "+r"(d[c][1]), "+r"(d[c][2]), "+r"(d[c][3])
          : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
    }
  }
  const long long t1 = clock64();
  int32_t s = 0;
#pragma unroll
  for (int c = 0; c < kMmaChains; ++c)
#pragma unroll
    for (int j = 0; j < 4; ++j) s += d[c][j];
  out[tid] = static_cast<uint32_t>(s);
  if ((threadIdx.x & 31) == 0) atomicMax(reinterpret_cast<unsigned long long*>(cycles), static_cast<unsigned long long>(t1 - t0));
}

// Back-to-back tcgen05 MMAs of one CTA per SM (no data movement): the tensor pipe's own rate,
// on zero operands or (kRandom) on pseudo-random +-1 operands -- int8 0x01 / 0xFF, bf16 +1 / -1
// -- like the contraction's.  One thread issues `iters` groups of 4 MMAs into one TMEM
// accumulator and waits for them through tcgen05.commit (bounded wait).
template <bool kI8, bool kRandom, bool kF4 = false>
__global__ void __launch_bounds__(128, 1) tcgen05_probe(int iters, uint32_t* out, long long* cycles, uint32_t* err) {
  using namespace tcdev;
  extern __shared__ __align__(1024) uint8_t smem[];
  struct Bars {
    uint64_t done;
    uint32_t tmem_base;
    uint32_t abort_flag;
  };
  if ((smem_u32(smem) & 1023u) != 0u) {
    if (threadIdx.x == 0) atomicOr(err, kErrLayout);
    return;
  }
  uint8_t* sa = smem;                  // 128 rows x 128 B
  uint8_t* sb = smem + 128 * 128;      // 256 rows x 128 B
  Bars* B = reinterpret_cast<Bars*>(smem + 128 * 128 + 256 * 128);
  for (int i = threadIdx.x; i < (128 + 256) * 128 / 4; i += blockDim.x) {
    uint32_t w = 0;
    if (kRandom) {
      uint32_t h = (static_cast<uint32_t>(i) + 0x9E3779B9u * (blockIdx.x + 1)) * 0x85EBCA6Bu;
      h ^= h >> 13;
      h *= 0xC2B2AE35u;
      h ^= h >> 16;
      if (kF4) {  // e2m1 +1.0 / -1.0 nibbles
        for (int b = 0; b < 8; ++b) w |= (((h >> b) & 1u) ? 0x2u : 0xAu) << (4 * b);
      } else if (kI8) {
        for (int b = 0; b < 4; ++b) w |= (((h >> b) & 1u) ? 0x01u : 0xFFu) << (8 * b);
      } else {
        w = (((h & 1u) ? 0x3F80u : 0xBF80u)) | (((h & 2u) ? 0x3F80u : 0xBF80u) << 16);
      }
    }
    reinterpret_cast<uint32_t*>(smem)[i] = w;
  }
  if (threadIdx.x == 0) {
    mbar_init(&B->done, 1);
    B->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (threadIdx.x < 32) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&B->tmem_base)),
                 "r"(256));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = B->tmem_base;
  if (kF4) {  // unit block scale factors in the columns after the M128 x N128 accumulator
    tc_fill_32x32(tmem + (static_cast<uint32_t>((threadIdx.x >> 5) * 32) << 16) + 128u, 0x7F7F7F7Fu);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  if (threadIdx.x == 0 && kF4) {
    // kind::mxf4, e2m1 operands, M=128, N=128, K=64 per instruction
    const uint32_t idesc = idesc_for(2, 128, 128);
    const uint64_t da = smem_desc_sw128(sa), db = smem_desc_sw128(sb);
    const long long t0 = clock64();
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        tc_mma_f4(tmem, da + 2u * j, db + 2u * j, idesc, (it > 0 || j > 0) ? 1u : 0u, tmem + 128u, tmem + 144u);
    }
    tc_commit(&B->done);
    mbar_wait(&B->done, 0, B, err, false);
    const long long t1 = clock64();
    atomicMax(reinterpret_cast<unsigned long long*>(cycles), static_cast<unsigned long long>(t1 - t0));
    out[blockIdx.x] = 1u;
  } else if (threadIdx.x == 0) {
    // s32 (i8) or f32 (bf16) accumulator, K-major, M=128, N=256
    const uint32_t idesc = kI8 ? ((2u << 4) | (1u << 7) | (1u << 10) | ((256u >> 3) << 17) | ((128u >> 4) << 24))
                               : ((1u << 4) | (1u << 7) | (1u << 10) | ((256u >> 3) << 17) | ((128u >> 4) << 24));
    const uint64_t da = smem_desc_sw128(sa), db = smem_desc_sw128(sb);
    const long long t0 = clock64();
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t acc = (it > 0 || j > 0) ? 1u : 0u;
        if (kI8)
          asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem),
                       "l"(da + 2u * j), "l"(db + 2u * j), "r"(idesc), "r"(acc) : "memory");
        else
          asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem),
                       "l"(da + 2u * j), "l"(db + 2u * j), "r"(idesc), "r"(acc) : "memory");
      }
    }
    tc_commit(&B->done);
    mbar_wait(&B->done, 0, B, err, false);
    const long long t1 = clock64();
    atomicMax(reinterpret_cast<unsigned long long*>(cycles), static_cast<unsigned long long>(t1 - t0));
    out[blockIdx.x] = 1u;
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256));
  }
}

// The bounded-wait path of the tensor-core kernels, on its own: one thread waits (with the
// kernels' wait routine) on an mbarrier that nothing arrives on, gives up after `limit_ns`,
// records kErrTimeout in the error word and returns -- the device stays usable.
__global__ void wait_check_kernel(uint32_t* err, unsigned long long limit_ns) {
  using namespace tcdev;
  __shared__ struct {
    uint64_t bar;
    uint32_t abort_flag;
  } B;
  if (threadIdx.x != 0) return;
  mbar_init(&B.bar, 1);
  B.abort_flag = 0;
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  mbar_wait(&B.bar, 0, &B, err, true, false, limit_ns);
}

}  // namespace

cudaError_t wait_check(double limit_ms, uint32_t* status) {
  uint32_t* err = nullptr;
  cudaError_t e = cudaMalloc(&err, sizeof(uint32_t));
  if (e == cudaSuccess) e = cudaMemset(err, 0, sizeof(uint32_t));
  if (e == cudaSuccess) {
    wait_check_kernel<<<1, 32>>>(err, static_cast<unsigned long long>(limit_ms * 1e6));
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(status, err, sizeof(uint32_t), cudaMemcpyDeviceToHost);
  if (err) cudaFree(err);
  return e;
}

cudaError_t probe_peak(int kind, double* ops_per_s, double* sm_mhz) {
  if (kind >= 3 && kind <= 7) {
    const int sms = current_sm_count();
    const int iters = 2048;
    const int smem = 120 * 1024;  // more than half an SM's shared memory: one CTA per SM
    uint32_t* out = nullptr;
    long long* cyc = nullptr;
    uint32_t* err = nullptr;
    cudaEvent_t e0 = nullptr, e1 = nullptr;
    cudaError_t e = cudaMalloc(&out, sms * sizeof(uint32_t));
    if (e == cudaSuccess) e = cudaMalloc(&cyc, sizeof(long long));
    if (e == cudaSuccess) e = cudaMalloc(&err, sizeof(uint32_t));
    if (e == cudaSuccess) e = cudaMemset(err, 0, sizeof(uint32_t));
    if (e == cudaSuccess) e = cudaEventCreate(&e0);
    if (e == cudaSuccess) e = cudaEventCreate(&e1);
    auto kern = kind == 3   ? tcgen05_probe<true, false>
                : kind == 4 ? tcgen05_probe<false, false>
                : kind == 5 ? tcgen05_probe<true, true>
                : kind == 6 ? tcgen05_probe<false, true>
                            : tcgen05_probe<false, true, true>;
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    float best = 0.f;
    long long cycles = 0;
    for (int rep = 0; rep < 4 && e == cudaSuccess; ++rep) {
      cudaMemset(cyc, 0, sizeof(long long));
      cudaEventRecord(e0, 0);
      kern<<<sms, 128, smem>>>(iters, out, cyc, err);
      e = cudaGetLastError();
      cudaEventRecord(e1, 0);
      if (e == cudaSuccess) e = cudaEventSynchronize(e1);
      float ms = 0.f;
      if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, e0, e1);
      if (e == cudaSuccess && rep > 0 && (best == 0.f || ms < best)) {
        best = ms;
        cudaMemcpy(&cycles, cyc, sizeof(long long), cudaMemcpyDeviceToHost);
      }
    }
    uint32_t herr = 0;
    if (e == cudaSuccess) e = cudaMemcpy(&herr, err, sizeof(herr), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && herr) e = cudaErrorLaunchTimeout;
    if (e == cudaSuccess && best > 0.f) {
      const double macs = kind == 7 ? static_cast<double>(sms) * iters * 4.0 * 128.0 * 128.0 * 64.0
                                    : static_cast<double>(sms) * iters * 4.0 * 128.0 * 256.0 *
                                          ((kind == 3 || kind == 5) ? 32.0 : 16.0);
      if (ops_per_s) *ops_per_s = macs / (best * 1e-3);
      if (sm_mhz) *sm_mhz = static_cast<double>(cycles) / (best * 1e3);
    }
    if (e0) cudaEventDestroy(e0);
    if (e1) cudaEventDestroy(e1);
    if (out) cudaFree(out);
    if (cyc) cudaFree(cyc);
    if (err) cudaFree(err);
    return e;
  }
  const int sms = current_sm_count();
  const int blocks = sms * 4;
  const int64_t threads = static_cast<int64_t>(blocks) * kProbeThreads;
  const int iters = kind == 2 ? 2048 : 8192;
  uint32_t* out = nullptr;
  long long* cyc = nullptr;
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  cudaError_t err = cudaMalloc(&out, threads * sizeof(uint32_t));
  if (err == cudaSuccess) err = cudaMalloc(&cyc, sizeof(long long));
  if (err == cudaSuccess) err = cudaEventCreate(&e0);
  if (err == cudaSuccess) err = cudaEventCreate(&e1);
  float best_ms = 0.f;
  long long cycles = 0;
  for (int rep = 0; rep < 4 && err == cudaSuccess; ++rep) {
    cudaMemset(cyc, 0, sizeof(long long));
    cudaEventRecord(e0, 0);
    if (kind == 0)
      popc_probe<<<blocks, kProbeThreads>>>(iters, out, cyc);
    else if (kind == 1)
      lop3_probe<<<blocks, kProbeThreads>>>(iters, out, cyc);
    else
      b1mma_probe<<<blocks, kProbeThreads>>>(iters, out, cyc);
    err = cudaGetLastError();
    cudaEventRecord(e1, 0);
    if (err == cudaSuccess) err = cudaEventSynchronize(e1);
    float ms = 0.f;
    if (err == cudaSuccess) err = cudaEventElapsedTime(&ms, e0, e1);
    if (err == cudaSuccess && rep > 0 && (best_ms == 0.f || ms < best_ms)) {
      best_ms = ms;
      cudaMemcpy(&cycles, cyc, sizeof(long long), cudaMemcpyDeviceToHost);
    }
  }
  if (err == cudaSuccess && best_ms > 0.f) {
    double ops;
    if (kind == 0 || kind == 1)
      ops = static_cast<double>(threads) * iters * kChains * 32.0;
    else
      ops = static_cast<double>(threads / 32) * iters * kMmaChains * (16.0 * 8.0 * 256.0);
    if (ops_per_s) *ops_per_s = ops / (best_ms * 1e-3);
    if (sm_mhz) *sm_mhz = static_cast<double>(cycles) / (best_ms * 1e3);
  }
  if (e0) cudaEventDestroy(e0);
  if (e1) cudaEventDestroy(e1);
  if (out) cudaFree(out);
  if (cyc) cudaFree(cyc);
  return err;
}

}  // namespace bconv
