// Instruction-throughput probes: the measured ceilings the contraction kernels are held to.
//
//   kind 0: XOR + POPC + IADD, the inner-loop mix of the POPC contraction; reported as
//           bit operations per second (32 per POPC).
//   kind 1: LOP3 alone; reported as bit operations per second (32 per instruction).
//   kind 2: b1 tensor MMA, mma.sync m16n8k256 .xor.popc; reported as bit
//           multiply-accumulates per second (16*8*256 per instruction).
//
// Every thread runs independent dependency chains so that issue rate, not latency, is the
// limit.  Results are stored so the work cannot be removed.  The grid fills every SM with
// four 256-thread CTAs.
#include "common.cuh"

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

}  // namespace

cudaError_t probe_peak(int kind, double* ops_per_s, double* sm_mhz) {
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
