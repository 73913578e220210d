// C ABI of the binary convolution library: handles, validation, weight preparation and
// the launch sequence of each forward.  The declarations and their contracts are in
// include/bconv.h.
//
// A forward is, in stream order:
//   XNOR / AND:       pack (x~, sign, bits [, A])  [-> beta]  -> POPC contraction + epilogue
//   binaryWeights:    [pack (A only) -> beta ->]  FP32 contraction + epilogue (x~ fused)
// Every buffer a forward touches besides the caller's input and output is allocated at
// create time.
#include <stdlib.h>
#include <string.h>

#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <memory>
#include <mutex>
#include <new>
#include <vector>

#include "bconv.h"
#include "common.cuh"
#include "tc_conv.cuh"

namespace bconv {

int current_sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (dev >= 0 && dev < 64) cache[dev] = sms;
  return sms;
}

namespace {

struct DeviceGuard {
  int prev = -1;
  bool ok = true;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) {
      ok = false;
      return;
    }
    if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

// Device allocations owned by a handle, freed together.
struct DevMem {
  std::vector<void*> ptrs;
  template <typename T>
  cudaError_t alloc(T** p, size_t count) {
    *p = nullptr;
    if (count == 0) count = 1;
    void* q = nullptr;
    cudaError_t e = cudaMalloc(&q, count * sizeof(T));
    if (e != cudaSuccess) return e;
    ptrs.push_back(q);
    *p = static_cast<T*>(q);
    return cudaSuccess;
  }
  void release() {
    for (void* p : ptrs) cudaFree(p);
    ptrs.clear();
  }
};

struct Profile {
  std::vector<cudaEvent_t> start, stop;
  int used = 0;
  bool active = false;
  int every = 1;  // time every `every`-th forward of the window
  int seen = 0;
  // Whether this forward's contraction is timed (advances the sampling counter).
  bool take() {
    if (!active || used >= static_cast<int>(start.size())) return false;
    return (seen++ % every) == 0;
  }
  void clear() {
    for (auto e : start) cudaEventDestroy(e);
    for (auto e : stop) cudaEventDestroy(e);
    start.clear();
    stop.clear();
    used = 0;
    active = false;
  }
};

bconv_status_t from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return BCONV_OK;
  if (e == cudaErrorMemoryAllocation) return BCONV_ERR_OOM;
  if (e == cudaErrorNoDevice || e == cudaErrorInsufficientDriver) return BCONV_ERR_NO_DEVICE;
  return BCONV_ERR_CUDA;
}

// Everything both handle kinds share: parameters on the device, workspace, settings.
struct Layer {
  int device = 0;
  int type = kXnor;
  uint32_t flags = 0;
  int relu = 0;
  int algo = BCONV_ALGO_AUTO;
  // geometry of the contraction
  int N = 0, H = 0, W = 0, Ni = 0, No = 0, kh = 1, kw = 1, sy = 1, sx = 1, Ho = 1, Wo = 1;
  bool fc = false;
  int nw = 0, nw_pad = 0, no_pad = 0;
  // binaryWeights contraction view: per-pixel channels (conv) or the whole flattened image
  // as the channels of one pixel (FC), padded to whole pipeline steps
  int bw_ni = 0, bw_ni_pad = 0;
  float *bw_in_scale = nullptr, *bw_in_bias = nullptr;
  // device parameters
  float *scale = nullptr, *bias = nullptr, *in_scale = nullptr, *in_bias = nullptr;
  uint32_t* wt = nullptr;  // POPC weights
  int32_t* wpop = nullptr;
  float* wf = nullptr;     // binaryWeights weights
  // workspace
  uint32_t* bits = nullptr;
  float *A = nullptr, *beta = nullptr;
  uint32_t* err = nullptr;
  // tensor-core path: int8 codes [N][H][W][cip], int8 weights [no_tc][taps*cip], tensor maps
  bool tc_ok = false;
  bool tc_pair = false;  // contraction on SM pairs (cta_group::2), else one SM per tile
  // Set on the image chunks of a host-buffer forward after the first: that first chunk (same
  // shapes, same plan) owns the device weights and the others read them.
  const Layer* weights_from = nullptr;
  int cip = 0;
  int8_t* codes = nullptr;
  int8_t* wq = nullptr;
  float* ws = nullptr;  // FC split-K partial sums [N][No]
  TcArgs tc{};
  // Rows-staged contraction (tc_halo_kernel): codes in a zero-bordered grid, its plan
  bool halo = false;
  bool halo2 = false;     // the rows-staged contraction on SM pairs (tc_halo2_kernel)
  bool halo_off = false;  // set when a bit-packed output needs the per-tap kernel instead
  HaloArgs hx{};
  PadMap pad{};
  float* A_pad = nullptr;  // A in the zero-bordered grid (rows-staged layers with beta)
  bool f32_off = false;  // binaryWeights: a bit-packed output asks for the parts path (not tc.f32)
  // tc.f32: tensor maps over the last few input buffers, reused by pointer
  CUtensorMap tmX[4];
  const float* tmX_ptr[4] = {nullptr, nullptr, nullptr, nullptr};
  int tmX_next = 0;
  // Fully-connected contraction with 256-channel items (tc_fc_kernel): its plan
  bool fcb = false;
  FcArgs fx{};
  CUtensorMap tmA{}, tmB{}, tmBp{}, tmWs{}, tmOut{};
  const float* tm_out_ptr = nullptr;
  // chained layers: the next layer's input terms (bit-packed output) and what emitting the
  // bits needs -- the slice partials of A on the tensor-core path, an fp32 output buffer
  // for the kernel families that binarize in a separate pass
  bool has_next = false;
  float *next_scale = nullptr, *next_bias = nullptr;
  float* a_part = nullptr;
  uint32_t* a_count = nullptr;
  float* y_scratch = nullptr;
  // host-buffer forward staging (allocated on first use)
  float *stage_in = nullptr, *stage_out = nullptr;
  // The host-buffer forward runs the batch as image chunks, so that one chunk's copy in, the
  // previous chunk's compute and the one before's copy out overlap: the creation parameters
  // (kept on the host), one layer per chunk (made on first use), two copy streams and events.
  std::vector<uint32_t> h_packed;
  std::vector<float> h_scale, h_bias, h_in_scale, h_in_bias;
  float h_scale_value = 1.f;
  std::vector<std::unique_ptr<struct Layer>> chunks;
  cudaStream_t copy_in = nullptr, copy_out = nullptr;
  std::vector<cudaEvent_t> chunk_events;
  DevMem mem;
  DevMem tc_mem;        // the tensor-core path's own buffers (weights, codes, workspaces)
  int codes_override = -1;  // BCONV_CODES_* for this layer's tensor-core plan (-1: the global setting)
  Profile prof;

  int64_t in_elems() const { return static_cast<int64_t>(N) * H * W * Ni; }
  int64_t out_elems() const { return static_cast<int64_t>(N) * Ho * Wo * No; }
  bool use_beta() const { return (flags & BCONV_FLAG_USE_BETA_SCALING) != 0; }
};

struct HandleBase {
  uint32_t magic;
  Layer L;
};
constexpr uint32_t kConvMagic = 0xBC0A7001u;
constexpr uint32_t kFcMagic = 0xBC0A7002u;

}  // namespace
}  // namespace bconv

struct bconv_handle_s : bconv::HandleBase {};
struct bfc_handle_s : bconv::HandleBase {};

namespace bconv {
namespace {

bool valid_type(int t) { return t == kBinaryWeights || t == kXnor || t == kAnd; }

}  // namespace

bconv_status_t check_conv_shape(const bconv_desc_t* d) {
  if (d->neuron != BCONV_NEURON_NONE && d->neuron != BCONV_NEURON_RELU) return BCONV_ERR_INVALID_ARG;
  if (d->batch < 0 || d->in_h <= 0 || d->in_w <= 0 || d->in_channels <= 0 || d->out_channels <= 0 ||
      d->kernel_h <= 0 || d->kernel_w <= 0 || d->stride_y <= 0 || d->stride_x <= 0 || d->groups <= 0)
    return BCONV_ERR_INVALID_ARG;
  if (d->groups != 1) return BCONV_ERR_UNSUPPORTED;
  // a window wider than twice the image plus one has taps that no output can reach; the bounds
  // are tested one by one (in 64 bits) before any product is formed
  if (static_cast<int64_t>(d->kernel_h) > 2 * static_cast<int64_t>(d->in_h) + 1 ||
      static_cast<int64_t>(d->kernel_w) > 2 * static_cast<int64_t>(d->in_w) + 1 || d->kernel_h > 4096 ||
      d->kernel_w > 4096)
    return BCONV_ERR_UNSUPPORTED;
  const int64_t taps = static_cast<int64_t>(d->kernel_h) * d->kernel_w;
  if (taps > 4096 || d->in_channels > (1 << 20) || d->out_channels > (1 << 20)) return BCONV_ERR_UNSUPPORTED;
  // the integer window sums (at most taps x in_channels in magnitude) must fit int32
  if (taps * d->in_channels > INT32_MAX) return BCONV_ERR_UNSUPPORTED;
  return BCONV_OK;
}

namespace {

// cuTensorMapEncodeTiled from the driver, found through the runtime (the library does not
// link the driver library, so it loads on machines without one).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 4-D tiled map, dims innermost first, 128-byte swizzle, out-of-range elements read as 0.
bool encode_4d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, const uint64_t dims[4],
               const uint64_t strides_bytes[3], const uint32_t box[4], const uint32_t elem_strides[4] = nullptr,
               CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint32_t estr[4] = {1, 1, 1, 1};
  if (elem_strides)
    for (int i = 0; i < 4; ++i) estr[i] = elem_strides[i];
  return enc(m, dt, 4, const_cast<void*>(base), reinterpret_cast<const cuuint64_t*>(dims),
             reinterpret_cast<const cuuint64_t*>(strides_bytes), reinterpret_cast<const cuuint32_t*>(box), estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1, uint64_t stride1,
               uint32_t b0, uint32_t b1, CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {d0, d1};
  const cuuint64_t strides[1] = {stride1};
  const cuuint32_t box[2] = {b0, b1};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int next_pow2(int v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

// Output map over `out` ([N][Ho][Wo][No] fp32) with the tile's box: 32 channels x Cw x R x Bn.
bool encode_out_map(Layer& L, CUtensorMap* m, const float* out) {
  const uint64_t d[4] = {static_cast<uint64_t>(L.No), static_cast<uint64_t>(L.Wo), static_cast<uint64_t>(L.Ho),
                         static_cast<uint64_t>(L.N)};
  const uint64_t row = static_cast<uint64_t>(L.No) * 4;
  const uint64_t strides[3] = {row, row * L.Wo, row * L.Wo * L.Ho};
  const uint32_t box[4] = {32, static_cast<uint32_t>(L.tc.Cw), static_cast<uint32_t>(L.tc.R),
                           static_cast<uint32_t>(L.tc.Bn)};
  return encode_4d(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, out, d, strides, box);
}

// Map over `in` ([N][H][W][Ni] fp32) for binaryWeights from fp32 input (tc.f32): boxes of 32
// channels (128-byte rows, 128-byte swizzle) x Cw x R x Bn pixels stepping by the strides, as
// the one-SM kernel loads them per tap.  Maps of the last four input buffers are kept;
// nullptr if `in` cannot be mapped (not 16-byte aligned).
const CUtensorMap* input_map(Layer& L, const float* in) {
  for (int i = 0; i < 4; ++i)
    if (L.tmX_ptr[i] == in) return &L.tmX[i];
  if ((reinterpret_cast<uintptr_t>(in) & 15u) != 0) return nullptr;
  const int i = L.tmX_next;
  const uint64_t dims[4] = {static_cast<uint64_t>(L.Ni), static_cast<uint64_t>(L.W), static_cast<uint64_t>(L.H),
                            static_cast<uint64_t>(L.N)};
  const uint64_t row = static_cast<uint64_t>(L.Ni) * sizeof(float);
  const uint64_t strides[3] = {row, row * L.W, row * L.W * L.H};
  const uint32_t box[4] = {32, static_cast<uint32_t>(L.tc.sx * L.tc.Cw), static_cast<uint32_t>(L.tc.sy * L.tc.R),
                           static_cast<uint32_t>(L.tc.Bn)};
  const uint32_t estr[4] = {1, static_cast<uint32_t>(L.tc.sx), static_cast<uint32_t>(L.tc.sy), 1};
  if (!encode_4d(&L.tmX[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, in, dims, strides, box, estr)) return nullptr;
  L.tmX_ptr[i] = in;
  L.tmX_next = (i + 1) % 4;
  return &L.tmX[i];
}

// The tensor-core path: XNOR/AND as int8 codes (kind 0) and binaryWeights as three exact
// bf16 parts of x~ (kind 1), for No % 4 == 0 (16-byte output rows for the TMA store) and
// strided windows whose TMA box (stride x tile extent) stays within 256 elements.
// Sets up its buffers, weights and maps.
// Kernel family and operand codes for layers created from now on (BCONV_CTA_*, BCONV_CODES_*).
std::atomic<int> g_cta_mode{BCONV_CTA_AUTO};
std::atomic<int> g_tc_codes{BCONV_CODES_AUTO};
std::atomic<int> g_staging{BCONV_STAGING_AUTO};

// k-block stages on the busiest SM under each family's plan (the plans' own work lists).
double plan_stages_single(TcArgs t, int sms) {
  const int kb = t.kh * t.kw * t.kb_per_tap;
  const int tiles = t.m_tiles * t.n_tiles;
  const int grid = tc_plan(t, sms);
  if (grid <= 0) return 0.0;
  if (t.pieces > 1) return (static_cast<double>(t.full_tiles / grid) + 1.0 / t.pieces) * kb;
  return static_cast<double>((tiles + grid - 1) / grid) * kb;
}

double plan_stages_pair(TcArgs t, int pairs) {
  const int kb = t.kh * t.kw * t.kb_per_tap;
  const int grid_pairs = tc2_plan(t, pairs) / 2;
  if (grid_pairs <= 0) return 0.0;
  const int64_t items = t.full_tiles;
  if (t.sk) return static_cast<double>((items * kb + grid_pairs - 1) / grid_pairs);
  return static_cast<double>((items + grid_pairs - 1) / grid_pairs) * kb;
}

// The FC on e2m1 codes with 256-channel items (tc_fc_kernel).  Weight row c (output channel,
// rows padded to 256 per tile) holds, per pixel, cip codes as cip / 2 bytes: the layer's bits as
// +1.0 / -1.0 (XNOR) or 1.0 / 0 (AND), channel 2j in the low nibble, zero codes past Ni.
bconv_status_t setup_fc(Layer& L, const uint32_t* packed) {
  FcArgs& f = L.fx;
  f = FcArgs{};
  const int hw = L.H * L.W;
  const int64_t px_bytes = L.cip / 2;
  f.N = L.N;
  f.No = L.No;
  f.hw = hw;
  f.kb_total = hw * (L.cip / 256);
  if (!tc_fc_plan(f, current_sm_count())) return BCONV_OK;  // (checked by the caller)
  const int64_t rows = static_cast<int64_t>(f.n_tiles) * 256;
  const int64_t row_bytes = static_cast<int64_t>(hw) * px_bytes;
  const Layer* src = L.weights_from;
  const bool borrowed = src && src->fcb && src->wq && src->fx.n_tiles == f.n_tiles && src->fx.kb_total == f.kb_total;
  cudaError_t e = cudaSuccess;
  if (borrowed) {
    L.wq = src->wq;
  } else {
    const uint8_t neg = (L.type == kXnor) ? 0xAu : 0x0u;  // e2m1 -1.0, or 0
    std::vector<uint8_t> hb(static_cast<size_t>(rows * row_bytes), 0u);
    for (int c = 0; c < L.No; ++c)
      for (int p = 0; p < hw; ++p) {
        uint8_t* dst = hb.data() + static_cast<size_t>(c) * row_bytes + static_cast<int64_t>(p) * px_bytes;
        for (int f0 = 0; f0 < L.Ni; ++f0) {
          const uint32_t word = packed[(static_cast<int64_t>(c) * hw + p) * L.nw + f0 / kWordBits];
          const uint8_t code = ((word >> (f0 % kWordBits)) & 1u) ? 0x2u : neg;
          dst[f0 / 2] |= static_cast<uint8_t>(code << (4 * (f0 % 2)));
        }
      }
    // as contiguous (N tile, k-block) blocks of 256 rows x 128 bytes, each with the 128-byte
    // swizzle applied (16-byte chunk c of row r at c ^ (r % 8)): one bulk copy per stage
    {
      std::vector<uint8_t> blocks(hb.size());
      for (int nt = 0; nt < f.n_tiles; ++nt)
        for (int kb = 0; kb < f.kb_total; ++kb)
          for (int r = 0; r < 256; ++r) {
            const uint8_t* src_row = hb.data() + static_cast<size_t>(nt * 256 + r) * row_bytes + static_cast<int64_t>(kb) * 128;
            uint8_t* dst = blocks.data() + ((static_cast<size_t>(nt) * f.kb_total + kb) * 256 + r) * 128;
            for (int c = 0; c < 8; ++c) memcpy(dst + 16 * (c ^ (r & 7)), src_row + 16 * c, 16);
          }
      hb.swap(blocks);
    }
    e = L.tc_mem.alloc(&L.wq, hb.size());
    if (e == cudaSuccess) e = cudaMemcpy(L.wq, hb.data(), hb.size(), cudaMemcpyHostToDevice);
  }
  if (e == cudaSuccess) e = L.tc_mem.alloc(&L.codes, static_cast<size_t>(L.N) * row_bytes);
  if (e != cudaSuccess) return from_cuda(e);
  const bool ok = encode_2d(&L.tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, L.codes, static_cast<uint64_t>(row_bytes),
                            static_cast<uint64_t>(L.N), static_cast<uint64_t>(row_bytes), 128, 128);
  if (!ok) return BCONV_OK;  // the POPC path stays available
  f.b_blocks = reinterpret_cast<const uint8_t*>(L.wq);
  f.scale = L.scale;
  f.bias = L.bias;
  f.relu = L.relu;
  f.err = L.err;
  L.tc.kind = 2;
  L.tc.BN = 256;
  L.tc.n_tiles = f.n_tiles;
  L.tc.k_splits = f.k_splits;
  L.tc.N = L.N;
  L.tc.No = L.No;
  L.fcb = true;
  L.tc_ok = true;
  return BCONV_OK;
}

bconv_status_t setup_tc(Layer& L, const uint32_t* packed) {
  if (L.No % 4 != 0 || L.N == 0) return BCONV_OK;
  if (!tensor_map_encoder()) return BCONV_OK;
  const int taps = L.kh * L.kw;
  TcArgs& t = L.tc;
  // Operand codes: XNOR/AND as e2m1 (fp4) values on one SM per tile (kind 2) unless int8 is
  // asked for or the spread is forced onto SM pairs (kind 0); binaryWeights as three bf16 parts
  // (kind 1).
  const int mode = g_cta_mode.load();
  const int codes = L.codes_override >= 0 ? L.codes_override : g_tc_codes.load();
  // An XNOR / AND window sum adds up to (reduction length) terms of magnitude 1.  fp32 adds
  // such integers exactly only below 2^24: beyond that the e2m1 path (fp32 accumulators) and the
  // FC's split reduction (fp32 reduce-add) could round, so such layers keep int32 sums -- int8
  // codes with s32 accumulators for a convolution, the POPC family (int32 split sums) for an FC.
  const int64_t red_len = L.fc ? static_cast<int64_t>(L.H) * L.W * L.Ni : static_cast<int64_t>(taps) * L.Ni;
  const bool fp32_exact = red_len <= (int64_t{1} << 24);
  if (L.type != kBinaryWeights && !fp32_exact && L.fc) return BCONV_OK;
  t.kind = L.type == kBinaryWeights                                                   ? 1
           : (codes == BCONV_CODES_INT8 || mode == BCONV_CTA_PAIR || !fp32_exact) ? 0
                                                                                   : 2;
  if (L.fc && t.kind == 2) {  // the e2m1 FC kernel adds int16 partial sums: at most 127 k-blocks a split
    FcArgs f{};
    f.N = L.N;
    f.No = L.No;
    f.kb_total = L.H * L.W * (round_up(L.Ni, 256) / 256);
    if (!tc_fc_plan(f, current_sm_count())) t.kind = 0;
  }
  // channels per part, padded to whole 128-byte rows; bytes of activation operand per pixel
  // (kind 1: three bf16 parts) and of weights per output channel and tap (kind 1: one bf16
  // copy, which every part is multiplied with; kind 2: two codes per byte)
  L.cip = t.kind == 0 ? round_up(L.Ni, 128) : t.kind == 1 ? round_up(L.Ni, 64) : round_up(L.Ni, 256);
  const int bpp = t.kind == 0 ? L.cip : t.kind == 1 ? 6 * L.cip : L.cip / 2;
  const int bpb = t.kind == 0 ? L.cip : t.kind == 1 ? 2 * L.cip : L.cip / 2;
  t.kb_px = bpb / 128;
  t.px_bytes = bpp;
  t.part_bytes = t.kind == 1 ? 2 * L.cip : 0;
  L.fcb = false;
  if (L.fc && t.kind == 2) return setup_fc(L, packed);
  // The FC runs on SM pairs when its batch fills both CTAs of a pair (256 images per pair
  // tile, so the weight matrix streams from memory once, with half of every weight tile per
  // SM); otherwise a single SM keeps up to 256 images in one tile (two 128-row sub-tiles
  // sharing every weight stage; int8 codes only).
  const bool fc_pair = L.fc && L.N > 128 && mode != BCONV_CTA_SINGLE && t.kind != 2 &&
                       tc2_max_pairs(t.kind, std::min(256, round_up(L.No, 32))) > 0;
  t.mt = (L.fc && L.N > 128 && !fc_pair && t.kind == 0) ? 2 : 1;
  // kind 2 tiles are at most 128 channels wide: TMEM holds two accumulators and the scale factors
  t.BN = std::min(t.mt == 2 || t.kind == 2 ? 128 : 256, round_up(L.No, 32));
  t.n_tiles = (L.No + t.BN - 1) / t.BN;
  t.No = L.No;
  t.N = L.N;
  t.tmem_cols = static_cast<uint32_t>(std::max(32, next_pow2(2 * t.mt * t.BN + (t.kind == 2 ? 32 : 0))));
  t.relu = L.relu;
  t.err = L.err;
  t.scale = L.scale;
  t.bias = L.bias;
  if (L.fc) {
    t.Ho = 1; t.Wo = 1; t.kh = 1; t.kw = 1; t.sy = 1; t.sx = 1;
    t.kb_per_tap = L.H * L.W * bpb / 128;
    t.R = 1; t.Cw = 1; t.Bn = 128;
    t.tiles_x = 1; t.tiles_y = 1;
  } else {
    t.Ho = L.Ho; t.Wo = L.Wo; t.kh = L.kh; t.kw = L.kw; t.sy = L.sy; t.sx = L.sx;
    t.kb_per_tap = bpb / 128;
    // 128 output pixels per tile as Bn images x R rows x Cw columns (powers of two, so that
    // every 32-row quarter is a box too): the shape with the fewest tiles, i.e. the least
    // MMA work on pixels past the image edges (56 x 56 -> 8 x 8 x 2 images: none), then
    // the smallest window footprint; the TMA box (stride x extent) stays within 256.
    int64_t best_tiles = -1, best_halo = 0;
    for (int cw = 1; cw <= 128; cw *= 2)
      for (int r = 1; cw * r <= 128; r *= 2) {
        const int bn = 128 / (cw * r);
        if (t.sx * cw > 256 || t.sy * r > 256) continue;
        const int64_t tiles = static_cast<int64_t>((L.Wo + cw - 1) / cw) * ((L.Ho + r - 1) / r) * ((L.N + bn - 1) / bn);
        const int64_t halo = static_cast<int64_t>(cw * t.sx + L.kw - 1) * (r * t.sy + L.kh - 1) * bn;
        if (best_tiles < 0 || tiles < best_tiles || (tiles == best_tiles && halo < best_halo)) {
          best_tiles = tiles;
          best_halo = halo;
          t.Cw = cw;
          t.R = r;
        }
      }
    if (best_tiles < 0) return BCONV_OK;  // no box fits the TMA limits
    t.Bn = 128 / (t.Cw * t.R);
    t.tiles_x = (L.Wo + t.Cw - 1) / t.Cw;
    t.tiles_y = (L.Ho + t.R - 1) / t.R;
  }
  t.m_tiles = t.tiles_x * t.tiles_y * ((L.N + t.Bn * t.mt - 1) / (t.Bn * t.mt));
  const int kb_total = t.kh * t.kw * t.kb_per_tap;
  t.k_splits = 1;
  if (L.fc) {  // spread the reduction so that the tiles fill the GPU (or its SM pairs)
    const int workers = fc_pair ? tc2_max_pairs(t.kind, t.BN) : current_sm_count();
    const int64_t tiles = static_cast<int64_t>(fc_pair ? (t.m_tiles + 1) / 2 : t.m_tiles) * t.n_tiles;
    int64_t best = -1;
    for (int sp = 1; sp <= 16 && kb_total / sp >= 4; ++sp) {
      const int64_t cost = ceil_div(tiles * sp, workers) * ceil_div(kb_total, sp);
      if (best < 0 || cost < best) {
        best = cost;
        t.k_splits = sp;
      }
    }
  }

  // Kernel family.  The FC follows fc_pair.  A convolution runs on SM pairs only when their
  // plan needs clearly fewer k-block stages on the busiest SM: under 95 % of the one-SM plan's
  // for int8 codes, under 80 % for binaryWeights, whose stages cost the pairs relatively more
  // (each CTA still loads all three 16 KB activation parts per stage, and the balanced split
  // adds its exchange).  Measured on B200: batch 16, 56 x 56, 256 -> 256, 3 x 3 (54 stages per
  // SM either way) 44.2 us per forward on single SMs against 48.3 us on pairs; batch 8,
  // 112 x 112, 128 -> 128, stride 2, binaryWeights (27 stages on single SMs with the tail cut
  // in halves, 24 on pairs with the balanced split) 46.9 us against 53.7 us.
  const double pair_factor = t.kind == 1 ? 0.80 : 0.95;
  // binaryWeights without beta: the contraction reads the fp32 input itself and splits it in
  // shared memory (no 3-part buffer: the parts cost 1.5x the input to write and again to read)
  t.f32 = (t.kind == 1 && !L.fc && !L.use_beta() && !L.f32_off && L.Ni % 4 == 0 && mode != BCONV_CTA_PAIR &&
           g_staging.load() != BCONV_STAGING_PER_TAP && tc_f32_stages(t.BN) > 0)
              ? 1
              : 0;
  t.in_scale = L.in_scale;
  t.in_bias = L.in_bias;
  t.Ni = L.Ni;
  int pairs = 0;
  if (L.fc) {
    pairs = fc_pair ? tc2_max_pairs(t.kind, t.BN) : 0;
  } else if (mode != BCONV_CTA_SINGLE && t.kind != 2 && !t.f32) {
    pairs = tc2_max_pairs(t.kind, t.BN);
    if (pairs > 0 && mode == BCONV_CTA_AUTO &&
        !(plan_stages_pair(t, pairs) < pair_factor * plan_stages_single(t, current_sm_count())))
      pairs = 0;
  }

  t.stages = pairs > 0 ? tc2_stages(t.kind, t.BN) : t.f32 ? tc_f32_stages(t.BN) : tc_stages(t.kind, t.BN, t.mt);
  if (t.stages < 2) return BCONV_OK;  // no room for a pipeline: the SIMT family stays

  // Rows-staged contraction: e2m1 codes, stride 1, image rows that fit a tile (kernel
  // tc_halo_kernel); its codes live in a zero-bordered grid
  L.halo = false;
  L.halo2 = false;
  L.pad = PadMap{};
  const int staging = g_staging.load();
  if (t.kind == 2 && !L.fc && L.sy == 1 && L.sx == 1 && pairs == 0 && !L.halo_off &&
      staging != BCONV_STAGING_PER_TAP) {
    HaloArgs& h = L.hx;
    h = HaloArgs{};
    h.N = L.N; h.H = L.H; h.W = L.W; h.kh = L.kh; h.kw = L.kw;
    h.Hp = L.H + L.kh - 1;
    h.Wp = L.W + L.kw - 1;
    h.kb_per_tap = t.kb_per_tap;
    h.BN = t.BN; h.n_tiles = t.n_tiles; h.No = L.No;
    // more than 128 output channels: SM pairs with 256-channel MMAs (each SM's MMAs then run
    // at the tensor pipe's rate); else one SM per 128-slot tile
    HaloArgs h2 = h;
    if (mode != BCONV_CTA_SINGLE && tc_halo2_plan(h2, 0)) {
      h = h2;
      L.halo = true;
      L.halo2 = true;
    } else if (mode != BCONV_CTA_PAIR && tc_halo_plan(h, current_sm_count())) {
      L.halo = true;
    }
    if (L.halo) {
      L.pad = PadMap{L.H, L.W, h.Hp, h.Wp, L.kh / 2, L.kw / 2};
      t.BN = h.BN;  // the plan may narrow (one SM) or widen (pairs) the tiles
      t.n_tiles = h.n_tiles;
    }
  }
  // Weights [no_tc][taps][bpb bytes]: kind 0 int8 +-1 (XNOR) or 0/1 (AND); kind 1 bf16 +-1.
  // Every padding slot is 0.
  const int no_tc = t.n_tiles * t.BN;
  const int64_t kt = static_cast<int64_t>(taps) * bpb;
  const Layer* src = L.weights_from;
  const bool borrowed = src && src->tc_ok && src->wq && src->tc_pair == (pairs > 0) && src->tc.BN == t.BN &&
                        src->tc.kind == t.kind && src->tc.n_tiles == t.n_tiles && src->cip == L.cip;
  std::vector<int8_t> hq(borrowed ? 0 : static_cast<size_t>(no_tc) * kt, 0);
  const int8_t zero_code = (L.type == kXnor) ? -1 : 0;
  const uint8_t zero_f4 = (L.type == kXnor) ? 0xAu : 0x0u;  // e2m1 -1.0, or 0
  for (int c = 0; c < (borrowed ? 0 : L.No); ++c)
    for (int tp = 0; tp < taps; ++tp)
      for (int f = 0; f < L.Ni; ++f) {
        const uint32_t word = packed[(static_cast<int64_t>(c) * taps + tp) * L.nw + f / kWordBits];
        const bool bit = ((word >> (f % kWordBits)) & 1u) != 0;
        int8_t* row = hq.data() + static_cast<size_t>(c) * kt + static_cast<int64_t>(tp) * bpb;
        if (t.kind == 0) {
          row[f] = bit ? 1 : zero_code;
        } else if (t.kind == 2) {
          row[f / 2] = static_cast<int8_t>(static_cast<uint8_t>(row[f / 2]) | ((bit ? 0x2u : zero_f4) << (4 * (f % 2))));
        } else {
          const uint16_t v = bit ? 0x3F80u : 0xBF80u;  // bf16 +1 / -1
          memcpy(row + 2 * f, &v, 2);
        }
      }
  if (pairs == 0 && !L.halo2 && !borrowed) {
    // the one-SM kernel copies each (N tile, k-block) stage of BN rows x 128 bytes as one
    // block: lay the blocks out contiguously with the 128-byte swizzle already applied
    const int kbt = static_cast<int>(kt / 128);
    std::vector<int8_t> tiles(hq.size());
    for (int nt = 0; nt < t.n_tiles; ++nt)
      for (int kb = 0; kb < kbt; ++kb)
        for (int r = 0; r < t.BN; ++r) {
          const int8_t* src = hq.data() + static_cast<size_t>(nt * t.BN + r) * kt + static_cast<int64_t>(kb) * 128;
          int8_t* dst = tiles.data() + (static_cast<size_t>(nt) * kbt + kb) * t.BN * 128 + static_cast<size_t>(r) * 128;
          for (int c = 0; c < 8; ++c) memcpy(dst + 16 * (c ^ (r & 7)), src + 16 * c, 16);
        }
    hq.swap(tiles);
  }
  const int64_t npix = L.halo ? static_cast<int64_t>(L.N) * L.hx.Hp * L.hx.Wp : static_cast<int64_t>(L.N) * L.H * L.W;
  cudaError_t e = cudaSuccess;
  if (borrowed) {
    L.wq = src->wq;
  } else {
    e = L.tc_mem.alloc(&L.wq, hq.size());
    if (e == cudaSuccess) e = cudaMemcpy(L.wq, hq.data(), hq.size(), cudaMemcpyHostToDevice);
  }
  if (e == cudaSuccess && !t.f32) e = L.tc_mem.alloc(&L.codes, static_cast<size_t>(npix) * bpp);
  // the border of the padded grid is written once, here, and never again
  if (e == cudaSuccess && L.halo) e = cudaMemset(L.codes, 0, static_cast<size_t>(npix) * bpp);
  if (e == cudaSuccess && L.halo && L.use_beta()) e = L.tc_mem.alloc(&L.A_pad, static_cast<size_t>(npix));
  if (e == cudaSuccess && L.halo && L.use_beta()) e = cudaMemset(L.A_pad, 0, sizeof(float) * static_cast<size_t>(npix));
  if (e == cudaSuccess && t.k_splits > 1) e = L.tc_mem.alloc(&L.ws, static_cast<size_t>(L.N) * L.No);
  if (e == cudaSuccess && t.k_splits > 1) e = cudaMemset(L.ws, 0, sizeof(float) * static_cast<size_t>(L.N) * L.No);
  if (e != cudaSuccess) return from_cuda(e);

  bool ok = true;
  if (L.halo) {
    ok = encode_2d(&L.tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, L.codes, static_cast<uint64_t>(bpp),
                   static_cast<uint64_t>(npix), static_cast<uint64_t>(bpp), 128,
                   static_cast<uint32_t>(L.hx.halo_rows));
    if (L.halo2)  // each CTA of a pair reads its 128 rows of a 256-row weight tile
      ok = ok && encode_2d(&L.tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, L.wq, static_cast<uint64_t>(kt),
                           static_cast<uint64_t>(no_tc), static_cast<uint64_t>(kt), 128, 128);
  } else if (L.fc) {
    const uint64_t K = static_cast<uint64_t>(L.H) * L.W * bpp;
    const uint64_t dims[4] = {K, 1, 1, static_cast<uint64_t>(L.N)};
    const uint64_t strides[3] = {K, K, K};
    const uint32_t box[4] = {128, 1, 1, 128};
    ok = encode_4d(&L.tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, L.codes, dims, strides, box);
  } else if (t.f32) {
    // the activation map is over each forward's input (input_map)
  } else {
    // box: 128 bytes of channels x (stride x Cw) columns x (stride x R) rows x Bn images,
    // stepping by the stride, so the copy lands Cw x R x Bn pixels = 128 rows
    const uint64_t dims[4] = {static_cast<uint64_t>(bpp), static_cast<uint64_t>(L.W), static_cast<uint64_t>(L.H),
                              static_cast<uint64_t>(L.N)};
    const uint64_t strides[3] = {static_cast<uint64_t>(bpp), static_cast<uint64_t>(bpp) * L.W,
                                 static_cast<uint64_t>(bpp) * L.W * L.H};
    const uint32_t box[4] = {128, static_cast<uint32_t>(t.sx * t.Cw), static_cast<uint32_t>(t.sy * t.R),
                             static_cast<uint32_t>(t.Bn)};
    const uint32_t estr[4] = {1, static_cast<uint32_t>(t.sx), static_cast<uint32_t>(t.sy), 1};
    ok = encode_4d(&L.tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, L.codes, dims, strides, box, estr);
  }
  // On SM pairs each CTA loads half of every weight tile (boxes of BN/2 rows).
  if (pairs > 0) {
    L.tc_pair = true;
    tc2_plan(t, pairs);
    if (t.sk) {  // partial sums of the items cut between pairs, and their ready flags
      const int cuts = t.grid_ctas / 2 - 1;
      cudaError_t e2 = L.tc_mem.alloc(&t.sk_part, static_cast<size_t>(cuts) * 2 * t.BN * 128);
      if (e2 == cudaSuccess) e2 = L.tc_mem.alloc(&t.sk_flag, static_cast<size_t>(cuts) * 2);
      if (e2 == cudaSuccess) e2 = cudaMemset(t.sk_flag, 0, sizeof(uint32_t) * cuts * 2);
      if (e2 != cudaSuccess) return from_cuda(e2);
    }
    ok = ok && encode_2d(&L.tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, L.wq, static_cast<uint64_t>(kt),
                         static_cast<uint64_t>(no_tc), static_cast<uint64_t>(kt), 128,
                         static_cast<uint32_t>(t.BN / 2));
    ok = ok && encode_2d(&L.tmBp, CU_TENSOR_MAP_DATA_TYPE_UINT8, L.wq, static_cast<uint64_t>(kt),
                         static_cast<uint64_t>(no_tc), static_cast<uint64_t>(kt), 128,
                         static_cast<uint32_t>(t.BN / t.pieces / 2));
  } else {
    t.grid_ctas = tc_plan(t, current_sm_count());  // work list: tail tiles cut along N
    if (t.f32 && t.m_tiles * t.n_tiles > t.grid_ctas) {
      // binaryWeights from fp32 input: the converting warps' work does not shrink with a tail
      // piece's channels, so the CTAs take equal contiguous shares of all tiles' k-blocks
      // instead (a tile cut between two CTAs finished by the first, with the second's raw
      // sums).  Batch 8, 112 x 112, 128 -> 128, stride 2: 36 k-blocks converted on the busiest
      // SM with tail pieces, 24 with equal shares.
      t.sk = 1;
      t.pieces = 1;
      t.full_tiles = t.m_tiles * t.n_tiles;
      const int cuts = t.grid_ctas - 1;
      cudaError_t e2 = L.tc_mem.alloc(&t.sk_part, static_cast<size_t>(cuts) * t.BN * 128);
      if (e2 == cudaSuccess) e2 = L.tc_mem.alloc(&t.sk_flag, static_cast<size_t>(cuts));
      if (e2 == cudaSuccess) e2 = cudaMemset(t.sk_flag, 0, sizeof(uint32_t) * cuts);
      if (e2 != cudaSuccess) return from_cuda(e2);
    }
    t.b_tiles = L.wq;
    L.hx.b_tiles = L.wq;
    L.hx.scale = L.scale;
    L.hx.bias = L.bias;
    L.hx.relu = L.relu;
    L.hx.err = L.err;
  }
  if (ok && t.k_splits > 1) ok = encode_out_map(L, &L.tmWs, L.ws);
  if (!ok) return BCONV_OK;  // the POPC path stays available
  L.tc_ok = true;
  return BCONV_OK;
}

// Copy the parameter arrays (expanding defaults) and prepare the weights for the
// contraction kernel of this layer type.
bconv_status_t upload_params(Layer& L, const uint32_t* packed, const float* scale, const float* bias,
                             const float* in_scale, const float* in_bias, float scale_value) {
  const int taps = L.kh * L.kw;
  std::vector<float> hs(L.No), hb(L.No, 0.f);
  for (int c = 0; c < L.No; ++c) hs[c] = scale ? scale[c] : scale_value;
  if (bias) memcpy(hb.data(), bias, sizeof(float) * L.No);
  cudaError_t e = L.mem.alloc(&L.scale, L.No);
  if (e == cudaSuccess) e = L.mem.alloc(&L.bias, L.No);
  if (e == cudaSuccess) e = cudaMemcpy(L.scale, hs.data(), sizeof(float) * L.No, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(L.bias, hb.data(), sizeof(float) * L.No, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return from_cuda(e);
  if (in_scale || in_bias) {  // both arrays exist on the device once either is given
    std::vector<float> is(L.Ni, 1.f), ib(L.Ni, 0.f);
    if (in_scale) memcpy(is.data(), in_scale, sizeof(float) * L.Ni);
    if (in_bias) memcpy(ib.data(), in_bias, sizeof(float) * L.Ni);
    e = L.mem.alloc(&L.in_scale, L.Ni);
    if (e == cudaSuccess) e = L.mem.alloc(&L.in_bias, L.Ni);
    if (e == cudaSuccess) e = cudaMemcpy(L.in_scale, is.data(), sizeof(float) * L.Ni, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(L.in_bias, ib.data(), sizeof(float) * L.Ni, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return from_cuda(e);
  }

  // Host weights: [No][taps][nw] LSB-first words.  Bits at or beyond Ni are cleared.
  const int tail = L.Ni % kWordBits;
  const uint32_t last_mask = tail ? ((1u << tail) - 1u) : 0xffffffffu;
  auto wword = [&](int c, int t, int w) -> uint32_t {
    uint32_t v = packed[(static_cast<int64_t>(c) * taps + t) * L.nw + w];
    return w == L.nw - 1 ? (v & last_mask) : v;
  };

  const Layer* src = L.weights_from;  // same shapes: its SIMT-family weights serve as they are
  if (L.type == kBinaryWeights) {
    // [bw_ni_pad][no_pad] of +-1.0f, zero for padding rows and columns.  Row index
    // t*ni_pad + f for a convolution; t*Ni + f (the flattened image) for the FC.
    const bool borrowed = src && src->wf;
    std::vector<float> hw(borrowed ? 0 : static_cast<size_t>(L.fc ? 1 : taps) * L.bw_ni_pad * L.no_pad, 0.f);
    for (int c = 0; c < (borrowed ? 0 : L.No); ++c)
      for (int t = 0; t < taps; ++t)
        for (int f = 0; f < L.Ni; ++f) {
          const uint32_t bit = (wword(c, t, f / kWordBits) >> (f % kWordBits)) & 1u;
          const int64_t row = L.fc ? static_cast<int64_t>(t) * L.Ni + f : static_cast<int64_t>(t) * L.bw_ni_pad + f;
          hw[row * L.no_pad + c] = bit ? 1.f : -1.f;
        }
    if (borrowed) {
      L.wf = src->wf;
    } else {
      e = L.mem.alloc(&L.wf, hw.size());
      if (e == cudaSuccess) e = cudaMemcpy(L.wf, hw.data(), hw.size() * sizeof(float), cudaMemcpyHostToDevice);
    }
    if (e == cudaSuccess && L.fc && L.in_scale) {  // terms repeated over the flattened image
      std::vector<float> is(static_cast<size_t>(L.bw_ni)), ib(static_cast<size_t>(L.bw_ni));
      std::vector<float> s1(L.Ni, 1.f), b0(L.Ni, 0.f);
      if (in_scale) memcpy(s1.data(), in_scale, sizeof(float) * L.Ni);
      if (in_bias) memcpy(b0.data(), in_bias, sizeof(float) * L.Ni);
      for (int64_t k = 0; k < L.bw_ni; ++k) {
        is[k] = s1[k % L.Ni];
        ib[k] = b0[k % L.Ni];
      }
      e = L.mem.alloc(&L.bw_in_scale, is.size());
      if (e == cudaSuccess) e = L.mem.alloc(&L.bw_in_bias, ib.size());
      if (e == cudaSuccess) e = cudaMemcpy(L.bw_in_scale, is.data(), is.size() * sizeof(float), cudaMemcpyHostToDevice);
      if (e == cudaSuccess) e = cudaMemcpy(L.bw_in_bias, ib.data(), ib.size() * sizeof(float), cudaMemcpyHostToDevice);
    } else {
      L.bw_in_scale = L.in_scale;
      L.bw_in_bias = L.in_bias;
    }
    return from_cuda(e);
  }

  // POPC weights: reduction-major [taps*nw_pad][no_pad], zero padding; per-tap popcounts.
  if (src && src->wt && src->wpop) {
    L.wt = src->wt;
    L.wpop = src->wpop;
    return BCONV_OK;
  }
  const int64_t K = static_cast<int64_t>(taps) * L.nw_pad;
  std::vector<uint32_t> hw(static_cast<size_t>(K) * L.no_pad, 0u);
  std::vector<int32_t> hp(static_cast<size_t>(L.No) * taps, 0);
  for (int c = 0; c < L.No; ++c)
    for (int t = 0; t < taps; ++t) {
      int32_t pc = 0;
      for (int w = 0; w < L.nw; ++w) {
        const uint32_t v = wword(c, t, w);
        hw[(static_cast<int64_t>(t) * L.nw_pad + w) * L.no_pad + c] = v;
        pc += __builtin_popcount(v);
      }
      hp[static_cast<size_t>(c) * taps + t] = pc;
    }
  e = L.mem.alloc(&L.wt, hw.size());
  if (e == cudaSuccess) e = L.mem.alloc(&L.wpop, hp.size());
  if (e == cudaSuccess) e = cudaMemcpy(L.wt, hw.data(), hw.size() * sizeof(uint32_t), cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(L.wpop, hp.data(), hp.size() * sizeof(int32_t), cudaMemcpyHostToDevice);
  return from_cuda(e);
}

bconv_status_t alloc_workspace(Layer& L) {
  const int64_t npix = static_cast<int64_t>(L.N) * L.H * L.W;
  cudaError_t e = L.mem.alloc(&L.err, 1);
  if (e == cudaSuccess) e = cudaMemset(L.err, 0, sizeof(uint32_t));
  if (e == cudaSuccess && L.type != kBinaryWeights) e = L.mem.alloc(&L.bits, npix * L.nw_pad);
  if (e == cudaSuccess && L.use_beta()) e = L.mem.alloc(&L.A, npix);
  if (e == cudaSuccess && L.use_beta()) e = L.mem.alloc(&L.beta, static_cast<int64_t>(L.N) * L.Ho * L.Wo);
  return from_cuda(e);
}

// Keep what creating the layer took, for the chunk layers of the host-buffer forward.
void keep_host_params(Layer& L, const uint32_t* packed, const float* scale, const float* bias,
                      const float* in_scale, const float* in_bias, float scale_value) {
  const int64_t taps = L.fc ? 1 : static_cast<int64_t>(L.kh) * L.kw;
  const int64_t words = L.fc ? static_cast<int64_t>(L.No) * L.H * L.W * words_for(L.Ni)
                             : static_cast<int64_t>(L.No) * taps * words_for(L.Ni);
  L.h_packed.assign(packed, packed + words);
  if (scale) L.h_scale.assign(scale, scale + L.No);
  if (bias) L.h_bias.assign(bias, bias + L.No);
  if (in_scale) L.h_in_scale.assign(in_scale, in_scale + L.Ni);
  if (in_bias) L.h_in_bias.assign(in_bias, in_bias + L.Ni);
  L.h_scale_value = scale_value;
}

bconv_status_t finish_create(Layer& L, const uint32_t* packed, const float* scale, const float* bias,
                             const float* in_scale, const float* in_bias, float scale_value) {
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
    cudaGetLastError();
    return BCONV_ERR_NO_DEVICE;
  }
  if (cudaGetDevice(&L.device) != cudaSuccess) return BCONV_ERR_CUDA;
  L.nw = words_for(L.Ni);
  L.nw_pad = round_up(L.nw, kWordPad);
  L.bw_ni = L.fc ? L.H * L.W * L.Ni : L.Ni;
  L.bw_ni_pad = round_up(L.bw_ni, kBwChanPad);
  L.no_pad = round_up(L.No, kTileN);
  bconv_status_t st = upload_params(L, packed, scale, bias, in_scale, in_bias, scale_value);
  if (st == BCONV_OK) st = alloc_workspace(L);
  if (st == BCONV_OK) st = setup_tc(L, packed);
  if (st != BCONV_OK) {
    L.tc_mem.release();
    L.mem.release();
  }
  return st;
}

bool use_tc(const Layer& L) {
  return L.tc_ok && (L.algo == BCONV_ALGO_AUTO || L.algo == BCONV_ALGO_TCGEN05);
}

// The input and output forms of one forward: fp32 (in / out) or bit-packed (bits + A).
struct Io {
  const float* in = nullptr;
  const uint32_t* in_bits = nullptr;
  const float* in_a = nullptr;
  float* out = nullptr;
  uint32_t* out_bits = nullptr;
  float* out_a = nullptr;
};

// Whether the tensor-core epilogue writes the bit-packed output itself.
bool tc_emits_bits(const Layer& L) { return use_tc(L) && !L.fc && L.tc.k_splits == 1; }

// Tensor-core forward: int8 codes (+ A) -> [beta] -> tcgen05 contraction [-> finalize].
bconv_status_t run_forward_tc(Layer& L, const Io& io, cudaStream_t s) {
  const float* in = io.in;
  float* out = io.out;
  const bool beta = L.use_beta();
  const float* A = io.in_bits ? io.in_a : L.A;
  cudaError_t e = cudaSuccess;
  if (io.in_bits) {
    e = L.tc.kind == 2 ? launch_unpack_bits_f4(io.in_bits, static_cast<int64_t>(L.N) * L.H * L.W, L.Ni, L.cip,
                                               L.type, L.codes, s, L.pad)
                       : launch_unpack_bits_i8(io.in_bits, static_cast<int64_t>(L.N) * L.H * L.W, L.Ni, L.cip,
                                               L.type, L.codes, s);
    if (e == cudaSuccess && L.halo && beta)  // the caller's A into the padded grid the kernel reads
      e = launch_pad_copy(io.in_a, static_cast<int64_t>(L.N) * L.H * L.W, L.pad, L.A_pad, s);
  } else if (L.tc.kind != 1) {
    PackI8Args p{};
    p.in = in;
    p.npix = static_cast<int64_t>(L.N) * L.H * L.W;
    p.ni = L.Ni;
    p.cip = L.cip;
    p.in_scale = L.in_scale;
    p.in_bias = L.in_bias;
    p.codes = L.codes;
    p.A = beta ? (L.halo ? L.A_pad : L.A) : nullptr;  // A follows the codes into the padded grid
    p.op = L.type;
    p.f4 = L.tc.kind == 2;
    p.pad = L.pad;
    p.err = L.err;
    e = launch_pack_i8(p, s);
  } else if (L.tc.f32) {
    e = cudaSuccess;  // binaryWeights from fp32 input: the contraction reads `in` itself (no pack, no A)
  } else {
    PackBf16x3Args p{};
    p.in = in;
    p.npix = static_cast<int64_t>(L.N) * L.H * L.W;
    p.ni = L.Ni;
    p.cip = L.cip;
    p.in_scale = L.in_scale;
    p.in_bias = L.in_bias;
    p.parts = reinterpret_cast<uint16_t*>(L.codes);
    p.A = beta ? L.A : nullptr;
    e = launch_pack_bf16x3(p, s);
  }
  if (e != cudaSuccess) return from_cuda(e);
  if (L.fcb) {  // the FC kernel forms beta and finishes split tiles in its own epilogue
    FcArgs f = L.fx;
    f.A = beta ? A : nullptr;
    f.out = out;
    const bool timed = L.prof.take();
    if (timed) cudaEventRecord(L.prof.start[L.prof.used], s);
    e = launch_tc_fc(&L.tmA, f, s);
    if (timed) cudaEventRecord(L.prof.stop[L.prof.used++], s);
    return from_cuda(e);
  }
  // the convolution forms beta from A inside its epilogue, a split FC inside the finalize
  if (beta && L.fc && L.tc.k_splits == 1) {
    BetaArgs b{A, L.beta, L.N, L.H, L.W, L.Ho, L.Wo, L.kh, L.kw, L.sy, L.sx};
    e = launch_beta_image_mean(b, s);
    if (e != cudaSuccess) return from_cuda(e);
  }
  TcArgs t = L.tc;
  t.beta = beta ? L.beta : nullptr;
  t.A = (beta && !L.fc) ? A : nullptr;
  t.H = L.H;
  t.W = L.W;
  const CUtensorMap* om = &L.tmWs;
  if (io.out_bits) {  // the epilogue binarizes; the output map is not used
    t.out_bits = io.out_bits;
    t.out_a = io.out_a;
    t.next_scale = L.next_scale;
    t.next_bias = L.next_bias;
    t.nwo = words_for(L.No);
    t.a_part = L.a_part;
    t.a_count = L.a_count;
    om = &L.tmOut;
  } else if (t.k_splits > 1) {
    // the workspace is zero: at allocation, then as each finalize reads it
  } else if (!L.halo) {  // the rows-staged kernel stores without a tensor map
    if (out != L.tm_out_ptr) {
      if (!encode_out_map(L, &L.tmOut, out)) return BCONV_ERR_CUDA;
      L.tm_out_ptr = out;
    }
    om = &L.tmOut;
  }
  const bool timed = L.prof.take();
  if (timed) cudaEventRecord(L.prof.start[L.prof.used], s);
  if (L.halo) {
    HaloArgs h = L.hx;
    h.A = beta ? L.A_pad : nullptr;
    h.out = out;
    e = L.halo2 ? launch_tc_halo2(&L.tmA, &L.tmB, h, s) : launch_tc_halo(&L.tmA, h, s);
  } else if (t.f32) {
    const CUtensorMap* xm = input_map(L, in);
    e = xm ? launch_tc_conv(xm, om, t, s) : cudaErrorInvalidValue;
  } else {
    e = L.tc_pair ? launch_tc_conv2(&L.tmA, &L.tmB, &L.tmBp, om, t, s) : launch_tc_conv(&L.tmA, om, t, s);
  }
  if (timed) cudaEventRecord(L.prof.stop[L.prof.used++], s);
  if (e != cudaSuccess) return from_cuda(e);
  if (t.k_splits > 1)
    e = launch_tc_finalize(L.ws, out, L.scale, L.bias, beta ? A : nullptr, L.H * L.W, L.N, L.No, L.relu, s);
  return from_cuda(e);
}

// The launch sequence of one forward on the POPC / SIMT families (fp32 output).
bconv_status_t run_forward_simt(Layer& L, const Io& io, cudaStream_t s) {
  const float* in = io.in;
  float* out = io.out;
  const int64_t npix = static_cast<int64_t>(L.N) * L.H * L.W;
  cudaError_t e = cudaSuccess;
  const bool beta = L.use_beta();
  const float* A = io.in_bits ? io.in_a : L.A;

  // 1. input transform + sign + pack (+ A), or the caller's bits into the padded layout
  if (io.in_bits) {
    e = launch_repack_bits(io.in_bits, npix, L.Ni, L.nw_pad, L.bits, s);
    if (e != cudaSuccess) return from_cuda(e);
  } else if (L.type != kBinaryWeights || beta) {
    PackArgs p{};
    p.in = in;
    p.npix = npix;
    p.ni = L.Ni;
    p.nw_pad = L.nw_pad;
    p.in_scale = L.in_scale;
    p.in_bias = L.in_bias;
    p.bits = L.type != kBinaryWeights ? L.bits : nullptr;
    p.A = beta ? L.A : nullptr;
    e = launch_pack(p, s);
    if (e != cudaSuccess) return from_cuda(e);
  }
  // 2. beta
  if (beta) {
    BetaArgs b{A, L.beta, L.N, L.H, L.W, L.Ho, L.Wo, L.kh, L.kw, L.sy, L.sx};
    e = L.fc ? launch_beta_image_mean(b, s) : launch_beta_conv(b, s);
    if (e != cudaSuccess) return from_cuda(e);
  }
  // 3. contraction + epilogue (timed when profiling)
  const bool timed = L.prof.take();
  if (timed) cudaEventRecord(L.prof.start[L.prof.used], s);
  if (L.type == kBinaryWeights) {
    BwArgs b{};
    b.in = in;
    b.in_scale = L.bw_in_scale;
    b.in_bias = L.bw_in_bias;
    b.wf = L.wf;
    b.scale = L.scale;
    b.bias = L.bias;
    b.beta = beta ? L.beta : nullptr;
    b.out = out;
    b.ni = L.bw_ni; b.ni_pad = L.bw_ni_pad; b.no = L.No; b.no_pad = L.no_pad;
    b.relu = L.relu;
    b.vec_out = (L.No % 4 == 0) && (reinterpret_cast<uintptr_t>(out) & 15) == 0;
    if (L.fc) {  // one "pixel" per image whose channels are the flattened image, one tap
      b.N = L.N; b.H = 1; b.W = 1; b.Ho = 1; b.Wo = 1; b.kh = 1; b.kw = 1; b.sy = 1; b.sx = 1;
    } else {
      b.N = L.N; b.H = L.H; b.W = L.W; b.Ho = L.Ho; b.Wo = L.Wo;
      b.kh = L.kh; b.kw = L.kw; b.sy = L.sy; b.sx = L.sx;
    }
    e = launch_bw_conv(b, s);
  } else {
    PopcArgs p{};
    p.bits = L.bits;
    p.wt = L.wt;
    p.wpop = L.wpop;
    p.scale = L.scale;
    p.bias = L.bias;
    p.beta = beta ? L.beta : nullptr;
    p.out = out;
    p.no = L.No;
    p.no_pad = L.no_pad;
    p.op = L.type;
    p.relu = L.relu;
    p.vec_out = (L.No % 4 == 0) && (reinterpret_cast<uintptr_t>(out) & 15) == 0;
    if (L.fc) {  // one "pixel" per image holding all H*W*nw_pad words, one tap
      p.N = L.N; p.H = 1; p.W = 1; p.Ho = 1; p.Wo = 1; p.kh = 1; p.kw = 1; p.sy = 1; p.sx = 1;
      p.nw = L.H * L.W * L.nw_pad;
      p.nbits = L.H * L.W * L.Ni;
    } else {
      p.N = L.N; p.H = L.H; p.W = L.W; p.Ho = L.Ho; p.Wo = L.Wo;
      p.kh = L.kh; p.kw = L.kw; p.sy = L.sy; p.sx = L.sx;
      p.nw = L.nw_pad;
      p.nbits = L.Ni;
    }
    const int64_t m_tiles = ceil_div(static_cast<int64_t>(p.N) * p.Ho * p.Wo, 128);
    const int ksteps = p.kh * p.kw * (p.nw / kWordPad);
    p.split_k = popc_split_k_for(m_tiles, p.no_pad / kTileN, ksteps, current_sm_count());
    e = launch_popc_gemm(p, s);
  }
  if (timed) cudaEventRecord(L.prof.stop[L.prof.used++], s);
  return from_cuda(e);
}

// One forward with the given input and output forms.
// The fp32-input binaryWeights contraction maps the input for the TMA: it needs it 16-byte
// aligned (a forward with another input runs on the SIMT family).
bool tc_input_ok(const Layer& L, const float* in) {
  return use_tc(L) && (!L.tc.f32 || (reinterpret_cast<uintptr_t>(in) & 15u) == 0);
}

bconv_status_t run_io(Layer& L, const Io& io, cudaStream_t s) {
  if (L.N == 0) return BCONV_OK;
  if (io.out_bits && !tc_emits_bits(L)) {
    // fp32 output into the handle's buffer, then the next layer's transform, sign and A
    Io fp = io;
    fp.out = L.y_scratch;
    fp.out_bits = nullptr;
    fp.out_a = nullptr;
    bconv_status_t st = tc_input_ok(L, io.in) ? run_forward_tc(L, fp, s) : run_forward_simt(L, fp, s);
    if (st != BCONV_OK) return st;
    PackArgs p{};
    p.in = L.y_scratch;
    p.npix = static_cast<int64_t>(L.N) * L.Ho * L.Wo;
    p.ni = L.No;
    p.nw_pad = words_for(L.No);
    p.in_scale = L.next_scale;
    p.in_bias = L.next_bias;
    p.bits = io.out_bits;
    p.A = io.out_a;
    return from_cuda(launch_pack(p, s));
  }
  // The tensor-core kernels write the output in 16-byte pieces (TMA boxes, float4 stores); an
  // output that is not 16-byte aligned goes to the SIMT family, which can write it.
  const bool aligned = (reinterpret_cast<uintptr_t>(io.out) & 15u) == 0;
  return tc_input_ok(L, io.in) && aligned ? run_forward_tc(L, io, s) : run_forward_simt(L, io, s);
}

bconv_status_t run_forward(Layer& L, const float* in, float* out, cudaStream_t s) {
  Io io;
  io.in = in;
  io.out = out;
  return run_io(L, io, s);
}

// Buffers a bit-packed output needs with the current kernel family (kept until destroy).
// Set the tensor-core path up again with the given operand codes (the previous plan's
// buffers are freed first; cudaFree waits for work still using them).
bconv_status_t replan_tc(Layer& L, int codes) {
  L.tc_mem.release();
  L.tc = TcArgs{};
  L.tc_ok = false;
  L.tc_pair = false;
  L.wq = nullptr;
  L.codes = nullptr;
  L.ws = nullptr;
  L.tm_out_ptr = nullptr;
  L.halo = false;
  L.halo2 = false;
  L.A_pad = nullptr;
  L.fcb = false;
  for (int i = 0; i < 4; ++i) L.tmX_ptr[i] = nullptr;  // their boxes follow the old tile shape
  L.tmX_next = 0;
  L.codes_override = codes;
  return setup_tc(L, L.h_packed.data());
}

bconv_status_t ensure_bits_buffers(Layer& L) {
  if (!L.has_next || L.N == 0) return BCONV_OK;
  cudaError_t e = cudaSuccess;
  if (tc_emits_bits(L)) {
    const int slices = L.tc.n_tiles * L.tc.pieces;
    if (slices > 1 && !L.a_part) {
      e = L.mem.alloc(&L.a_part, static_cast<size_t>(slices) * L.N * L.Ho * L.Wo);
      if (e == cudaSuccess) e = L.mem.alloc(&L.a_count, static_cast<size_t>(L.tc.m_tiles));
      if (e == cudaSuccess) e = cudaMemset(L.a_count, 0, sizeof(uint32_t) * L.tc.m_tiles);
    }
  } else if (!L.y_scratch) {
    e = L.mem.alloc(&L.y_scratch, static_cast<size_t>(L.out_elems()));
  }
  return from_cuda(e);
}

bconv_status_t set_output_terms(Layer& L, const float* next_scale, const float* next_bias) {
  std::vector<float> hs(L.No, 1.f), hb(L.No, 0.f);
  if (next_scale) memcpy(hs.data(), next_scale, sizeof(float) * L.No);
  if (next_bias) memcpy(hb.data(), next_bias, sizeof(float) * L.No);
  cudaError_t e = cudaSuccess;
  if (!L.next_scale) e = L.mem.alloc(&L.next_scale, L.No);
  if (e == cudaSuccess && !L.next_bias) e = L.mem.alloc(&L.next_bias, L.No);
  if (e == cudaSuccess) e = cudaMemcpy(L.next_scale, hs.data(), sizeof(float) * L.No, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(L.next_bias, hb.data(), sizeof(float) * L.No, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return from_cuda(e);
  // A convolution on e2m1 codes whose pixels span several channel tiles re-plans on int8 codes
  // (256-channel tiles) for a bit-packed output: each pixel's words and sum of |x~'| are then
  // formed within one work item instead of being added across items.  Measured on B200, batch
  // 16, 56 x 56, 256 -> 256 as a chain's middle layer: 53.3 us per forward on e2m1 codes
  // (two 128-channel tiles), 37.1 us on int8.
  // (The per-tap kernel's e2m1 tiles are at most 128 channels wide, whatever the rows-staged
  // plan used.)
  if (L.tc_ok && L.tc.kind == 2 && !L.fc && L.No > 128 && L.codes_override < 0) {
    L.halo_off = true;
    const bconv_status_t st = replan_tc(L, BCONV_CODES_INT8);
    if (st != BCONV_OK) return st;
  } else if (L.halo) {  // the rows-staged kernel writes fp32 only: the per-tap kernel emits the bits
    L.halo_off = true;
    const bconv_status_t st = replan_tc(L, L.codes_override);
    if (st != BCONV_OK) return st;
  } else if (L.tc_ok && L.tc.f32) {  // so does the fp32-input kernel: the parts path emits them
    L.f32_off = true;
    const bconv_status_t st = replan_tc(L, L.codes_override);
    if (st != BCONV_OK) return st;
  }
  L.has_next = true;
  return ensure_bits_buffers(L);
}

bconv_status_t forward_io(Layer& L, const bconv_io_t* io, cudaStream_t s) {
  if (!io) return BCONV_ERR_INVALID_ARG;
  if ((io->in == nullptr) == (io->in_bits == nullptr)) return BCONV_ERR_INVALID_ARG;
  if ((io->out == nullptr) == (io->out_bits == nullptr)) return BCONV_ERR_INVALID_ARG;
  if (io->in_bits) {
    if (L.type == kBinaryWeights) return BCONV_ERR_UNSUPPORTED;  // needs the full-precision input
    if (L.in_scale) return BCONV_ERR_INVALID_ARG;  // the producer of the bits applied the input terms
    if (L.use_beta() && !io->in_a) return BCONV_ERR_INVALID_ARG;
  }
  if (io->out_bits && (!io->out_a || !L.has_next)) return BCONV_ERR_INVALID_ARG;
  Io v;
  v.in = io->in;
  v.in_bits = io->in_bits;
  v.in_a = io->in_a;
  v.out = io->out;
  v.out_bits = io->out_bits;
  v.out_a = io->out_a;
  return run_io(L, v, s);
}

// Image chunks of a host-buffer forward: 4 (else 2) when that divides the batch and keeps
// every chunk's copies at 2 MB or more.  With k chunks the copies in and out overlap except
// for about 1/k of the transfer at either end, and each chunk adds its launch and copy
// overheads.  Measured on B200 with page-locked buffers (copies alone: 45 GB/s in, 56 GB/s
// out): batch 16 x 56 x 56 x 256 in and out, 1.61 / 1.42 / 1.45 / 1.60 ms per call with
// 2 / 4 / 8 / 16 chunks; the FC of 256 x 7 x 7 x 512, 0.57 / 0.55 / 0.58 / 0.64 ms.
int host_chunks(const Layer& L) {
  const int64_t bytes = (L.in_elems() + L.out_elems()) * static_cast<int64_t>(sizeof(float));
  if (L.h_packed.empty() || bytes < (int64_t{8} << 20)) return 1;
  for (int k : {4, 2})
    if (L.N % k == 0 && bytes / k >= (int64_t{2} << 20)) return k;
  return 1;
}

void clear_chunks(Layer& L) {
  for (auto& c : L.chunks) {
    c->tc_mem.release();
    c->mem.release();
  }
  L.chunks.clear();
}

// The chunk layers: the same layer on batch N / k, set up from the kept host parameters; the
// first owns the device weights, the others read them, and all report to the parent's error word.
bconv_status_t make_chunks(Layer& L, int k) {
  clear_chunks(L);
  for (int i = 0; i < k; ++i) {
    std::unique_ptr<Layer> c(new (std::nothrow) Layer());
    if (!c) return BCONV_ERR_OOM;
    c->type = L.type;
    c->flags = L.flags;
    c->relu = L.relu;
    c->fc = L.fc;
    c->N = L.N / k; c->H = L.H; c->W = L.W; c->Ni = L.Ni; c->No = L.No;
    c->kh = L.kh; c->kw = L.kw; c->sy = L.sy; c->sx = L.sx; c->Ho = L.Ho; c->Wo = L.Wo;
    c->weights_from = i > 0 ? L.chunks[0].get() : nullptr;
    auto opt = [](const std::vector<float>& v) { return v.empty() ? nullptr : v.data(); };
    const bconv_status_t st = finish_create(*c, L.h_packed.data(), opt(L.h_scale), opt(L.h_bias), opt(L.h_in_scale),
                                            opt(L.h_in_bias), L.h_scale_value);
    if (st != BCONV_OK) {
      clear_chunks(L);
      return st;
    }
    c->err = L.err;  // one error word for the layer
    c->tc.err = L.err;
    L.chunks.push_back(std::move(c));
  }
  cudaError_t e = cudaSuccess;
  if (!L.copy_in) e = cudaStreamCreateWithFlags(&L.copy_in, cudaStreamNonBlocking);
  if (e == cudaSuccess && !L.copy_out) e = cudaStreamCreateWithFlags(&L.copy_out, cudaStreamNonBlocking);
  while (e == cudaSuccess && L.chunk_events.size() < static_cast<size_t>(2 * k + 1)) {
    cudaEvent_t ev;
    e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming);
    if (e == cudaSuccess) L.chunk_events.push_back(ev);
  }
  return from_cuda(e);
}

bconv_status_t forward_host(Layer& L, const float* hin, float* hout, cudaStream_t s) {
  if (!hin || !hout) return BCONV_ERR_INVALID_ARG;
  cudaError_t e = cudaSuccess;
  if (!L.stage_in) e = L.mem.alloc(&L.stage_in, L.in_elems());
  if (e == cudaSuccess && !L.stage_out) e = L.mem.alloc(&L.stage_out, L.out_elems());
  if (e != cudaSuccess) return from_cuda(e);
  const int k = host_chunks(L);
  if (k > 1 && L.chunks.size() != static_cast<size_t>(k) && make_chunks(L, k) != BCONV_OK) clear_chunks(L);
  if (k > 1 && L.chunks.size() == static_cast<size_t>(k)) {
    // copy in on one stream, compute on `stream`, copy out on another, chunk by chunk
    const int64_t in_c = L.in_elems() / k, out_c = L.out_elems() / k;
    cudaEvent_t start = L.chunk_events[2 * k];
    e = cudaEventRecord(start, s);  // the staging buffers are free once earlier work on `stream` is done
    if (e == cudaSuccess) e = cudaStreamWaitEvent(L.copy_in, start, 0);
    for (int i = 0; i < k && e == cudaSuccess; ++i) {
      Layer& c = *L.chunks[i];
      c.algo = L.algo;
      e = cudaMemcpyAsync(L.stage_in + i * in_c, hin + i * in_c, in_c * sizeof(float), cudaMemcpyHostToDevice,
                          L.copy_in);
      if (e == cudaSuccess) e = cudaEventRecord(L.chunk_events[2 * i], L.copy_in);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(s, L.chunk_events[2 * i], 0);
      if (e != cudaSuccess) break;
      const bconv_status_t st = run_forward(c, L.stage_in + i * in_c, L.stage_out + i * out_c, s);
      if (st != BCONV_OK) {
        cudaStreamSynchronize(L.copy_in);
        cudaStreamSynchronize(L.copy_out);
        return st;
      }
      e = cudaEventRecord(L.chunk_events[2 * i + 1], s);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(L.copy_out, L.chunk_events[2 * i + 1], 0);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(hout + i * out_c, L.stage_out + i * out_c, out_c * sizeof(float), cudaMemcpyDeviceToHost,
                            L.copy_out);
    }
    const cudaError_t e1 = cudaStreamSynchronize(L.copy_out);
    const cudaError_t e2 = cudaStreamSynchronize(s);
    return from_cuda(e != cudaSuccess ? e : (e1 != cudaSuccess ? e1 : e2));
  }
  e = cudaMemcpyAsync(L.stage_in, hin, L.in_elems() * sizeof(float), cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return from_cuda(e);
  bconv_status_t st = run_forward(L, L.stage_in, L.stage_out, s);
  if (st != BCONV_OK) return st;
  e = cudaMemcpyAsync(hout, L.stage_out, L.out_elems() * sizeof(float), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  return from_cuda(e);
}

bconv_status_t sync_status(Layer& L, cudaStream_t s) {
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return from_cuda(e);
  uint32_t word = 0;
  e = cudaMemcpy(&word, L.err, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return from_cuda(e);
  if (word) {
    cudaMemset(L.err, 0, sizeof(uint32_t));
    if (L.a_count) cudaMemset(L.a_count, 0, sizeof(uint32_t) * L.tc.m_tiles);  // an aborted launch may leave counts
    if (L.tc.sk_flag)  // and flags (pairs: two per cut between pairs; one SM: one per cut between CTAs)
      cudaMemset(L.tc.sk_flag, 0, sizeof(uint32_t) * (L.tc_pair ? (L.tc.grid_ctas / 2 - 1) * 2 : L.tc.grid_ctas - 1));
    if (L.ws) cudaMemset(L.ws, 0, sizeof(float) * static_cast<size_t>(L.N) * L.No);  // and partial sums
    if (word & kErrTimeout) return BCONV_ERR_TIMEOUT;
    return BCONV_ERR_CUDA;  // kErrLayout: a kernel refused an unexpected shared-memory layout
  }
  return BCONV_OK;
}

bconv_status_t set_algo(Layer& L, int algo) {
  const bool ok = algo == BCONV_ALGO_AUTO || (algo == BCONV_ALGO_POPC && (L.type == kXnor || L.type == kAnd)) ||
                  (algo == BCONV_ALGO_SIMT_F32 && L.type == kBinaryWeights) ||
                  (algo == BCONV_ALGO_TCGEN05 && L.tc_ok);
  if (ok) {
    L.algo = algo;
    return ensure_bits_buffers(L);
  }
  if (algo < 0 || algo > BCONV_ALGO_TCGEN05) return BCONV_ERR_INVALID_ARG;
  return BCONV_ERR_UNSUPPORTED;
}

int launches_per_forward(const Layer& L) {
  if (L.N > 0 && use_tc(L) && L.tc.f32) return 1;  // binaryWeights from fp32 input: the contraction alone
  if (L.N > 0 && use_tc(L) && L.fcb) return 2;  // pack, the FC kernel (which finishes its own tiles)
  if (L.N > 0 && use_tc(L))  // pack, contraction; a split FC adds the finalize, an unsplit FC with beta its mean
    return 2 + (L.tc.k_splits > 1 ? 1 : ((L.fc && L.use_beta()) ? 1 : 0));
  int n = 1;  // contraction
  if (L.type != kBinaryWeights || L.use_beta()) n += 1;  // pack
  if (L.use_beta()) n += 1;                              // beta
  return n;
}

int effective_algo(const Layer& L) {
  if (use_tc(L)) return BCONV_ALGO_TCGEN05;
  return L.type == kBinaryWeights ? BCONV_ALGO_SIMT_F32 : BCONV_ALGO_POPC;
}

bconv_status_t profile_begin(Layer& L, int32_t n) {
  if (n <= 0 || n > (1 << 20)) return BCONV_ERR_INVALID_ARG;
  L.prof.clear();
  for (int i = 0; i < n; ++i) {
    cudaEvent_t a, b;
    if (cudaEventCreate(&a) != cudaSuccess) return BCONV_ERR_CUDA;
    if (cudaEventCreate(&b) != cudaSuccess) {
      cudaEventDestroy(a);
      return BCONV_ERR_CUDA;
    }
    L.prof.start.push_back(a);
    L.prof.stop.push_back(b);
  }
  L.prof.active = true;
  L.prof.every = 1;
  L.prof.seen = 0;
  return BCONV_OK;
}

bconv_status_t profile_stride(Layer& L, int32_t every) {
  if (every <= 0) return BCONV_ERR_INVALID_ARG;
  L.prof.every = every;
  L.prof.seen = 0;
  return BCONV_OK;
}

bconv_status_t profile_end(Layer& L, float* total_ms, int32_t* launches) {
  float total = 0.f;
  for (int i = 0; i < L.prof.used; ++i) {
    if (cudaEventSynchronize(L.prof.stop[i]) != cudaSuccess) return BCONV_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, L.prof.start[i], L.prof.stop[i]) != cudaSuccess) return BCONV_ERR_CUDA;
    total += ms;
  }
  if (total_ms) *total_ms = total;
  if (launches) *launches = L.prof.used;
  L.prof.clear();
  return BCONV_OK;
}

void destroy(Layer& L) {
  DeviceGuard g(L.device);
  L.prof.clear();
  clear_chunks(L);
  for (cudaEvent_t ev : L.chunk_events) cudaEventDestroy(ev);
  L.chunk_events.clear();
  if (L.copy_in) cudaStreamDestroy(L.copy_in);
  if (L.copy_out) cudaStreamDestroy(L.copy_out);
  L.copy_in = L.copy_out = nullptr;
  L.tc_mem.release();
  L.mem.release();
}

template <typename H>
H* checked(H* h, uint32_t magic) {
  return (h && h->magic == magic) ? h : nullptr;
}

}  // namespace
}  // namespace bconv

using namespace bconv;

extern "C" {

bconv_status_t bconv_create(const bconv_desc_t* d, const uint32_t* packed_weights, const float* scale,
                            const float* bias, const float* in_scale, const float* in_bias, bconv_type_t type,
                            uint32_t flags, bconv_handle_t* out) {
  if (!out) return BCONV_ERR_INVALID_ARG;
  *out = nullptr;
  if (!d || !packed_weights) return BCONV_ERR_INVALID_ARG;
  if (!valid_type(type) || (flags & ~static_cast<uint32_t>(BCONV_FLAG_USE_BETA_SCALING))) return BCONV_ERR_INVALID_ARG;
  const bconv_status_t shape = check_conv_shape(d);
  if (shape != BCONV_OK) return shape;
  bconv_handle_s* h = new (std::nothrow) bconv_handle_s();
  if (!h) return BCONV_ERR_OOM;
  h->magic = kConvMagic;
  Layer& L = h->L;
  L.type = type;
  L.flags = flags;
  L.relu = d->neuron == BCONV_NEURON_RELU;
  L.N = d->batch; L.H = d->in_h; L.W = d->in_w; L.Ni = d->in_channels; L.No = d->out_channels;
  L.kh = d->kernel_h; L.kw = d->kernel_w; L.sy = d->stride_y; L.sx = d->stride_x;
  L.Ho = (L.H + L.sy - 1) / L.sy;
  L.Wo = (L.W + L.sx - 1) / L.sx;
  const bconv_status_t st = finish_create(L, packed_weights, scale, bias, in_scale, in_bias, d->scale_value);
  if (st == BCONV_OK) keep_host_params(L, packed_weights, scale, bias, in_scale, in_bias, d->scale_value);
  if (st != BCONV_OK) {
    h->magic = 0;
    delete h;
    return st;
  }
  *out = h;
  return BCONV_OK;
}

bconv_status_t bconv_forward(bconv_handle_t h, const float* in, float* out, struct CUstream_st* stream) {
  if (!checked(h, kConvMagic) || (h->L.N > 0 && (!in || !out))) return BCONV_ERR_INVALID_ARG;
  DeviceGuard g(h->L.device);
  if (!g.ok) return BCONV_ERR_CUDA;
  return run_forward(h->L, in, out, stream);
}

bconv_status_t bconv_set_output_terms(bconv_handle_t h, const float* next_in_scale, const float* next_in_bias) {
  if (!checked(h, kConvMagic)) return BCONV_ERR_INVALID_ARG;
  DeviceGuard g(h->L.device);
  if (!g.ok) return BCONV_ERR_CUDA;
  return set_output_terms(h->L, next_in_scale, next_in_bias);
}

bconv_status_t bconv_forward_io(bconv_handle_t h, const bconv_io_t* io, struct CUstream_st* stream) {
  if (!checked(h, kConvMagic)) return BCONV_ERR_INVALID_ARG;
  DeviceGuard g(h->L.device);
  if (!g.ok) return BCONV_ERR_CUDA;
  return forward_io(h->L, io, stream);
}

bconv_status_t bconv_forward_host(bconv_handle_t h, const float* host_in, float* host_out,
                                  struct CUstream_st* stream) {
  if (!checked(h, kConvMagic)) return BCONV_ERR_INVALID_ARG;
  DeviceGuard g(h->L.device);
  if (!g.ok) return BCONV_ERR_CUDA;
  return forward_host(h->L, host_in, host_out, stream);
}

bconv_status_t bconv_get_output_dims(bconv_handle_t h, int32_t* n, int32_t* ho, int32_t* wo, int32_t* c) {
  if (!checked(h, kConvMagic)) return BCONV_ERR_INVALID_ARG;
  if (n) *n = h->L.N;
  if (ho) *ho = h->L.Ho;
  if (wo) *wo = h->L.Wo;
  if (c) *c = h->L.No;
  return BCONV_OK;
}

int32_t bconv_input_feature_channels(bconv_handle_t h) { return checked(h, kConvMagic) ? h->L.Ni : -1; }
int32_t bconv_output_feature_channels(bconv_handle_t h) { return checked(h, kConvMagic) ? h->L.No : -1; }

bconv_status_t bconv_set_algo(bconv_handle_t h, bconv_algo_t algo) {
  if (!checked(h, kConvMagic)) return BCONV_ERR_INVALID_ARG;
  return set_algo(h->L, algo);
}

int32_t bconv_launches_per_forward(bconv_handle_t h) {
  return checked(h, kConvMagic) ? launches_per_forward(h->L) : -1;
}

int32_t bconv_effective_algo(bconv_handle_t h) { return checked(h, kConvMagic) ? effective_algo(h->L) : -1; }

bconv_status_t bconv_sync_status(bconv_handle_t h, struct CUstream_st* stream) {
  if (!checked(h, kConvMagic)) return BCONV_ERR_INVALID_ARG;
  DeviceGuard g(h->L.device);
  return sync_status(h->L, stream);
}

bconv_status_t bconv_profile_begin(bconv_handle_t h, int32_t max_launches) {
  if (!checked(h, kConvMagic)) return BCONV_ERR_INVALID_ARG;
  DeviceGuard g(h->L.device);
  return profile_begin(h->L, max_launches);
}

bconv_status_t bconv_profile_stride(bconv_handle_t h, int32_t every) {
  if (!checked(h, kConvMagic)) return BCONV_ERR_INVALID_ARG;
  return profile_stride(h->L, every);
}

bconv_status_t bconv_profile_end(bconv_handle_t h, float* total_ms, int32_t* launches) {
  if (!checked(h, kConvMagic)) return BCONV_ERR_INVALID_ARG;
  DeviceGuard g(h->L.device);
  return profile_end(h->L, total_ms, launches);
}

bconv_status_t bconv_destroy(bconv_handle_t h) {
  if (!h) return BCONV_OK;
  if (!checked(h, kConvMagic)) return BCONV_ERR_INVALID_ARG;
  destroy(h->L);
  h->magic = 0;
  delete h;
  return BCONV_OK;
}

bconv_status_t bfc_create(const bfc_desc_t* d, const uint32_t* packed_weights, const float* scale,
                          const float* bias, const float* in_scale, const float* in_bias, bconv_type_t type,
                          uint32_t flags, bfc_handle_t* out) {
  if (!out) return BCONV_ERR_INVALID_ARG;
  *out = nullptr;
  if (!d || !packed_weights) return BCONV_ERR_INVALID_ARG;
  if (!valid_type(type) || (flags & ~static_cast<uint32_t>(BCONV_FLAG_USE_BETA_SCALING))) return BCONV_ERR_INVALID_ARG;
  if (d->neuron != BCONV_NEURON_NONE && d->neuron != BCONV_NEURON_RELU) return BCONV_ERR_INVALID_ARG;
  if (d->batch < 0 || d->in_h <= 0 || d->in_w <= 0 || d->in_channels <= 0 || d->out_channels <= 0 ||
      d->groups <= 0)
    return BCONV_ERR_INVALID_ARG;
  if (d->stride_y != 1 || d->stride_x != 1) return BCONV_ERR_INVALID_ARG;
  if (d->groups != 1) return BCONV_ERR_UNSUPPORTED;
  const int64_t k_bits = static_cast<int64_t>(d->in_h) * d->in_w * d->in_channels;
  if (k_bits > (1 << 26) || d->out_channels > (1 << 20)) return BCONV_ERR_UNSUPPORTED;
  bfc_handle_s* h = new (std::nothrow) bfc_handle_s();
  if (!h) return BCONV_ERR_OOM;
  h->magic = kFcMagic;
  Layer& L = h->L;
  L.fc = true;
  L.type = type;
  L.flags = flags;
  L.relu = d->neuron == BCONV_NEURON_RELU;
  L.N = d->batch; L.H = d->in_h; L.W = d->in_w; L.Ni = d->in_channels; L.No = d->out_channels;
  L.kh = d->in_h; L.kw = d->in_w; L.sy = 1; L.sx = 1;
  L.Ho = 1;
  L.Wo = 1;
  const bconv_status_t st = finish_create(L, packed_weights, scale, bias, in_scale, in_bias, d->scale_value);
  if (st == BCONV_OK) keep_host_params(L, packed_weights, scale, bias, in_scale, in_bias, d->scale_value);
  if (st != BCONV_OK) {
    h->magic = 0;
    delete h;
    return st;
  }
  *out = h;
  return BCONV_OK;
}

bconv_status_t bfc_forward(bfc_handle_t h, const float* in, float* out, struct CUstream_st* stream) {
  if (!checked(h, kFcMagic) || (h->L.N > 0 && (!in || !out))) return BCONV_ERR_INVALID_ARG;
  DeviceGuard g(h->L.device);
  if (!g.ok) return BCONV_ERR_CUDA;
  return run_forward(h->L, in, out, stream);
}

bconv_status_t bfc_set_output_terms(bfc_handle_t h, const float* next_in_scale, const float* next_in_bias) {
  if (!checked(h, kFcMagic)) return BCONV_ERR_INVALID_ARG;
  DeviceGuard g(h->L.device);
  if (!g.ok) return BCONV_ERR_CUDA;
  return set_output_terms(h->L, next_in_scale, next_in_bias);
}

bconv_status_t bfc_forward_io(bfc_handle_t h, const bconv_io_t* io, struct CUstream_st* stream) {
  if (!checked(h, kFcMagic)) return BCONV_ERR_INVALID_ARG;
  DeviceGuard g(h->L.device);
  if (!g.ok) return BCONV_ERR_CUDA;
  return forward_io(h->L, io, stream);
}

bconv_status_t bfc_forward_host(bfc_handle_t h, const float* host_in, float* host_out, struct CUstream_st* stream) {
  if (!checked(h, kFcMagic)) return BCONV_ERR_INVALID_ARG;
  DeviceGuard g(h->L.device);
  if (!g.ok) return BCONV_ERR_CUDA;
  return forward_host(h->L, host_in, host_out, stream);
}

int32_t bfc_input_feature_channels(bfc_handle_t h) { return checked(h, kFcMagic) ? h->L.Ni : -1; }
int32_t bfc_output_feature_channels(bfc_handle_t h) { return checked(h, kFcMagic) ? h->L.No : -1; }

bconv_status_t bfc_set_algo(bfc_handle_t h, bconv_algo_t algo) {
  if (!checked(h, kFcMagic)) return BCONV_ERR_INVALID_ARG;
  return set_algo(h->L, algo);
}

int32_t bfc_launches_per_forward(bfc_handle_t h) { return checked(h, kFcMagic) ? launches_per_forward(h->L) : -1; }

int32_t bfc_effective_algo(bfc_handle_t h) { return checked(h, kFcMagic) ? effective_algo(h->L) : -1; }

bconv_status_t bfc_sync_status(bfc_handle_t h, struct CUstream_st* stream) {
  if (!checked(h, kFcMagic)) return BCONV_ERR_INVALID_ARG;
  DeviceGuard g(h->L.device);
  return sync_status(h->L, stream);
}

bconv_status_t bfc_profile_begin(bfc_handle_t h, int32_t max_launches) {
  if (!checked(h, kFcMagic)) return BCONV_ERR_INVALID_ARG;
  DeviceGuard g(h->L.device);
  return profile_begin(h->L, max_launches);
}

bconv_status_t bfc_profile_stride(bfc_handle_t h, int32_t every) {
  if (!checked(h, kFcMagic)) return BCONV_ERR_INVALID_ARG;
  return profile_stride(h->L, every);
}

bconv_status_t bfc_profile_end(bfc_handle_t h, float* total_ms, int32_t* launches) {
  if (!checked(h, kFcMagic)) return BCONV_ERR_INVALID_ARG;
  DeviceGuard g(h->L.device);
  return profile_end(h->L, total_ms, launches);
}

bconv_status_t bfc_destroy(bfc_handle_t h) {
  if (!h) return BCONV_OK;
  if (!checked(h, kFcMagic)) return BCONV_ERR_INVALID_ARG;
  destroy(h->L);
  h->magic = 0;
  delete h;
  return BCONV_OK;
}

const char* bconv_status_string(bconv_status_t s) {
  switch (s) {
    case BCONV_OK: return "ok";
    case BCONV_ERR_INVALID_ARG: return "invalid argument";
    case BCONV_ERR_UNSUPPORTED: return "unsupported configuration";
    case BCONV_ERR_CUDA: return "CUDA error";
    case BCONV_ERR_OOM: return "out of device memory";
    case BCONV_ERR_TIMEOUT: return "a kernel gave up a bounded wait";
    case BCONV_ERR_NO_DEVICE: return "no CUDA device";
  }
  return "unknown status";
}

bconv_status_t bconv_pack_bits(const uint8_t* bits, int64_t rows, int32_t nbits, uint32_t* out) {
  if (!bits || !out || rows < 0 || nbits <= 0) return BCONV_ERR_INVALID_ARG;
  const int nw = words_for(nbits);
  for (int64_t r = 0; r < rows; ++r) {
    const uint8_t* src = bits + r * nbits;
    uint32_t* dst = out + r * nw;
    for (int w = 0; w < nw; ++w) dst[w] = 0u;
    for (int f = 0; f < nbits; ++f)
      if (src[f]) dst[f / kWordBits] |= 1u << (f % kWordBits);
  }
  return BCONV_OK;
}

int32_t bconv_version(void) { return 100; }

bconv_status_t bconv_set_cta_mode(bconv_cta_mode_t mode) {
  if (mode != BCONV_CTA_AUTO && mode != BCONV_CTA_SINGLE && mode != BCONV_CTA_PAIR) return BCONV_ERR_INVALID_ARG;
  bconv::g_cta_mode.store(mode);
  return BCONV_OK;
}

int32_t bconv_cta_mode(bconv_handle_t h) {
  if (!checked(h, kConvMagic)) return -1;
  return h->L.tc_ok ? ((h->L.tc_pair || h->L.halo2) ? BCONV_CTA_PAIR : BCONV_CTA_SINGLE) : 0;
}

int32_t bfc_cta_mode(bfc_handle_t h) {
  if (!checked(h, kFcMagic)) return -1;
  return h->L.tc_ok ? (h->L.tc_pair ? BCONV_CTA_PAIR : BCONV_CTA_SINGLE) : 0;
}

bconv_status_t bconv_set_staging(bconv_staging_t staging) {
  if (staging < BCONV_STAGING_AUTO || staging > BCONV_STAGING_INPUT) return BCONV_ERR_INVALID_ARG;
  g_staging.store(staging);
  return BCONV_OK;
}

int32_t bconv_staging(bconv_handle_t h) {
  if (!checked(h, kConvMagic)) return -1;
  if (!h->L.tc_ok) return 0;
  return h->L.halo ? BCONV_STAGING_ROWS : h->L.tc.f32 ? BCONV_STAGING_INPUT : BCONV_STAGING_PER_TAP;
}

bconv_status_t bconv_set_tc_codes(bconv_tc_codes_t codes) {
  if (codes != BCONV_CODES_AUTO && codes != BCONV_CODES_INT8 && codes != BCONV_CODES_FP4) return BCONV_ERR_INVALID_ARG;
  bconv::g_tc_codes.store(codes);
  return BCONV_OK;
}

namespace {
int32_t tc_codes_of(const bconv::Layer& L) {
  if (!L.tc_ok) return 0;
  return L.tc.kind == 0 ? BCONV_CODES_INT8 : L.tc.kind == 2 ? BCONV_CODES_FP4 : BCONV_CODES_BF16X3;
}
}  // namespace

int32_t bconv_tc_codes(bconv_handle_t h) { return checked(h, kConvMagic) ? tc_codes_of(h->L) : -1; }
int32_t bfc_tc_codes(bfc_handle_t h) { return checked(h, kFcMagic) ? tc_codes_of(h->L) : -1; }

bconv_status_t bconv_check_wait_timeout(double limit_ms) {
  if (!(limit_ms > 0.0) || limit_ms > 1000.0) return BCONV_ERR_INVALID_ARG;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
    cudaGetLastError();
    return BCONV_ERR_NO_DEVICE;
  }
  uint32_t word = 0;
  const cudaError_t e = wait_check(limit_ms, &word);
  if (e != cudaSuccess) return from_cuda(e);
  return (word & kErrTimeout) ? BCONV_ERR_TIMEOUT : BCONV_OK;
}

bconv_status_t bconv_measure_peak(int32_t kind, double* ops_per_s, double* sm_mhz) {
  if (kind < 0 || kind > 7 || !ops_per_s) return BCONV_ERR_INVALID_ARG;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
    cudaGetLastError();
    return BCONV_ERR_NO_DEVICE;
  }
  return from_cuda(probe_peak(kind, ops_per_s, sm_mhz));
}

}  // extern "C"
