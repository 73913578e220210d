// Declarations of the tensor-core (tcgen05) contraction; internal to the library.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace bconv {

// Geometry and epilogue operands of one tensor-core launch.  An M tile is 128 output pixels
// arranged as Bn images x R rows x Cw columns (R*Cw*Bn = 128); the FC layer is the case
// H = W = 1 with Bn = 128 images per tile.
struct TcArgs {
  int N, Ho, Wo;
  int kh, kw;          // window (1 x 1 for the FC)
  int sy, sx;          // stride (the activation map steps the box by it)
  int kind;            // 0: int8 codes, s32 accumulator; 1: bf16 parts, f32 accumulator
  int kb_per_tap;      // k-blocks per tap (a k-block is 128 bytes of weights per output channel)
  // Where k-block cb of a tap sits in a pixel of the activation map: kb_px k-blocks per pixel,
  // px_bytes bytes per pixel; kind 1 keeps the three bf16 parts of x~ part_bytes apart, and a
  // pipeline stage holds all three parts of one k-block against its single weight block.
  int kb_px;
  int px_bytes;
  int part_bytes;
  int stages;          // pipeline stages in shared memory (as many as fit, at most 4 / 6)
  int BN;              // output channels per tile (multiple of 32, <= 256)
  int n_tiles;         // ceil(No / BN)
  int m_tiles;         // tiles_y * tiles_x * ceil(N / Bn)
  int tiles_x, tiles_y;
  int R, Cw, Bn;
  int mt;              // M sub-tiles per CTA tile sharing each weight stage: 1, or 2 for the FC
                       // (the second sub-tile is the next Bn images; needs R = Cw = 1)
  int k_splits;        // > 1: partial sums reduced into an fp32 workspace
  // Work list: tiles [0, full_tiles) whole, then the remaining tail tiles cut along N into
  // `pieces` parts of BN / pieces channels each (so the last wave spreads over more SMs).
  int full_tiles;
  int pieces;
  int grid_ctas;       // CTAs launched (pair kernel: 2 x co-resident clusters)
  int No;
  uint32_t tmem_cols;  // power of two >= 2*BN
  const float* scale;
  const float* bias;
  const float* beta;   // [N][Ho][Wo] or nullptr (ignored when A is given)
  const float* A;      // [N][H][W] channel means: beta is then formed in the epilogue
  int H, W;            // input extent (for the window of A)
  int relu;
  uint32_t* err;
  // Bit-packed output for a following binary layer (out_bits == nullptr: fp32 through the
  // output tensor map).  Per output pixel p and channel c, x~ = next_scale[c] * y + next_bias[c]
  // gives bit c % 32 of out_bits[p * nwo + c / 32] (1 for x~ >= 0) and out_a[p] = mean_c |x~|.
  // When a pixel's channels span several work items, each item leaves its partial sum of
  // |x~| in a_part[slice][p] and the last of them to finish (counted in a_count[m tile])
  // adds the slices in slice order, so the result does not depend on timing.
  uint32_t* out_bits;
  float* out_a;
  const float* next_scale;  // [No]
  const float* next_bias;   // [No]
  int nwo;                  // ceil(No / 32)
  float* a_part;            // [n_tiles * pieces][N * Ho * Wo]
  uint32_t* a_count;        // [m_tiles], zero between launches
  // Balanced split of the reduction (SM-pair kernel; sk != 0): the work list's items x
  // k-blocks are cut into equal contiguous shares, one per pair.  An item cut between pairs
  // p and p+1 is finished by p (which computes its first k-blocks, last in its share); p+1
  // computes the rest first and leaves its raw partial sums in sk_part[p][rank] with
  // sk_flag[p][rank] = 1, which p adds (int32 exactly, fp32 in a fixed order) and resets.
  // The one-SM fp32-input kernel does the same per CTA (sk_part[c], sk_flag[c] for the tile cut
  // between CTAs c and c + 1) when the tiles outnumber the CTAs.
  int sk;
  uint32_t* sk_part;        // pairs: [pairs - 1][2][BN / 32][32][128]; one SM: [CTAs - 1][BN / 32][32][128] words
  uint32_t* sk_flag;        // pairs: [pairs - 1][2]; one SM: [CTAs - 1]; zero between launches
  // binaryWeights straight from the fp32 input (f32 != 0; one SM per tile, BN <= 128, no beta):
  // tmA is then a map over the input x [N][H][W][Ni] fp32 (boxes of 32 channels x Cw x R x Bn
  // pixels with the convolution's strides as element strides, 128-byte swizzle), and
  // converting warps form x~ = fma(x, in_scale, in_bias) -- zero for out-of-image taps and
  // channels >= Ni -- and its exact three bf16 parts in shared memory, so no parts buffer is
  // written or read.
  int f32;
  const float* in_scale;  // [Ni] or nullptr
  const float* in_bias;
  int Ni;
  // Weights for the one-SM kernel: [n_tiles][kh * kw * kb_per_tap][BN][128] bytes, one
  // contiguous block per (N tile, k-block) already in the shared-memory order of the 128-byte
  // swizzle (16-byte chunk c of row r stored at chunk c ^ (r % 8)), so that each stage is one
  // bulk copy.  The pair kernel reads row-major weights through tensor maps instead.
  const int8_t* b_tiles;
};

// Convolution with the activation rows held in shared memory (stride 1, e2m1 codes, fp32 output):
// codes (and A) in a zero-bordered [N][Hp][Wp] grid (Hp = H + kh - 1, Wp = W + kw - 1), outputs
// enumerated over the same grid, a tile = 128 consecutive slots, one halo load per k-block
// serving every tap.
struct HaloArgs {
  int N, H, W, Hp, Wp;
  int kh, kw;
  int kb_per_tap;      // 128-byte k-blocks per pixel
  int BN, n_tiles, No;
  // filled by tc_halo_plan
  int m_tiles;         // ceil(N * Hp * Wp / 128)
  int halo_len;        // rows a tile's MMAs read: 128 + (kh - 1) * Wp + kw - 1
  int halo_rows;       // rows per halo box (<= 256)
  int halo_boxes;      // boxes per halo
  int halo_bytes;      // shared memory per halo stage (a 1024-byte multiple)
  int resident;        // the weights of the CTA's N tile stay in shared memory
  int wstages;         // weight ring stages otherwise
  int grid_ctas;       // a multiple of n_tiles
  uint32_t tmem_cols;
  const float* scale;
  const float* bias;
  const float* A;      // [N][Hp][Wp] channel means in the zero-bordered grid, or nullptr
  int relu;
  uint32_t* err;
  const int8_t* b_tiles;  // [n_tiles][kh * kw * kb_per_tap][BN][128] bytes, pre-swizzled
  float* out;             // [N][H][W][No] fp32, 16-byte aligned
};
bool tc_halo_plan(HaloArgs& a, int sm_count);  // false: the shape does not fit this kernel
int tc_halo_smem_bytes(const HaloArgs& a);
// tmA: 2-D map over the padded codes [N*Hp*Wp][bytes per pixel], box 128 bytes x halo_rows,
// 128-byte swizzle.
cudaError_t launch_tc_halo(const CUtensorMap* tmA, const HaloArgs& a, cudaStream_t s);

// The same on SM pairs (tc_halo2_kernel): M = 256 over two CTAs, N = 256 channels per pair,
// each CTA holding half of the weight tile.  Weights row-major [n_tiles * 256][kh * kw *
// kb_per_tap * 128] bytes, read through tmB (box 128 bytes x 128 rows, 128-byte swizzle).
// max_pairs <= 0: the co-resident two-CTA clusters of the current device.
bool tc_halo2_plan(HaloArgs& a, int max_pairs);
int tc_halo2_max_pairs(const HaloArgs& a);
cudaError_t launch_tc_halo2(const CUtensorMap* tmA, const CUtensorMap* tmB, const HaloArgs& a, cudaStream_t s);

// Fully-connected layer on e2m1 codes: activations [N][K / 2] bytes, weights
// [n_tiles * 256][K / 2] bytes (K = the flattened image's padded channels; a k-block = 256 codes
// = 128 bytes); items of 128 images x 256 channels x a share of the k-blocks, one per CTA, the
// k_splits items of a tile forming one cluster that adds its partial sums through distributed
// shared memory.
struct FcArgs {
  int N, No;
  int hw;             // pixels per image (the window of beta)
  int kb_total;       // k-blocks of the flattened image
  // filled by tc_fc_plan
  int m_tiles, n_tiles, k_splits, kb_per_split;  // k_splits: 1, 2, 4 or 8; kb_per_split <= 127
  const float* scale;
  const float* bias;
  const float* A;     // [N][hw] channel means, or nullptr (no beta)
  int relu;
  uint32_t* err;
  float* out;         // [N][No] output, 16-byte aligned
  // weight codes as contiguous blocks [n_tiles][kb_total][256 rows][128 bytes], each already in
  // the shared-memory order of the 128-byte swizzle (16-byte chunk c of row r at c ^ (r % 8)):
  // one 32 KB bulk copy per stage
  const uint8_t* b_blocks;
};
// false: the shape does not fit this kernel (more than 127 k-blocks per split even with 8
// splits, whose int16 partial sums would overflow, or no cluster fits the device)
bool tc_fc_plan(FcArgs& a, int sm_count);
int tc_fc_smem_bytes();
// tmA: 2-D map over the activation codes {K / 2 bytes, N}, box 128 x 128, 128-byte swizzled;
// the weights come from a.b_blocks.
cudaError_t launch_tc_fc(const CUtensorMap* tmA, const FcArgs& a, cudaStream_t s);


int tc_stages(int kind, int bn, int mt);  // stages that fit; < 2: the layout does not fit
int tc_f32_stages(int bn);                // binaryWeights from fp32 input: part stages, 0 if it does not fit
int tc_smem_bytes(const TcArgs& a);
// One CTA per tile; weights from a.b_tiles.
cudaError_t launch_tc_conv(const CUtensorMap* tmA, const CUtensorMap* tmOut, const TcArgs& a, cudaStream_t s);
// Grid size and tail split for a launch on `sm_count` SMs (fills full_tiles / pieces).
int tc_plan(TcArgs& a, int sm_count);

// SM-pair kernel (tcgen05.mma.cta_group::2, M = 256 per cluster of two CTAs); convolutions only.
// tmB / tmBp are weight maps with boxes of BN/2 and BN/pieces/2 rows.
int tc2_stages(int kind, int bn);
int tc2_smem_bytes(int kind, int bn, int stages);
int tc2_plan(TcArgs& a, int pairs);      // pairs = clusters that can be resident at once
int tc2_max_pairs(int kind, int bn);     // co-resident two-CTA clusters on the current device (0: none)
cudaError_t launch_tc_conv2(const CUtensorMap* tmA, const CUtensorMap* tmB, const CUtensorMap* tmBp,
                            const CUtensorMap* tmOut, const TcArgs& a, cudaStream_t s);
// The epilogue of a split reduction: y from the fp32 workspace [rows][no] (zeroed as it is
// read), with beta = mean of A [rows][hw] over each image when A is given.  ws and out are
// 16-byte aligned, no % 4 == 0 (the tensor-core path's condition).
cudaError_t launch_tc_finalize(float* ws, float* out, const float* scale, const float* bias, const float* A, int hw,
                               int rows, int no, int relu, cudaStream_t s);

// int8 operand codes: XNOR -> bin(x~) in {-1,+1}, AND -> {0,1}; channels in [ni, cip) are 0.
// With f4 the codes are e2m1 (fp4) values, two per byte (channel 2j in the low nibble):
// +1.0 = 0x2, -1.0 = 0xA (XNOR) or 0 (AND), padding 0; the code buffer then holds cip / 2
// bytes per pixel and cip is a multiple of 256.
struct PackI8Args {
  const float* in;        // [npix][ni]
  int64_t npix;
  int ni;
  int cip;                // channels per pixel in the code buffer (multiple of 128)
  const float* in_scale;  // [ni] or nullptr
  const float* in_bias;   // [ni] or nullptr
  int8_t* codes;          // [npix][cip] (f4: [npix][cip / 2] bytes)
  float* A;               // [npix] or nullptr
  int op;                 // kXnor or kAnd
  int f4;
  // Destination grid: pixel (n, y, x) of the [N][h][w] input goes to code pixel
  // (n, y + pad_t, x + pad_l) of an [N][hp][wp] buffer whose other pixels are left alone
  // (hp == 0: the codes have the input's own [N][h][w] layout).
  PadMap pad;
  uint32_t* err;          // error word for a wait that timed out (the staged e2m1 kernel), or nullptr
};
cudaError_t launch_pack_i8(const PackI8Args& a, cudaStream_t s);

// binaryWeights operand for the tensor cores: x~ split exactly into three bf16 parts,
// x~ = hi + mid + lo (each the leading 8 significant bits of what the previous parts leave;
// every difference is exact in fp32), stored per pixel as [part][cip] bf16; channels in
// [ni, cip) are 0.
struct PackBf16x3Args {
  const float* in;        // [npix][ni]
  int64_t npix;
  int ni;
  int cip;                // channels per part (multiple of 64)
  const float* in_scale;  // [ni] or nullptr
  const float* in_bias;   // [ni] or nullptr
  uint16_t* parts;        // [npix][3][cip] bf16 bits
  float* A;               // [npix] or nullptr
};
cudaError_t launch_pack_bf16x3(const PackBf16x3Args& a, cudaStream_t s);

}  // namespace bconv
