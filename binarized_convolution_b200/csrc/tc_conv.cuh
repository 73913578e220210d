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
  int kb_per_tap;      // 128-byte channel blocks per tap
  int BN;              // output channels per tile (multiple of 32, <= 256)
  int n_tiles;         // ceil(No / BN)
  int m_tiles;         // tiles_y * tiles_x * ceil(N / Bn)
  int tiles_x, tiles_y;
  int R, Cw, Bn;
  int k_splits;        // > 1: partial sums reduced into an fp32 workspace
  int No;
  uint32_t tmem_cols;  // power of two >= 2*BN
  const float* scale;
  const float* bias;
  const float* beta;   // [N][Ho][Wo] or nullptr
  int relu;
  uint32_t* err;
};

int tc_smem_bytes(int bn);
cudaError_t launch_tc_conv(const CUtensorMap* tmA, const CUtensorMap* tmB, const CUtensorMap* tmOut, const TcArgs& a,
                           cudaStream_t s);
cudaError_t launch_tc_finalize(const float* ws, float* out, const float* scale, const float* bias, const float* beta,
                               int64_t total, int no, int rows_per_beta, int relu, cudaStream_t s);

// int8 operand codes: XNOR -> bin(x~) in {-1,+1}, AND -> {0,1}; channels in [ni, cip) are 0.
struct PackI8Args {
  const float* in;        // [npix][ni]
  int64_t npix;
  int ni;
  int cip;                // channels per pixel in the code buffer (multiple of 128)
  const float* in_scale;  // [ni] or nullptr
  const float* in_bias;   // [ni] or nullptr
  int8_t* codes;          // [npix][cip]
  float* A;               // [npix] or nullptr
  int op;                 // kXnor or kAnd
};
cudaError_t launch_pack_i8(const PackI8Args& a, cudaStream_t s);

}  // namespace bconv
