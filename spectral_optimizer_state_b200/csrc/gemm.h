// The Newton-Schulz product kernel's launch interface (gemm.cu): the problems one persistent
// launch carries and how it is launched.  Kept apart from the other passes' declarations so
// that the kernel's own sources are gemm.cu, this header and device_utils.cuh.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace muon {

// ------------------------------------------------------------------ GEMM
// The epilogue forms  v = alpha * s_l * acc + beta * cin + (row == col ? diag : 0)
// and writes it as planes through TMA tensor stores (mirrored too if sym).

// Epilogue warps per CTA (each signals a finished tile once).
constexpr int kEpilogueWarps = 8;

// Problems (one per group, iteration and phase) a single launch may carry.
constexpr int kMaxProblems = 30;

struct alignas(64) GemmProblem {
  CUtensorMap tmA;   // A operand [planes][L][M][K], K contiguous, box {64, 128}
  CUtensorMap tmB;   // B operand: K-major [planes][L][N][K] box {64, 256}; MN-major as the
                     // 5-D chunked view {64 n, K, N/64, L, planes} with box {64, 64, 4, 1, 1}
                     // (one load per stage).
  CUtensorMap tmB2;  // K-major B: box {64, 128} for tiles <= 128 wide
  CUtensorMap tmOut;  // output [planes][L][M][N], box {32, 32}, 64-byte swizzle
  int M, N, K, L;
  int nseg;          // 1 (bf16) or 6 (three-plane split)
  int b_mn_major;    // 0: B stored N x K; 1: B stored K x N
  int sym;           // output symmetric: compute upper tiles only, mirror the rest
  int reverse;       // walk the matrices last to first (L2 reuse of the previous phase)
  int tiles_per_matrix;
  int tile_base;     // first global tile index of this problem
  int k_tiles;       // ceil(K / 64)
  int planes;        // planes of out / cin (1 or 3)
  float alpha, beta, diag;
  const float* mat_scale;  // per-matrix factor s_l, or null for 1
  const uint16_t* cin;     // [planes][L][M][cin_pitch], null when beta == 0
  long long cin_plane, cin_mat;
  int cin_pitch;
  // Cross-phase ordering inside one launch.  Every epilogue warp that finishes
  // its share of a tile of matrix l adds 1 to done_self[l] once the tile's
  // stores have landed; a tile of matrix l may load only after
  // done_dep[l] >= dep_target (the previous phase of that matrix finished).
  unsigned* done_self;       // [L], or null
  const unsigned* done_dep;  // [L], or null when the inputs were written by an earlier launch
  unsigned dep_target;
};

struct GemmParams {
  GemmProblem prob[kMaxProblems];
  int nprob;
  int total_tiles;
  int* status;
  // test hook: CTA 0's first epilogue warp does not count its first finished tile, so the
  // tiles that depend on it can only end through their bounded waits (MUON_ERR_TIMEOUT)
  int drop_signal;
};

// 128 x 256 tiles, B operand boxes {64, 128}/{64, 256} (K-major) or {64, 64, 4} (MN-major).
size_t gemm_smem_bytes();
// `ctas`: persistent CTAs to launch (one per SM at most).
cudaError_t launch_gemm(const GemmParams& p, int ctas, cudaStream_t stream);

// Tiles one matrix of this problem shape contributes.
int gemm_tiles_per_matrix(int M, int N, int sym);

}  // namespace muon
