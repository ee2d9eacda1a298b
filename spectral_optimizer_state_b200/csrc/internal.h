// Structures shared by the host side of libmuon and its kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/muon.h"
#include "gemm.h"

namespace muon {

// ------------------------------------------------------------------ K1
// Momentum + Nesterov + Frobenius norm, writes X0 (un-normalised U) in the
// wide orientation into the workspace as PLANES bf16 planes.  One launch
// covers several same-dtype groups: the launch's blocks are cut into
// consecutive ranges, one per group, `nblk` blocks per matrix.
struct MomentumGroup {
  int mat0;                       // first matrix of the group in the launch's pointer tables
  int batch, rows, cols;          // of G / M (row-major)
  int nblk;                       // blocks per matrix
  int block0;                     // first block of the group in the launch
  int vec;                        // 16-byte vector path (cols % 8 == 0, aligned pointers)
  int pitch;                      // wide row pitch of x (elements), multiple of 8
  uint16_t* x;                    // [planes][batch][mrows][pitch] bf16 bits
  long long x_plane, x_mat;       // elements between planes / matrices
  float* partials;                // [batch][nblk]
  unsigned int* counters;         // [batch], zero between calls
  float* nu;                      // [batch] ||U||_F
  float* scale1;                  // [batch] 1/(nu+eps)
  float* scale2;                  // [batch] scale1^2
  int* flags;                     // [batch]
};

struct MomentumParams {
  const void* g[MUON_MAX_BATCH];  // rows x cols, bf16 or fp32 (launch-wide index)
  float* m[MUON_MAX_BATCH];       // rows x cols fp32 (null when no momentum)
  MomentumGroup grp[MUON_MAX_GROUPS];
  int ngroups;
  float beta;
  float gscale;                   // G is read as gscale * G
  int nesterov;
  float eps;
};

// One launch over p.ngroups groups (at most MUON_MAX_BATCH matrices in all);
// the caller fills every field but block0 / vec, which this sets.
cudaError_t launch_momentum(MomentumParams& p, bool g_is_f32, bool momentum, int planes, cudaStream_t stream);

// Number of blocks per matrix K1 uses for a rows x cols matrix.
int momentum_blocks_per_matrix(int rows, int cols);

// ------------------------------------------------------------------ K5 apply
struct ApplyGroup {
  int mat0, batch, rows, cols, nblk, block0, vec;
  int cvec;                 // the cap's v vectors are 16-byte aligned (read 8 at a time)
  const uint16_t* o;        // final iterate [planes][batch][m][pitch] bf16 bits (wide)
  long long o_plane, o_mat; // elements
  int pitch;
  float lrs;                // lr * s(rows, cols)
  const int* flags;         // [batch] matrices with a nonzero flag are left unchanged (null: none)
  const float* alpha;       // spectral cap coefficients [batch] (null: none)
};

struct ApplyParams {
  void* w[MUON_MAX_BATCH];  // caller matrices rows x cols (W, or Out), launch-wide index
  // spectral cap: O is replaced by O - alpha_l u_l v_l^T, u_l of length rows and
  // v_l of length cols of W (used by groups whose alpha is set)
  const float* cu[MUON_MAX_BATCH];
  const float* cv[MUON_MAX_BATCH];
  ApplyGroup grp[MUON_MAX_GROUPS];
  int ngroups;
  int planes;
  int apply;                // 1: W <- decay*W - lrs*O ; 0: W <- O
  float decay;
  const int* status;        // device status word: nothing is written after a timeout (null: none)
};

// One launch over p.ngroups groups of one W dtype; sets block0 / vec.
cudaError_t launch_apply(ApplyParams& p, bool w_f32, cudaStream_t stream);

// ------------------------------------------------------------------ spectral
struct GemvParams {
  const void* w[MUON_MAX_BATCH];   // rows x cols, bf16 or fp32
  const float* x[MUON_MAX_BATCH];  // input: length cols (rows GEMV) or rows (cols GEMV)
  float* y[MUON_MAX_BATCH];        // output: length rows (rows GEMV) or cols (cols GEMV)
  int rows, cols;
  float* partial;                  // cols GEMV: [batch][row_chunks][cols]
  int row_chunks, rows_per_chunk;
};

struct CapParams {
  const float* a[MUON_MAX_BATCH];  // length m (wide rows)
  const float* b[MUON_MAX_BATCH];  // length n (wide columns)
  const uint16_t* o;               // final iterate, wide, [planes][batch][m][pitch]
  long long o_plane, o_mat;
  int pitch, m, n, planes;
  double* partial;                 // [batch][ceil(m / 32)]: one per block of 32 rows
};
// Blocks of the cap coefficient pass per matrix (32 rows each).
inline int cap_alpha_blocks(int m) { return (m + 31) / 32; }

// `iters` power iterations, one pass over W each (u <- W v / |W v|, v <- W^T u / |W^T u|,
// sigma = |W^T u|), in one cooperative launch when the blocks fit on the GPU at once, else one
// launch per iteration: p.x = v (read, then overwritten), p.y = u; p.partial
// 2 x [batch][nblk][cols] (two iterations' partials), tsq_partial [batch][nblk] and
// counters [2 * batch] scratch (zeroed here).  nblk from power_pass_blocks; cols % 8 == 0,
// 16-byte aligned W, cols <= power_pass_max_cols().  Wait timeouts set `status`.
// With `shift` ([batch] sigma_max, device) the passes run the shifted iteration for the smallest
// singular value of a tall W instead (iters = shifted steps + 1; p.x = y, read then overwritten;
// p.y scratch of `rows` floats; sigma receives |W y|); it needs every pass in one launch
// (power_pass_together, or iters == 1).
int power_pass_max_cols();
int power_pass_blocks(int rows, int cols, int batch, bool f32, int sm_count);
bool power_pass_together(int cols, bool f32, int nblk, int batch, int sm_count);
cudaError_t launch_power_iteration_stream(GemvParams& p, int batch, bool f32, int nblk, int iters,
                                          float* tsq_partial, unsigned* counters, float* sigma, int* status,
                                          int sm_count, cudaStream_t s, const float* shift = nullptr);
// Smallest singular value of a wide W (rows <= cols, X = W) by `iters` shifted steps, one pass
// over W each plus a last one (colslab_kernel, one cooperative launch): slabs of S columns.
// colslab_width gives S (0: this path does not apply: rows > 4096, cols not a multiple of 64,
// or the grid does not fit on the GPU at once).  p.x = y (read, then overwritten), p.partial
// 2 x [batch][cols / S][rows], dsq [batch][cols / S], counters [2 * batch] scratch.
int colslab_width(int rows, int cols, int batch, bool f32, int sm_count);
cudaError_t launch_min_singular_slabs(GemvParams& p, int batch, bool f32, int S, int iters, const float* shift,
                                      float* dsq, unsigned* counters, float* sigma, int* status, cudaStream_t s);
cudaError_t launch_gemv_rows(const GemvParams& p, int batch, bool f32, cudaStream_t s);
cudaError_t launch_gemv_cols(const GemvParams& p, int batch, bool f32, cudaStream_t s);
cudaError_t launch_normalize(float* const* vecs_dev, int batch, int n, float* norm, cudaStream_t s);
cudaError_t launch_cap_alpha(const CapParams& p, int batch, float* alpha, cudaStream_t s);
cudaError_t launch_shift_normalize(float* const* y, const float* const* z, int batch, int n, const float* sigma_max,
                                   cudaStream_t s);

}  // namespace muon
