// Spectral diagnostics and the spectral cap.
//
// * Top singular triplet of each W by power iteration:
//     u = W v / |W v| ;  v = W^T u / |W^T u| ;  sigma = |W^T u|
//   (Muon Meets Mamba: Spectral Optimization for State Space Models, abstract:
//   Muon lowers the condition number of the projection it trains; the top
//   singular value is the quantity to watch.)
// * Cap coefficient alpha = u^T O v of the orthogonalised update O, so the
//   apply can use O - alpha u v^T (An Isotropy-Preserving Spectral Cap for
//   Muon: the update loses the direction that grows the top eigenvalue).
//
// All passes are memory-bound matrix-vector products over a batch of
// same-shape matrices.  Every reduction has a fixed order (per-row warp
// trees; per-row-chunk partials summed by a second pass), so results are
// deterministic.
#include <cuda_bf16.h>

#include <algorithm>

#include "device_utils.cuh"
#include "internal.h"

namespace muon {

namespace {

constexpr int kThreads = 256;

template <bool F32>
__device__ __forceinline__ void load8(const void* base, long long e, float (&x)[8]) {
  if (F32) {
    const float4* q = reinterpret_cast<const float4*>(static_cast<const float*>(base) + e);
    const float4 a = q[0], b = q[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  } else {
    const uint4 q = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + e);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

template <bool F32>
__device__ __forceinline__ float load1(const void* base, long long e) {
  return F32 ? static_cast<const float*>(base)[e] : bf16_bits_to_float(static_cast<const uint16_t*>(base)[e]);
}

// y[r] = sum_c W[r][c] x[c]; each warp takes rows_per_warp consecutive rows, x staged in shared memory
// once per block.
template <bool F32, bool VEC>
__global__ void __launch_bounds__(kThreads) gemv_rows_kernel(const __grid_constant__ GemvParams p, int rows_per_warp) {
  extern __shared__ float xs[];
  const int l = blockIdx.y;
  const float* x = p.x[l];
  for (int c = threadIdx.x; c < p.cols; c += kThreads) xs[c] = x[c];
  __syncthreads();
  const void* W = p.w[l];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = (blockIdx.x * (kThreads / 32) + warp) * rows_per_warp;
  const int r1 = min(p.rows, r0 + rows_per_warp);
  for (int r = r0; r < r1; ++r) {
    const long long row = static_cast<long long>(r) * p.cols;
    float acc = 0.f;
    if (VEC) {
#pragma unroll 2
      for (int c = lane * 8; c < p.cols; c += 32 * 8) {
        float w[8];
        load8<F32>(W, row + c, w);
#pragma unroll
        for (int t = 0; t < 8; ++t) acc = fmaf(w[t], xs[c + t], acc);
      }
    } else {
      for (int c = lane; c < p.cols; c += 32) acc = fmaf(load1<F32>(W, row + c), xs[c], acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) p.y[l][r] = acc;
  }
}

// partial[l][chunk][c] = sum over the chunk's rows of W[r][c] y[r]; thread owns 8 columns (VEC) or 1.
template <bool F32, bool VEC>
__global__ void __launch_bounds__(kThreads) gemv_cols_partial_kernel(const __grid_constant__ GemvParams p) {
  const int l = blockIdx.z;
  const void* W = p.w[l];
  const float* y = p.x[l];
  const int per = VEC ? 8 : 1;
  const int c0 = (blockIdx.x * blockDim.x + threadIdx.x) * per;
  if (c0 >= p.cols) return;
  const int r0 = blockIdx.y * p.rows_per_chunk;
  const int r1 = min(p.rows, r0 + p.rows_per_chunk);
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll 4
  for (int r = r0; r < r1; ++r) {
    const float yr = y[r];
    const long long e = static_cast<long long>(r) * p.cols + c0;
    if (VEC) {
      float w[8];
      load8<F32>(W, e, w);
#pragma unroll
      for (int t = 0; t < 8; ++t) acc[t] = fmaf(w[t], yr, acc[t]);
    } else {
      acc[0] = fmaf(load1<F32>(W, e), yr, acc[0]);
    }
  }
  float* out = p.partial + (static_cast<long long>(l) * p.row_chunks + blockIdx.y) * p.cols + c0;
  if (VEC) {
#pragma unroll
    for (int t = 0; t < 8; ++t) out[t] = acc[t];
  } else {
    out[0] = acc[0];
  }
}

// y[l][c] = sum_k partial[l][k][c] in chunk order.
__global__ void __launch_bounds__(kThreads) gemv_cols_reduce_kernel(const __grid_constant__ GemvParams p) {
  const int l = blockIdx.y;
  const int c = blockIdx.x * kThreads + threadIdx.x;
  if (c >= p.cols) return;
  const float* part = p.partial + static_cast<long long>(l) * p.row_chunks * p.cols + c;
  float s = 0.f;
  for (int k = 0; k < p.row_chunks; ++k) s += part[static_cast<long long>(k) * p.cols];
  p.y[l][c] = s;
}

// Sum of n partial sums, by one warp: lane k adds partials k, k + 32, ... in order, then a fixed
// xor-shuffle tree combines the lanes (the same order on every call); every lane gets the total.
__device__ __forceinline__ double warp_sum_partials(const float* part, int n, int lane) {
  double a = 0.0;
  for (int k = lane; k < n; k += 32) a += static_cast<double>(part[k]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
  return a;
}

// 8 consecutive elements of W as packed 16-byte vectors (bf16: one, fp32: two) and their values.
template <bool F32>
struct Raw8w {
  uint4 q[F32 ? 2 : 1];
};

template <bool F32>
__device__ __forceinline__ void load_raw(const void* base, long long e, Raw8w<F32>& r) {
  const uint4* p = F32 ? reinterpret_cast<const uint4*>(static_cast<const float*>(base) + e)
                       : reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + e);
#pragma unroll
  for (int i = 0; i < (F32 ? 2 : 1); ++i) r.q[i] = p[i];
}

template <bool F32>
__device__ __forceinline__ void unpack_raw(const Raw8w<F32>& r, float (&x)[8]) {
  if (F32) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      x[4 * i] = __uint_as_float(r.q[i].x);
      x[4 * i + 1] = __uint_as_float(r.q[i].y);
      x[4 * i + 2] = __uint_as_float(r.q[i].z);
      x[4 * i + 3] = __uint_as_float(r.q[i].w);
    }
  } else {
    const uint32_t w[4] = {r.q[0].x, r.q[0].y, r.q[0].z, r.q[0].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

// t_r = W[r, :] . v and z += t_r W[r, :] for one row held (packed) in registers.
template <bool F32, int NV>
__device__ __forceinline__ float power_row(const Raw8w<F32> (&w)[NV], const float* vs, int C, int lane,
                                           float (&z)[NV][8]) {
  float dot = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = 8 * lane + 256 * i;
    if (c < C) {
      float x[8];
      unpack_raw<F32>(w[i], x);
      // 16-byte reads of v: a lane's 8 values are contiguous, so scalar reads would be 8-way
      // bank conflicts across the warp
      const float4 va = *reinterpret_cast<const float4*>(vs + c);
      const float4 vb = *reinterpret_cast<const float4*>(vs + c + 4);
      const float vv[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
#pragma unroll
      for (int t = 0; t < 8; ++t) dot = fmaf(x[t], vv[t], dot);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = 8 * lane + 256 * i;
    if (c < C) {
      float x[8];
      unpack_raw<F32>(w[i], x);
#pragma unroll
      for (int t = 0; t < 8; ++t) z[i][t] = fmaf(dot, x[t], z[i][t]);
    }
  }
  return dot;
}

// One pass over the rows of W for a whole power iteration.  With t = W v, the
// next iterate's W^T u is W^T t / |t|, and W^T t = sum_r t_r W[r, :]: each warp
// loads its rows once (two rows in flight, NV packed 16-byte vectors per lane
// each), forms t_r against v (staged in shared memory) and adds t_r W[r, :] to its
// running sum z.  t goes to u (un-normalised), a fixed-order tree over the warps
// gives one partial z per block, and each block writes its partial sum of t_r^2.
// Requires cols % 8 == 0, 16-byte aligned rows and cols <= 256 * NV.
//
// v is read as v / |v| when zsq_prev is set (the un-normalised W^T t of the previous
// iteration, whose squared norm is the sum of zsq_prev's zblk partials); the first
// iteration takes the caller's vector as it is (u and the next v do not depend on its scale).
template <bool F32, int NV>
__global__ void __launch_bounds__(kThreads) power_pass_kernel(const __grid_constant__ GemvParams p,
                                                              int rows_per_block, float* tsq_partial,
                                                              const float* zsq_prev, int zblk) {
  extern __shared__ float sm[];
  float* vs = sm;                         // [cols]
  float* zs = sm + p.cols;                // [warps][cols]
  constexpr int kWarps = kThreads / 32;
  __shared__ float s_inv;
  const int l = blockIdx.y;
  const float* x = p.x[l];
  const int C = p.cols;
  if (threadIdx.x < 32) {
    float inv = 1.0f;
    if (zsq_prev != nullptr) {
      const float nz = static_cast<float>(sqrt(warp_sum_partials(zsq_prev + static_cast<long long>(l) * zblk, zblk,
                                                                 threadIdx.x)));
      inv = nz > 0.f ? 1.0f / nz : 0.f;
    }
    if (threadIdx.x == 0) s_inv = inv;
  }
  __syncthreads();
  const float inv = s_inv;
  for (int c = threadIdx.x; c < C; c += kThreads) vs[c] = x[c] * inv;
  __syncthreads();
  const void* W = p.w[l];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r_beg = blockIdx.x * rows_per_block;
  const int r_end = min(p.rows, r_beg + rows_per_block);
  float z[NV][8];
#pragma unroll
  for (int i = 0; i < NV; ++i)
#pragma unroll
    for (int t = 0; t < 8; ++t) z[i][t] = 0.f;
  float tsq = 0.f;
  for (int r0 = r_beg + warp; r0 < r_end; r0 += 2 * kWarps) {
    const int r1 = r0 + kWarps;
    const bool two = r1 < r_end;
    Raw8w<F32> w0[NV], w1[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int c = 8 * lane + 256 * i;
      if (c < C) {
        load_raw<F32>(W, static_cast<long long>(r0) * C + c, w0[i]);
        if (two) load_raw<F32>(W, static_cast<long long>(r1) * C + c, w1[i]);
      }
    }
    const float t0 = power_row<F32, NV>(w0, vs, C, lane, z);
    if (lane == 0) p.y[l][r0] = t0;
    tsq = fmaf(t0, t0, tsq);
    if (two) {
      const float t1 = power_row<F32, NV>(w1, vs, C, lane, z);
      if (lane == 0) p.y[l][r1] = t1;
      tsq = fmaf(t1, t1, tsq);
    }
  }
  // warps' z into shared memory, then a fixed-order sum over the warps
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = 8 * lane + 256 * i;
    if (c < C) {
      float4* d = reinterpret_cast<float4*>(zs + warp * C + c);
      d[0] = make_float4(z[i][0], z[i][1], z[i][2], z[i][3]);
      d[1] = make_float4(z[i][4], z[i][5], z[i][6], z[i][7]);
    }
  }
  __syncthreads();
  float* out = p.partial + (static_cast<long long>(l) * gridDim.x + blockIdx.x) * C;
  for (int c = threadIdx.x; c < C; c += kThreads) {
    float a = 0.f;
#pragma unroll
    for (int k = 0; k < kWarps; ++k) a += zs[k * C + c];
    out[c] = a;
  }
  // the warps' sums of t_r^2 (every lane holds its warp's), in warp order
  __shared__ float tq[kWarps];
  if (lane == 0) tq[warp] = tsq;
  __syncthreads();
  if (threadIdx.x == 0) {
    float a = 0.f;
#pragma unroll
    for (int k = 0; k < kWarps; ++k) a += tq[k];
    tsq_partial[static_cast<long long>(l) * gridDim.x + blockIdx.x] = a;
  }
}

template <typename T>
__device__ __forceinline__ T block_sum(T v, T* scratch) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  T r = 0;
  if (warp == 0) {
    r = lane < (kThreads / 32) ? scratch[lane] : T(0);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
  }
  return r;
}

// z = the pass's block partials summed in block order (one thread per column, the loads
// eight blocks ahead of the additions); z goes to v un-normalised and each block writes
// its partial sum of z^2.  grid (column blocks, batch).
__global__ void __launch_bounds__(kThreads) power_reduce_kernel(const __grid_constant__ GemvParams p, int nblk,
                                                                float* zsq_partial) {
  __shared__ double scratch[kThreads / 32];
  const int l = blockIdx.y;
  const int C = p.cols;
  const int c = blockIdx.x * kThreads + threadIdx.x;
  double zz = 0.0;
  if (c < C) {
    const float* part = p.partial + static_cast<long long>(l) * nblk * C + c;
    float a = 0.f;
    int b = 0;
    for (; b + 8 <= nblk; b += 8) {
      float q[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) q[k] = part[static_cast<long long>(b + k) * C];
#pragma unroll
      for (int k = 0; k < 8; ++k) a += q[k];
    }
    for (; b < nblk; ++b) a += part[static_cast<long long>(b) * C];
    const_cast<float*>(p.x[l])[c] = a;
    zz = static_cast<double>(a) * a;
  }
  const double tot = block_sum<double>(zz, scratch);
  if (threadIdx.x == 0) zsq_partial[static_cast<long long>(l) * gridDim.x + blockIdx.x] = static_cast<float>(tot);
}

// u = t / |t|, v = z / |z|, sigma = |z| / |t| (= |W^T u|), from the partial sums of t^2 and z^2
// (summed in order by every block).  A zero t leaves u, v at zero and sigma 0.
// grid (element blocks over max(rows, cols), batch).
__global__ void __launch_bounds__(kThreads) power_scale_kernel(const __grid_constant__ GemvParams p, int nblk,
                                                               const float* tsq_partial, int zblk,
                                                               const float* zsq_partial, float* sigma) {
  __shared__ float s_inv_t, s_inv_z;
  const int l = blockIdx.y;
  if (threadIdx.x < 32) {
    const double tt = warp_sum_partials(tsq_partial + static_cast<long long>(l) * nblk, nblk, threadIdx.x);
    const double zz = warp_sum_partials(zsq_partial + static_cast<long long>(l) * zblk, zblk, threadIdx.x);
    if (threadIdx.x == 0) {
      const float nt = static_cast<float>(sqrt(tt));
      const float nz = static_cast<float>(sqrt(zz));
      s_inv_t = nt > 0.f ? 1.0f / nt : 0.f;
      s_inv_z = nz > 0.f ? 1.0f / nz : 0.f;
      if (blockIdx.x == 0) sigma[l] = nt > 0.f ? nz / nt : 0.f;
    }
  }
  __syncthreads();
  const int i = blockIdx.x * kThreads + threadIdx.x;
  if (i < p.cols) const_cast<float*>(p.x[l])[i] *= s_inv_z;
  if (i < p.rows) p.y[l][i] *= s_inv_t;
}

struct VecParams {
  float* v[MUON_MAX_BATCH];
  int n;
  float* norm;
};

// v <- v / |v| per matrix; |v| into norm[l] (0 leaves v at zero).
__global__ void __launch_bounds__(kThreads) normalize_kernel(const __grid_constant__ VecParams p) {
  __shared__ double scratch[kThreads / 32];
  __shared__ float inv;
  float* v = p.v[blockIdx.x];
  const int n = p.n;
  float* norm = p.norm;
  double ss = 0.0;
  for (int i = threadIdx.x; i < n; i += kThreads) ss += static_cast<double>(v[i]) * v[i];
  const double tot = block_sum<double>(ss, scratch);
  if (threadIdx.x == 0) {
    const float nrm = static_cast<float>(sqrt(tot));
    if (norm) norm[blockIdx.x] = nrm;
    inv = nrm > 0.f ? 1.0f / nrm : 0.f;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += kThreads) v[i] *= inv;
}

struct ShiftParams {
  float* y[MUON_MAX_BATCH];
  const float* z[MUON_MAX_BATCH];
  const float* sigma_max;  // [batch]: the shift is sigma_max^2
  int n;
};

// y <- (s y - z) / |s y - z| per matrix (left as is when that is zero).
__global__ void __launch_bounds__(kThreads) shift_normalize_kernel(const __grid_constant__ ShiftParams p) {
  __shared__ double scratch[kThreads / 32];
  __shared__ float inv;
  const int l = blockIdx.x;
  float* y = p.y[l];
  const float* z = p.z[l];
  const float sm = p.sigma_max[l];
  const float s = sm * sm;
  double ss = 0.0;
  for (int i = threadIdx.x; i < p.n; i += kThreads) {
    const float t = fmaf(s, y[i], -z[i]);
    y[i] = t;
    ss += static_cast<double>(t) * t;
  }
  const double tot = block_sum<double>(ss, scratch);
  if (threadIdx.x == 0) {
    const float nrm = static_cast<float>(sqrt(tot));
    inv = nrm > 0.f ? 1.0f / nrm : 0.f;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < p.n; i += kThreads) y[i] *= inv;
}

// alpha partials: wide O (m x n, planes summed) against a (length m) and b (length n).
// One warp per row of O (rows_per_block == warps per block); each lane reads
// 16-byte vectors of every plane (the wide pitch is a multiple of 64 elements,
// so row starts are 128-byte aligned) and the ragged tail element by element.
__global__ void __launch_bounds__(kThreads) cap_alpha_partial_kernel(const __grid_constant__ CapParams p) {
  __shared__ double scratch[kThreads / 32];
  const int l = blockIdx.y;
  const float* a = p.a[l];
  const float* b = p.b[l];
  const uint16_t* o = p.o + static_cast<long long>(l) * p.o_mat;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * (kThreads / 32) + warp;
  double acc = 0.0;
  if (i < p.m) {
    const uint16_t* row = o + static_cast<long long>(i) * p.pitch;
    const int nv = p.n & ~7;
    float s = 0.f;
    for (int j = lane * 8; j < nv; j += 32 * 8) {
      float v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      for (int q = 0; q < p.planes; ++q) {
        const uint4 w = __ldcs(reinterpret_cast<const uint4*>(row + q * p.o_plane + j));
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          v[2 * t] += __uint_as_float(u[t] << 16);
          v[2 * t + 1] += __uint_as_float(u[t] & 0xFFFF0000u);
        }
      }
      // b is the caller's vector with no alignment promise: scalar reads (it stays in L1)
#pragma unroll
      for (int t = 0; t < 8; ++t) s = fmaf(v[t], __ldg(b + j + t), s);
    }
    for (int j = nv + lane; j < p.n; j += 32) {
      float v = 0.f;
      for (int q = 0; q < p.planes; ++q) v += bf16_bits_to_float(row[q * p.o_plane + j]);
      s = fmaf(v, b[j], s);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    acc = static_cast<double>(s) * a[i];
  }
  const double tot = block_sum<double>(lane == 0 ? acc : 0.0, scratch);
  if (threadIdx.x == 0) p.partial[static_cast<long long>(l) * gridDim.x + blockIdx.x] = tot;
}

__global__ void cap_alpha_reduce_kernel(const double* partial, int nblk, float* alpha) {
  if (threadIdx.x != 0) return;
  double s = 0.0;
  for (int k = 0; k < nblk; ++k) s += partial[static_cast<long long>(blockIdx.x) * nblk + k];
  alpha[blockIdx.x] = static_cast<float>(s);
}

}  // namespace

cudaError_t launch_gemv_rows(const GemvParams& p, int batch, bool f32, cudaStream_t s) {
  constexpr int kWarps = kThreads / 32;
  // rows per warp: up to 4 (fewer shared-memory fills of x) while keeping >= 4 blocks per SM
  const long long total_rows = static_cast<long long>(p.rows) * batch;
  const int rpw = static_cast<int>(std::max(1LL, std::min(4LL, total_rows / (kWarps * 148LL * 4))));
  const dim3 grid((p.rows + kWarps * rpw - 1) / (kWarps * rpw), batch);
  const size_t smem = sizeof(float) * p.cols;  // up to 128 KB (cols <= 32768)
  // the attribute is per device: set it on every launch that needs more than the default 48 KB
  if (smem > 48 * 1024) {
    const int lim = static_cast<int>(smem);
    cudaFuncSetAttribute(gemv_rows_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    cudaFuncSetAttribute(gemv_rows_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    cudaFuncSetAttribute(gemv_rows_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    cudaFuncSetAttribute(gemv_rows_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
  }
  bool vec = p.cols % 8 == 0;
  for (int l = 0; l < batch && vec; ++l)
    if (reinterpret_cast<uintptr_t>(p.w[l]) % 16) vec = false;
  if (f32) {
    if (vec) gemv_rows_kernel<true, true><<<grid, kThreads, smem, s>>>(p, rpw);
    else gemv_rows_kernel<true, false><<<grid, kThreads, smem, s>>>(p, rpw);
  } else {
    if (vec) gemv_rows_kernel<false, true><<<grid, kThreads, smem, s>>>(p, rpw);
    else gemv_rows_kernel<false, false><<<grid, kThreads, smem, s>>>(p, rpw);
  }
  return cudaGetLastError();
}

cudaError_t launch_gemv_cols(const GemvParams& p, int batch, bool f32, cudaStream_t s) {
  bool vec = p.cols % 8 == 0;
  for (int l = 0; l < batch && vec; ++l)
    if (reinterpret_cast<uintptr_t>(p.w[l]) % 16) vec = false;
  const int per = vec ? 8 : 1;
  // a block spans the columns (up to kThreads threads of `per` columns each): narrow matrices do
  // not leave most of a 256-thread block idle
  const int need = (p.cols + per - 1) / per;
  const int threads = std::min(kThreads, std::max(32, (need + 31) / 32 * 32));
  const dim3 grid((need + threads - 1) / threads, p.row_chunks, batch);
  if (f32) {
    if (vec) gemv_cols_partial_kernel<true, true><<<grid, threads, 0, s>>>(p);
    else gemv_cols_partial_kernel<true, false><<<grid, threads, 0, s>>>(p);
  } else {
    if (vec) gemv_cols_partial_kernel<false, true><<<grid, threads, 0, s>>>(p);
    else gemv_cols_partial_kernel<false, false><<<grid, threads, 0, s>>>(p);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  gemv_cols_reduce_kernel<<<dim3((p.cols + kThreads - 1) / kThreads, batch), kThreads, 0, s>>>(p);
  return cudaGetLastError();
}

int power_pass_max_cols() { return 256 * 8; }

cudaError_t launch_power_iteration_fused(GemvParams& p, int batch, bool f32, float* tsq_partial, int nblk,
                                         int rows_per_block, int iters, float* sigma, cudaStream_t s) {
  const int nv = (p.cols + 255) / 256;
  if (p.cols % 8 != 0 || nv < 1 || nv > 8 || iters < 1) return cudaErrorInvalidValue;
  const size_t smem = sizeof(float) * p.cols * (1 + kThreads / 32);
  const dim3 grid(nblk, batch);
  const int zblk = (p.cols + kThreads - 1) / kThreads;
  float* zsq_partial = tsq_partial + static_cast<long long>(batch) * nblk;
  cudaError_t e = cudaSuccess;
  for (int it = 0; it < iters; ++it) {
    const float* zprev = it == 0 ? nullptr : zsq_partial;
#define MUON_POWER_CASE(NVV)                                                                          \
  case NVV: {                                                                                        \
    auto kern = f32 ? power_pass_kernel<true, NVV> : power_pass_kernel<false, NVV>;                 \
    if (smem > 48 * 1024) {                                                                          \
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)); \
      if (e != cudaSuccess) return e;                                                                \
    }                                                                                                \
    kern<<<grid, kThreads, smem, s>>>(p, rows_per_block, tsq_partial, zprev, zblk);                 \
    break;                                                                                           \
  }
    switch (nv) {
      MUON_POWER_CASE(1)
      MUON_POWER_CASE(2)
      MUON_POWER_CASE(3)
      MUON_POWER_CASE(4)
      MUON_POWER_CASE(5)
      MUON_POWER_CASE(6)
      MUON_POWER_CASE(7)
      MUON_POWER_CASE(8)
    }
#undef MUON_POWER_CASE
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    power_reduce_kernel<<<dim3(zblk, batch), kThreads, 0, s>>>(p, nblk, zsq_partial);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int eblk = (std::max(p.rows, p.cols) + kThreads - 1) / kThreads;
  power_scale_kernel<<<dim3(eblk, batch), kThreads, 0, s>>>(p, nblk, tsq_partial, zblk, zsq_partial, sigma);
  return cudaGetLastError();
}

cudaError_t launch_normalize(float* const* vecs, int batch, int n, float* norm, cudaStream_t s) {
  VecParams p;
  for (int l = 0; l < batch; ++l) p.v[l] = vecs[l];
  p.n = n;
  p.norm = norm;
  normalize_kernel<<<batch, kThreads, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_shift_normalize(float* const* y, const float* const* z, int batch, int n, const float* sigma_max,
                                   cudaStream_t s) {
  ShiftParams p;
  for (int l = 0; l < batch; ++l) {
    p.y[l] = y[l];
    p.z[l] = z[l];
  }
  p.sigma_max = sigma_max;
  p.n = n;
  shift_normalize_kernel<<<batch, kThreads, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_cap_alpha(const CapParams& p, int batch, float* alpha, cudaStream_t s) {
  // one warp per row: p.rows_per_block must equal the warps of a block
  if (p.rows_per_block != kThreads / 32) return cudaErrorInvalidValue;
  const int nblk = (p.m + p.rows_per_block - 1) / p.rows_per_block;
  cap_alpha_partial_kernel<<<dim3(nblk, batch), kThreads, 0, s>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  cap_alpha_reduce_kernel<<<batch, 32, 0, s>>>(p.partial, nblk, alpha);
  return cudaGetLastError();
}

}  // namespace muon
