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
