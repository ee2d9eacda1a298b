// K1: momentum, Nesterov look-ahead and the Frobenius norm in one HBM pass.
//
//   M <- beta*M + G ;  U = G + beta*M (or U = M) ;  nu = ||U||_F
//
// (Muon Meets Mamba: Spectral Optimization for State Space Models, abstract:
// the update of each weight matrix is orthogonalised; the momentum, look-ahead
// and normalisation that precede the Newton-Schulz iteration are the optimizer
// state this pass maintains.)
//
// U is written, un-normalised, into the workspace in the WIDE orientation
// (min(rows, cols) rows): a wide matrix is copied row by row with 16-byte
// vectors, a tall one is transposed through a 64 x 64 shared-memory tile so
// both its reads and its writes stay coalesced.  The 1/(nu+eps) factor is not
// applied here -- the first Newton-Schulz iteration folds it into its
// epilogues -- so the pass stays single.  The norm is reduced
// deterministically: per-thread fp32 sums, a fixed warp-shuffle and block
// tree, per-block partials, and the last block of each matrix sums the
// partials in a fixed order in fp64.
#include <cuda_bf16.h>

#include "device_utils.cuh"
#include "internal.h"

namespace muon {

namespace {

constexpr int kThreads = 256;

template <typename T>
__device__ __forceinline__ float load_elem(const T* p);
template <>
__device__ __forceinline__ float load_elem<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float load_elem<uint16_t>(const uint16_t* p) {
  return bf16_bits_to_float(*p);
}

// Load 8 consecutive elements (16-byte aligned for bf16, 32-byte for fp32).
template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&v)[8]);
template <>
__device__ __forceinline__ void load8<uint16_t>(const uint16_t* p, float (&v)[8]) {
  uint4 q = __ldcs(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&v)[8]) {
  float4 a = __ldcs(reinterpret_cast<const float4*>(p));
  float4 b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void load8_f32(const float* p, float (&v)[8]) {
  float4 a = __ldcs(reinterpret_cast<const float4*>(p));
  float4 b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void store8_f32(float* p, const float (&v)[8]) {
  __stcs(reinterpret_cast<float4*>(p), make_float4(v[0], v[1], v[2], v[3]));
  __stcs(reinterpret_cast<float4*>(p) + 1, make_float4(v[4], v[5], v[6], v[7]));
}

// Store 8 values as PLANES bf16 planes at x (16-byte aligned), plane stride ps.
template <int PLANES>
__device__ __forceinline__ void store8_planes(uint16_t* x, long long ps, const float (&u)[8]) {
  uint32_t w[PLANES][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint16_t a[PLANES], b[PLANES];
    split_planes<PLANES>(u[2 * i], a);
    split_planes<PLANES>(u[2 * i + 1], b);
#pragma unroll
    for (int p = 0; p < PLANES; ++p) w[p][i] = static_cast<uint32_t>(a[p]) | (static_cast<uint32_t>(b[p]) << 16);
  }
#pragma unroll
  for (int p = 0; p < PLANES; ++p)
    *reinterpret_cast<uint4*>(x + p * ps) = make_uint4(w[p][0], w[p][1], w[p][2], w[p][3]);
}

template <int PLANES>
__device__ __forceinline__ void store1_planes(uint16_t* x, long long ps, float u) {
  uint16_t a[PLANES];
  split_planes<PLANES>(u, a);
#pragma unroll
  for (int p = 0; p < PLANES; ++p) x[p * ps] = a[p];
}

__device__ __forceinline__ float momentum_lookahead(float g, float* m, float beta, int nesterov) {
  const float mn = fmaf(beta, *m, g);
  *m = mn;
  return nesterov ? fmaf(beta, mn, g) : mn;
}

// Block-wide deterministic sum; result valid in thread 0.
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

// Write this block's partial, and let the last block of the matrix finish the norm.
__device__ void finish_norm(const MomentumParams& p, int l, float local) {
  __shared__ float fscratch[kThreads / 32];
  __shared__ double dscratch[kThreads / 32];
  __shared__ int is_last;
  const float blk = block_sum<float>(local, fscratch);
  if (threadIdx.x == 0) {
    p.partials[static_cast<long long>(l) * p.nblk + blockIdx.x] = blk;
    __threadfence();
    const unsigned prev = atomicAdd(&p.counters[l], 1u);
    is_last = (prev == static_cast<unsigned>(p.nblk) - 1u);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  double acc = 0.0;
  for (int b = threadIdx.x; b < p.nblk; b += kThreads)
    acc += static_cast<double>(__ldcg(&p.partials[static_cast<long long>(l) * p.nblk + b]));
  const double tot = block_sum<double>(acc, dscratch);
  if (threadIdx.x == 0) {
    const float nu = static_cast<float>(sqrt(tot));
    const float s1 = 1.0f / (nu + p.eps);
    const float s2 = s1 * s1;
    p.nu[l] = nu;
    p.scale1[l] = s1;
    p.scale2[l] = s2;
    const bool ok = isfinite(nu) && isfinite(s2);
    p.flags[l] = ok ? 0 : MUON_FLAG_NONFINITE;
    p.counters[l] = 0u;  // ready for the next call
  }
}

// Wide matrices (rows <= cols): X(i, j) = U(i, j).  VEC: cols % 8 == 0 and
// 16-byte aligned rows, 8 elements per thread step; else one element.
template <typename TG, bool MOM, int PLANES, bool VEC>
__global__ void __launch_bounds__(kThreads) momentum_wide_kernel(const __grid_constant__ MomentumParams p) {
  const int l = blockIdx.y;
  const TG* __restrict__ g = static_cast<const TG*>(p.g[l]);
  float* __restrict__ m = MOM ? p.m[l] : nullptr;
  uint16_t* __restrict__ x = p.x + static_cast<long long>(l) * p.x_mat;
  const int C = p.cols;
  float ss = 0.f;
  if (VEC) {
    const long long per_row = C / 8;
    const long long total = static_cast<long long>(p.rows) * per_row;
    const long long chunk = (total + p.nblk - 1) / p.nblk;
    const long long beg = chunk * blockIdx.x;
    const long long end = min(total, beg + chunk);
    for (long long v = beg + threadIdx.x; v < end; v += kThreads) {
      const long long i = v / per_row;
      const int j = static_cast<int>(v - i * per_row) * 8;
      const long long e = i * C + j;
      float gv[8], u[8];
      load8<TG>(g + e, gv);
      if (MOM) {
        float mv[8];
        load8_f32(m + e, mv);
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          mv[t] = fmaf(p.beta, mv[t], gv[t]);
          u[t] = p.nesterov ? fmaf(p.beta, mv[t], gv[t]) : mv[t];
        }
        store8_f32(m + e, mv);
      } else {
#pragma unroll
        for (int t = 0; t < 8; ++t) u[t] = gv[t];
      }
#pragma unroll
      for (int t = 0; t < 8; ++t) ss = fmaf(u[t], u[t], ss);
      store8_planes<PLANES>(x + i * p.pitch + j, p.x_plane, u);
    }
  } else {
    const long long total = static_cast<long long>(p.rows) * C;
    const long long chunk = (total + p.nblk - 1) / p.nblk;
    const long long beg = chunk * blockIdx.x;
    const long long end = min(total, beg + chunk);
    for (long long e = beg + threadIdx.x; e < end; e += kThreads) {
      const long long i = e / C;
      const int j = static_cast<int>(e - i * C);
      const float gv = load_elem<TG>(g + e);
      const float u = MOM ? momentum_lookahead(gv, m + e, p.beta, p.nesterov) : gv;
      ss = fmaf(u, u, ss);
      store1_planes<PLANES>(x + i * p.pitch + j, p.x_plane, u);
    }
  }
  finish_norm(p, l, ss);
}

// Tall matrices (rows > cols): X(j, i) = U(i, j) through a 64 x 64 tile.
template <typename TG, bool MOM, int PLANES, bool VEC>
__global__ void __launch_bounds__(kThreads) momentum_tall_kernel(const __grid_constant__ MomentumParams p) {
  __shared__ float tile[64][65];
  const int l = blockIdx.y;
  const TG* __restrict__ g = static_cast<const TG*>(p.g[l]);
  float* __restrict__ m = MOM ? p.m[l] : nullptr;
  uint16_t* __restrict__ x = p.x + static_cast<long long>(l) * p.x_mat;
  const int R = p.rows, C = p.cols;
  const int tiles_c = (C + 63) / 64;
  const int ntiles = ((R + 63) / 64) * tiles_c;
  const int rr = threadIdx.x >> 3;        // 0..31
  const int cc = (threadIdx.x & 7) * 8;   // 0..56
  float ss = 0.f;
  for (int tt = blockIdx.x; tt < ntiles; tt += gridDim.x) {
    const int r0 = (tt / tiles_c) * 64, c0 = (tt % tiles_c) * 64;
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
      const int i = r0 + rr + 32 * pass;
      const int j = c0 + cc;
      float u[8];
      if (VEC) {
        if (i < R && j < C) {
          const long long e = static_cast<long long>(i) * C + j;
          float gv[8];
          load8<TG>(g + e, gv);
          if (MOM) {
            float mv[8];
            load8_f32(m + e, mv);
#pragma unroll
            for (int t = 0; t < 8; ++t) {
              mv[t] = fmaf(p.beta, mv[t], gv[t]);
              u[t] = p.nesterov ? fmaf(p.beta, mv[t], gv[t]) : mv[t];
            }
            store8_f32(m + e, mv);
          } else {
#pragma unroll
            for (int t = 0; t < 8; ++t) u[t] = gv[t];
          }
        } else {
#pragma unroll
          for (int t = 0; t < 8; ++t) u[t] = 0.f;
        }
      } else {
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          u[t] = 0.f;
          if (i < R && j + t < C) {
            const long long e = static_cast<long long>(i) * C + j + t;
            const float gv = load_elem<TG>(g + e);
            u[t] = MOM ? momentum_lookahead(gv, m + e, p.beta, p.nesterov) : gv;
          }
        }
      }
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        ss = fmaf(u[t], u[t], ss);
        tile[rr + 32 * pass][cc + t] = u[t];
      }
    }
    __syncthreads();
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
      const int jl = rr + 32 * pass;      // local column of W = local row of X
      const int j = c0 + jl;
      const int i = r0 + cc;              // first of 8 consecutive W rows
      if (j < C && i < R) {
        float u[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) u[t] = tile[cc + t][jl];
        // pitch >= round_up(R, 8) and i % 8 == 0, so the 8-wide store stays in the row
        store8_planes<PLANES>(x + static_cast<long long>(j) * p.pitch + i, p.x_plane, u);
      }
    }
    __syncthreads();
  }
  finish_norm(p, l, ss);
}

template <typename TG, bool MOM, int PLANES>
cudaError_t launch_typed(const MomentumParams& p, int batch, bool tall, bool vec, cudaStream_t s) {
  dim3 grid(p.nblk, batch);
  if (tall) {
    if (vec) momentum_tall_kernel<TG, MOM, PLANES, true><<<grid, kThreads, 0, s>>>(p);
    else momentum_tall_kernel<TG, MOM, PLANES, false><<<grid, kThreads, 0, s>>>(p);
  } else {
    if (vec) momentum_wide_kernel<TG, MOM, PLANES, true><<<grid, kThreads, 0, s>>>(p);
    else momentum_wide_kernel<TG, MOM, PLANES, false><<<grid, kThreads, 0, s>>>(p);
  }
  return cudaGetLastError();
}

bool pointers_aligned(const MomentumParams& p, int batch, bool mom) {
  for (int l = 0; l < batch; ++l) {
    if (reinterpret_cast<uintptr_t>(p.g[l]) % 16) return false;
    if (mom && reinterpret_cast<uintptr_t>(p.m[l]) % 16) return false;
  }
  return true;
}

}  // namespace

int momentum_blocks_per_matrix(int rows, int cols) {
  const long long elems = static_cast<long long>(rows) * cols;
  if (rows > cols) {
    const long long tiles = static_cast<long long>((rows + 63) / 64) * ((cols + 63) / 64);
    // up to 4 tiles of 64 x 64 per block
    long long b = (tiles + 3) / 4;
    return static_cast<int>(b < 1 ? 1 : (b > 4096 ? 4096 : b));
  }
  long long b = (elems + 8191) / 8192;  // ~8K elements per block
  return static_cast<int>(b < 1 ? 1 : (b > 4096 ? 4096 : b));
}

cudaError_t launch_momentum(const MomentumParams& p, int batch, bool g_is_f32, bool momentum,
                            int planes, cudaStream_t stream) {
  const bool tall = p.rows > p.cols;
  const bool vec = (p.cols % 8 == 0) && pointers_aligned(p, batch, momentum);
  if (g_is_f32) {
    if (planes != 3) return cudaErrorInvalidValue;
    return momentum ? launch_typed<float, true, 3>(p, batch, tall, vec, stream)
                    : launch_typed<float, false, 3>(p, batch, tall, vec, stream);
  }
  if (planes != 1) return cudaErrorInvalidValue;
  return momentum ? launch_typed<uint16_t, true, 1>(p, batch, tall, vec, stream)
                  : launch_typed<uint16_t, false, 1>(p, batch, tall, vec, stream);
}

}  // namespace muon
