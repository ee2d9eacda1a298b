// K1: momentum, Nesterov look-ahead and the Frobenius norm in one HBM pass.
//
//   M <- beta*M + G ;  U = G + beta*M (or U = M) ;  nu = ||U||_F
//   (G read as gscale * G: a data-parallel caller's 1/N average, folded into this pass)
//
// (Muon Meets Mamba: Spectral Optimization for State Space Models, abstract:
// the update of each weight matrix is orthogonalised; the momentum, look-ahead
// and normalisation that precede the Newton-Schulz iteration are the optimizer
// state this pass maintains.)
//
// One launch covers every group of a call (blocks cut into per-group ranges),
// so the step has one momentum launch instead of one per shape.
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
#include "rowpos.cuh"

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
__device__ void finish_norm(const MomentumGroup& q, float eps, int l, int b, float local) {
  __shared__ float fscratch[kThreads / 32];
  __shared__ double dscratch[kThreads / 32];
  __shared__ int is_last;
  const float blk = block_sum<float>(local, fscratch);
  if (threadIdx.x == 0) {
    q.partials[static_cast<long long>(l) * q.nblk + b] = blk;
    __threadfence();
    const unsigned prev = atomicAdd(&q.counters[l], 1u);
    is_last = (prev == static_cast<unsigned>(q.nblk) - 1u);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  double acc = 0.0;
  for (int i = threadIdx.x; i < q.nblk; i += kThreads)
    acc += static_cast<double>(__ldcg(&q.partials[static_cast<long long>(l) * q.nblk + i]));
  const double tot = block_sum<double>(acc, dscratch);
  if (threadIdx.x == 0) {
    const float nu = static_cast<float>(sqrt(tot));
    const float s1 = 1.0f / (nu + eps);
    const float s2 = s1 * s1;
    q.nu[l] = nu;
    q.scale1[l] = s1;
    q.scale2[l] = s2;
    const bool ok = isfinite(nu) && isfinite(s2);
    q.flags[l] = ok ? 0 : MUON_FLAG_NONFINITE;
    q.counters[l] = 0u;  // ready for the next call
  }
}

// M, U of 8 consecutive elements from G (and M): one vector step of the wide path.
template <typename TG, bool MOM>
__device__ __forceinline__ void lookahead8(const MomentumParams& p, float (&gv)[8], float (&mv)[8], float (&u)[8]) {
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    gv[t] *= p.gscale;
    if (MOM) {
      mv[t] = fmaf(p.beta, mv[t], gv[t]);
      u[t] = p.nesterov ? fmaf(p.beta, mv[t], gv[t]) : mv[t];
    } else {
      u[t] = gv[t];
    }
  }
}

// Wide matrices (rows <= cols): X(i, j) = U(i, j).  Vector path: 8 elements per
// thread step, two steps in flight (both loads issued before either is used).
template <typename TG, bool MOM, int PLANES>
__device__ __forceinline__ void wide_body(const MomentumParams& p, const MomentumGroup& q, int l, int b) {
  const TG* __restrict__ g = static_cast<const TG*>(p.g[q.mat0 + l]);
  float* __restrict__ m = MOM ? p.m[q.mat0 + l] : nullptr;
  uint16_t* __restrict__ x = q.x + static_cast<long long>(l) * q.x_mat;
  const int C = q.cols;
  float ss = 0.f;
  if (q.vec) {
    const int per_row = C / 8;
    const long long total = static_cast<long long>(q.rows) * per_row;
    const long long chunk = (total + q.nblk - 1) / q.nblk;
    const long long beg = chunk * b;
    const long long end = min(total, beg + chunk);
    const RowStep one = rowstep_of(kThreads, per_row), two_steps = rowstep_of(2 * kThreads, per_row);
    RowPos pa = rowpos_at(beg + threadIdx.x, per_row);
    for (long long v0 = beg + threadIdx.x; v0 < end; v0 += 2 * kThreads, pa = rowpos_add(pa, two_steps, per_row)) {
      const long long v1 = v0 + kThreads;
      const bool two = v1 < end;
      const RowPos pb = rowpos_add(pa, one, per_row);
      const long long i0 = pa.i, i1 = pb.i;
      const int j0 = pa.j * 8, j1 = pb.j * 8;
      const long long e0 = i0 * C + j0, e1 = i1 * C + j1;
      float ga[8], gb[8], ma[8], mb[8], ua[8], ub[8];
      load8<TG>(g + e0, ga);
      if (MOM) load8_f32(m + e0, ma);
      if (two) {
        load8<TG>(g + e1, gb);
        if (MOM) load8_f32(m + e1, mb);
      }
      lookahead8<TG, MOM>(p, ga, ma, ua);
      if (MOM) store8_f32(m + e0, ma);
#pragma unroll
      for (int t = 0; t < 8; ++t) ss = fmaf(ua[t], ua[t], ss);
      store8_planes<PLANES>(x + i0 * q.pitch + j0, q.x_plane, ua);
      if (two) {
        lookahead8<TG, MOM>(p, gb, mb, ub);
        if (MOM) store8_f32(m + e1, mb);
#pragma unroll
        for (int t = 0; t < 8; ++t) ss = fmaf(ub[t], ub[t], ss);
        store8_planes<PLANES>(x + i1 * q.pitch + j1, q.x_plane, ub);
      }
    }
  } else {
    const long long total = static_cast<long long>(q.rows) * C;
    const long long chunk = (total + q.nblk - 1) / q.nblk;
    const long long beg = chunk * b;
    const long long end = min(total, beg + chunk);
    for (long long e = beg + threadIdx.x; e < end; e += kThreads) {
      const long long i = e / C;
      const int j = static_cast<int>(e - i * C);
      const float gv = p.gscale * load_elem<TG>(g + e);
      const float u = MOM ? momentum_lookahead(gv, m + e, p.beta, p.nesterov) : gv;
      ss = fmaf(u, u, ss);
      store1_planes<PLANES>(x + i * q.pitch + j, q.x_plane, u);
    }
  }
  finish_norm(q, p.eps, l, b, ss);
}

// Tall matrices (rows > cols): X(j, i) = U(i, j) through a 64 x 64 tile.
template <typename TG, bool MOM, int PLANES>
__device__ __forceinline__ void tall_body(const MomentumParams& p, const MomentumGroup& q, int l, int b) {
  __shared__ float tile[64][65];
  const TG* __restrict__ g = static_cast<const TG*>(p.g[q.mat0 + l]);
  float* __restrict__ m = MOM ? p.m[q.mat0 + l] : nullptr;
  uint16_t* __restrict__ x = q.x + static_cast<long long>(l) * q.x_mat;
  const int R = q.rows, C = q.cols;
  const int tiles_c = (C + 63) / 64;
  const int ntiles = ((R + 63) / 64) * tiles_c;
  const int rr = threadIdx.x >> 3;        // 0..31
  const int cc = (threadIdx.x & 7) * 8;   // 0..56
  float ss = 0.f;
  // tile tt = (row tile, column tile) walked in strides of nblk without a division per tile
  const RowStep tstep = rowstep_of(q.nblk, tiles_c);
  RowPos tp = rowpos_at(b, tiles_c);
  for (int tt = b; tt < ntiles; tt += q.nblk, tp = rowpos_add(tp, tstep, tiles_c)) {
    const int r0 = tp.i * 64, c0 = tp.j * 64;
    float u[2][8];
    if (q.vec) {
      // both passes' loads first: two rows of 8 in flight per thread
      float gv[2][8], mv[2][8];
      bool in[2];
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {
        const int i = r0 + rr + 32 * pass;
        const int j = c0 + cc;
        in[pass] = i < R && j < C;
        if (in[pass]) {
          const long long e = static_cast<long long>(i) * C + j;
          load8<TG>(g + e, gv[pass]);
          if (MOM) load8_f32(m + e, mv[pass]);
        }
      }
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {
        if (in[pass]) {
          lookahead8<TG, MOM>(p, gv[pass], mv[pass], u[pass]);
          if (MOM) {
            const long long e = static_cast<long long>(r0 + rr + 32 * pass) * C + c0 + cc;
            store8_f32(m + e, mv[pass]);
          }
        } else {
#pragma unroll
          for (int t = 0; t < 8; ++t) u[pass][t] = 0.f;
        }
      }
    } else {
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {
        const int i = r0 + rr + 32 * pass;
        const int j = c0 + cc;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          u[pass][t] = 0.f;
          if (i < R && j + t < C) {
            const long long e = static_cast<long long>(i) * C + j + t;
            const float gv = p.gscale * load_elem<TG>(g + e);
            u[pass][t] = MOM ? momentum_lookahead(gv, m + e, p.beta, p.nesterov) : gv;
          }
        }
      }
    }
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        ss = fmaf(u[pass][t], u[pass][t], ss);
        tile[rr + 32 * pass][cc + t] = u[pass][t];
      }
    }
    __syncthreads();
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
      const int jl = rr + 32 * pass;      // local column of W = local row of X
      const int j = c0 + jl;
      const int i = r0 + cc;              // first of 8 consecutive W rows
      if (j < C && i < R) {
        float uo[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) uo[t] = tile[cc + t][jl];
        // pitch >= round_up(R, 8) and i % 8 == 0, so the 8-wide store stays in the row
        store8_planes<PLANES>(x + static_cast<long long>(j) * q.pitch + i, q.x_plane, uo);
      }
    }
    __syncthreads();
  }
  finish_norm(q, p.eps, l, b, ss);
}

// Every group of the launch: the block range of group g starts at grp[g].block0.
template <typename TG, bool MOM, int PLANES>
__global__ void __launch_bounds__(kThreads, 4) momentum_kernel(const __grid_constant__ MomentumParams p) {
  int gi = 0;
  while (gi + 1 < p.ngroups && static_cast<int>(blockIdx.x) >= p.grp[gi + 1].block0) ++gi;
  const MomentumGroup& q = p.grp[gi];
  const int local = static_cast<int>(blockIdx.x) - q.block0;
  const int lr = local / q.nblk;
  const int b = local - lr * q.nblk;
  // matrices last to first: the Newton-Schulz launch reads matrix 0 first, so its U is written last
  const int l = q.batch - 1 - lr;
  if (q.rows > q.cols) tall_body<TG, MOM, PLANES>(p, q, l, b);
  else wide_body<TG, MOM, PLANES>(p, q, l, b);
}

bool pointers_aligned(const MomentumParams& p, const MomentumGroup& q, bool mom) {
  for (int l = 0; l < q.batch; ++l) {
    if (reinterpret_cast<uintptr_t>(p.g[q.mat0 + l]) % 16) return false;
    if (mom && reinterpret_cast<uintptr_t>(p.m[q.mat0 + l]) % 16) return false;
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

cudaError_t launch_momentum(MomentumParams& p, bool g_is_f32, bool momentum, int planes, cudaStream_t stream) {
  if (p.ngroups < 1 || p.ngroups > MUON_MAX_GROUPS) return cudaErrorInvalidValue;
  long long blocks = 0;
  for (int gi = 0; gi < p.ngroups; ++gi) {
    MomentumGroup& q = p.grp[gi];
    q.block0 = static_cast<int>(blocks);
    q.vec = (q.cols % 8 == 0) && pointers_aligned(p, q, momentum);
    blocks += static_cast<long long>(q.batch) * q.nblk;
  }
  if (blocks < 1 || blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(blocks));
  if (g_is_f32) {
    if (planes != 3) return cudaErrorInvalidValue;
    if (momentum) momentum_kernel<float, true, 3><<<grid, kThreads, 0, stream>>>(p);
    else momentum_kernel<float, false, 3><<<grid, kThreads, 0, stream>>>(p);
  } else {
    if (planes != 1) return cudaErrorInvalidValue;
    if (momentum) momentum_kernel<uint16_t, true, 1><<<grid, kThreads, 0, stream>>>(p);
    else momentum_kernel<uint16_t, false, 1><<<grid, kThreads, 0, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace muon
