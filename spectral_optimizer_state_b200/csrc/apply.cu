// K5: scale and apply the orthogonalised update with decoupled weight decay,
//
//   W <- (1 - lr*wd) * W - lr * s(rows, cols) * O          (apply)
//   Out <- O                                                (orthogonalise only)
//
// (Muon Meets Mamba: Spectral Optimization for State Space Models, abstract:
// Muon updates each weight matrix with its orthogonalised step; the shape
// scale and the decay taken from the pre-step W are the readings this library
// uses for what the page leaves open.)
//
// O is the last Newton-Schulz iterate in the workspace: wide orientation,
// PLANES bf16 planes summed in fp32.  A wide W is updated row by row with
// 16-byte vectors; a tall W (O stored transposed) goes through a 64 x 64
// shared-memory tile so the reads of O and the read-modify-write of W are
// both coalesced.  This pass is HBM-bound: it runs with full occupancy so
// enough bytes are in flight, which the GEMM epilogue (a few warps per SM
// behind a 200 KB shared-memory pipeline) cannot do.
#include <cuda_bf16.h>

#include "device_utils.cuh"
#include "internal.h"

namespace muon {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ void load8_planes(const uint16_t* o, long long ps, int planes, float (&v)[8]) {
#pragma unroll
  for (int t = 0; t < 8; ++t) v[t] = 0.f;
  for (int p = 0; p < planes; ++p) {
    const uint4 q = __ldcs(reinterpret_cast<const uint4*>(o + p * ps));
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] += __uint_as_float(w[i] << 16);
      v[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

__device__ __forceinline__ float load1_planes(const uint16_t* o, long long ps, int planes) {
  float v = 0.f;
  for (int p = 0; p < planes; ++p) v += bf16_bits_to_float(o[p * ps]);
  return v;
}

// dst[0..8) <- f(dst, v), dst 16-byte aligned (bf16) or 32-byte (fp32).
template <bool F32>
__device__ __forceinline__ void rmw8(void* dst, const float (&v)[8], bool apply, float decay, float lrs) {
  if (F32) {
    float4* p = reinterpret_cast<float4*>(dst);
    float c[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (apply) {
      const float4 a = p[0], b = p[1];
      c[0] = a.x; c[1] = a.y; c[2] = a.z; c[3] = a.w; c[4] = b.x; c[5] = b.y; c[6] = b.z; c[7] = b.w;
    }
    float o[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) o[t] = apply ? fmaf(decay, c[t], -lrs * v[t]) : v[t];
    p[0] = make_float4(o[0], o[1], o[2], o[3]);
    p[1] = make_float4(o[4], o[5], o[6], o[7]);
  } else {
    uint4* p = reinterpret_cast<uint4*>(dst);
    float c[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (apply) {
      const uint4 q = *p;
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        c[2 * i] = __uint_as_float(w[i] << 16);
        c[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
    }
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float a = apply ? fmaf(decay, c[2 * i], -lrs * v[2 * i]) : v[2 * i];
      const float b = apply ? fmaf(decay, c[2 * i + 1], -lrs * v[2 * i + 1]) : v[2 * i + 1];
      w[i] = static_cast<uint32_t>(float_to_bf16_bits(a)) | (static_cast<uint32_t>(float_to_bf16_bits(b)) << 16);
    }
    *p = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

template <bool F32>
__device__ __forceinline__ void rmw1(void* dst, long long e, float v, bool apply, float decay, float lrs) {
  if (F32) {
    float* W = static_cast<float*>(dst);
    W[e] = apply ? fmaf(decay, W[e], -lrs * v) : v;
  } else {
    uint16_t* W = static_cast<uint16_t*>(dst);
    W[e] = float_to_bf16_bits(apply ? fmaf(decay, bf16_bits_to_float(W[e]), -lrs * v) : v);
  }
}

// Wide W (rows <= cols): W(i, j) with O(i, j).  CAP: O - alpha u v^T (spectral cap).
template <bool F32, bool VEC, bool CAP>
__global__ void __launch_bounds__(kThreads) apply_wide_kernel(const __grid_constant__ ApplyParams p) {
  const int l = blockIdx.y;
  if (p.flags != nullptr && p.flags[l] != 0) return;
  if (p.status != nullptr && (*p.status & kStatusTimeout)) return;  // the iterate is incomplete
  void* w = p.w[l];
  const uint16_t* o = p.o + static_cast<long long>(l) * p.o_mat;
  const int C = p.cols;
  if (VEC) {
    const long long per_row = C / 8;
    const long long total = static_cast<long long>(p.rows) * per_row;
    const long long chunk = (total + p.nblk - 1) / p.nblk;
    const long long beg = chunk * blockIdx.x;
    const long long end = min(total, beg + chunk);
    for (long long v = beg + threadIdx.x; v < end; v += kThreads) {
      const long long i = v / per_row;
      const int j = static_cast<int>(v - i * per_row) * 8;
      float ov[8];
      load8_planes(o + i * p.pitch + j, p.o_plane, p.planes, ov);
      if (CAP) {
        const float au = p.alpha[l] * p.cu[l][i];
#pragma unroll
        for (int t = 0; t < 8; ++t) ov[t] = fmaf(-au, p.cv[l][j + t], ov[t]);
      }
      char* dst = static_cast<char*>(w) + (i * C + j) * (F32 ? 4 : 2);
      rmw8<F32>(dst, ov, p.apply, p.decay, p.lrs);
    }
  } else {
    const long long total = static_cast<long long>(p.rows) * C;
    const long long chunk = (total + p.nblk - 1) / p.nblk;
    const long long beg = chunk * blockIdx.x;
    const long long end = min(total, beg + chunk);
    for (long long e = beg + threadIdx.x; e < end; e += kThreads) {
      const long long i = e / C;
      const int j = static_cast<int>(e - i * C);
      float ov = load1_planes(o + i * p.pitch + j, p.o_plane, p.planes);
      if (CAP) ov = fmaf(-p.alpha[l] * p.cu[l][i], p.cv[l][j], ov);
      rmw1<F32>(w, e, ov, p.apply, p.decay, p.lrs);
    }
  }
}

// Tall W (rows > cols): W(r, c) with O(c, r), through a 64 x 64 tile.
template <bool F32, bool VEC, bool CAP>
__global__ void __launch_bounds__(kThreads) apply_tall_kernel(const __grid_constant__ ApplyParams p) {
  __shared__ float tile[64][65];
  const int l = blockIdx.y;
  if (p.flags != nullptr && p.flags[l] != 0) return;
  if (p.status != nullptr && (*p.status & kStatusTimeout)) return;  // the iterate is incomplete
  void* w = p.w[l];
  const uint16_t* o = p.o + static_cast<long long>(l) * p.o_mat;
  const int R = p.rows, C = p.cols;
  const int tiles_c = (C + 63) / 64;
  const int ntiles = ((R + 63) / 64) * tiles_c;
  const int rr = threadIdx.x >> 3;       // 0..31
  const int cc = (threadIdx.x & 7) * 8;  // 0..56
  for (int tt = blockIdx.x; tt < ntiles; tt += gridDim.x) {
    const int r0 = (tt / tiles_c) * 64, c0 = (tt % tiles_c) * 64;
    // O rows c (= W columns), 8 consecutive W rows r per thread: O(c, r..r+7)
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
      const int c = c0 + rr + 32 * pass;
      const int r = r0 + cc;
      float ov[8];
      if (c < C && r < R) {
        // the wide pitch is >= round_up(R, 8) and r % 8 == 0: the 8-wide read stays in the row
        load8_planes(o + static_cast<long long>(c) * p.pitch + r, p.o_plane, p.planes, ov);
      } else {
#pragma unroll
        for (int t = 0; t < 8; ++t) ov[t] = 0.f;
      }
#pragma unroll
      for (int t = 0; t < 8; ++t) tile[cc + t][rr + 32 * pass] = ov[t];
    }
    __syncthreads();
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
      const int rl = rr + 32 * pass;
      const int r = r0 + rl;
      const int c = c0 + cc;
      if (r < R) {
        float ov[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) ov[t] = tile[rl][cc + t];
        if (CAP) {
          const float au = p.alpha[l] * p.cu[l][r];
#pragma unroll
          for (int t = 0; t < 8; ++t)
            if (c + t < C) ov[t] = fmaf(-au, p.cv[l][c + t], ov[t]);
        }
        if (VEC) {
          if (c < C) {
            char* dst = static_cast<char*>(w) + (static_cast<long long>(r) * C + c) * (F32 ? 4 : 2);
            rmw8<F32>(dst, ov, p.apply, p.decay, p.lrs);
          }
        } else {
#pragma unroll
          for (int t = 0; t < 8; ++t)
            if (c + t < C) rmw1<F32>(w, static_cast<long long>(r) * C + c + t, ov[t], p.apply, p.decay, p.lrs);
        }
      }
    }
    __syncthreads();
  }
}

template <bool F32, bool CAP>
cudaError_t launch_typed(const ApplyParams& p, int batch, bool tall, bool vec, cudaStream_t s) {
  dim3 grid(p.nblk, batch);
  if (tall) {
    if (vec) apply_tall_kernel<F32, true, CAP><<<grid, kThreads, 0, s>>>(p);
    else apply_tall_kernel<F32, false, CAP><<<grid, kThreads, 0, s>>>(p);
  } else {
    if (vec) apply_wide_kernel<F32, true, CAP><<<grid, kThreads, 0, s>>>(p);
    else apply_wide_kernel<F32, false, CAP><<<grid, kThreads, 0, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_apply(const ApplyParams& p, int batch, bool w_f32, cudaStream_t stream) {
  const bool tall = p.rows > p.cols;
  bool vec = p.cols % 8 == 0;
  for (int l = 0; l < batch && vec; ++l)
    if (reinterpret_cast<uintptr_t>(p.w[l]) % 16) vec = false;
  // the cap term is its own instantiation: the plain pass keeps its register allocation
  if (p.alpha != nullptr)
    return w_f32 ? launch_typed<true, true>(p, batch, tall, vec, stream)
                 : launch_typed<false, true>(p, batch, tall, vec, stream);
  return w_f32 ? launch_typed<true, false>(p, batch, tall, vec, stream)
               : launch_typed<false, false>(p, batch, tall, vec, stream);
}

}  // namespace muon
