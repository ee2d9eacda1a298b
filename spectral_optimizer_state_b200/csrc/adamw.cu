// AdamW for the parameters Muon does not take (embeddings, norms, convolution
// weights, SSM scalars, and whichever projection group is not trained with
// Muon), one launch for any number of tensors of any shapes.
//
//   m <- b1 m + (1 - b1) g ;  v <- b2 v + (1 - b2) g^2
//   W <- W (1 - lr wd) - (lr / (1 - b1^t)) m / (sqrt(v) / sqrt(1 - b2^t) + eps)
//
// (Muon Meets Mamba: Spectral Optimization for State Space Models, abstract:
// the protocol trains the weight groups Muon does not take with AdamW.)
// HBM-bound: 22 bytes per element for bf16 weights (G 2, m 4, v 4, W 2 read;
// m 4, v 4, W 2 written).  Work is cut into 4096-element chunks; a block finds
// its tensor by binary search over the chunk prefix sums.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>

#include "../../include/muon.h"
#include "device_utils.cuh"

namespace {

constexpr int kThreads = 256;
constexpr long long kChunk = 4096;  // elements per chunk: 2 vectors of 8 per thread

struct AdamWParams {
  void* w[MUON_MAX_BATCH];
  const void* g[MUON_MAX_BATCH];
  float* m[MUON_MAX_BATCH];
  float* v[MUON_MAX_BATCH];
  long long numel[MUON_MAX_BATCH];
  int chunk_prefix[MUON_MAX_BATCH + 1];  // first chunk of each tensor; [count] = total
  int vec[MUON_MAX_BATCH];               // 16-byte aligned bases
  int count;
  float beta1, beta2, eps, decay, step_size, inv_sqrt_bc2;
};

template <bool F32>
__device__ __forceinline__ void load8(const void* p, long long e, float (&x)[8]) {
  if (F32) {
    const float4* q = reinterpret_cast<const float4*>(static_cast<const float*>(p) + e);
    const float4 a = __ldcs(q), b = __ldcs(q + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  } else {
    const uint4 q = __ldcs(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p) + e));
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

template <bool F32>
__device__ __forceinline__ void store8(void* p, long long e, const float (&x)[8]) {
  if (F32) {
    float4* q = reinterpret_cast<float4*>(static_cast<float*>(p) + e);
    q[0] = make_float4(x[0], x[1], x[2], x[3]);
    q[1] = make_float4(x[4], x[5], x[6], x[7]);
  } else {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      w[i] = static_cast<uint32_t>(muon::float_to_bf16_bits(x[2 * i])) |
             (static_cast<uint32_t>(muon::float_to_bf16_bits(x[2 * i + 1])) << 16);
    *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p) + e) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

__device__ __forceinline__ float adamw_elem(const AdamWParams& p, float w, float g, float& m, float& v) {
  m = fmaf(p.beta1, m, (1.0f - p.beta1) * g);
  v = fmaf(p.beta2, v, (1.0f - p.beta2) * g * g);
  const float den = fmaf(sqrtf(v), p.inv_sqrt_bc2, p.eps);
  return fmaf(p.decay, w, -p.step_size * (m / den));
}

template <bool F32>
__global__ void __launch_bounds__(kThreads) adamw_kernel(const __grid_constant__ AdamWParams p) {
  const int total = p.chunk_prefix[p.count];
  for (int c = blockIdx.x; c < total; c += gridDim.x) {
    int lo = 0, hi = p.count - 1;  // last tensor whose first chunk <= c
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.chunk_prefix[mid] <= c) lo = mid;
      else hi = mid - 1;
    }
    const int t = lo;
    const long long beg = static_cast<long long>(c - p.chunk_prefix[t]) * kChunk;
    const long long end = min(p.numel[t], beg + kChunk);
    void* W = p.w[t];
    const void* G = p.g[t];
    float* M = p.m[t];
    float* V = p.v[t];
    if (p.vec[t] && end - beg == kChunk) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const long long e = beg + (static_cast<long long>(h) * kThreads + threadIdx.x) * 8;
        float w[8], g[8], m[8], v[8];
        load8<F32>(W, e, w);
        load8<F32>(G, e, g);
        load8<true>(M, e, m);
        load8<true>(V, e, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = adamw_elem(p, w[i], g[i], m[i], v[i]);
        store8<F32>(W, e, w);
        store8<true>(M, e, m);
        store8<true>(V, e, v);
      }
    } else {
      for (long long e = beg + threadIdx.x; e < end; e += kThreads) {
        float w, g;
        if (F32) {
          w = static_cast<float*>(W)[e];
          g = static_cast<const float*>(G)[e];
        } else {
          w = muon::bf16_bits_to_float(static_cast<uint16_t*>(W)[e]);
          g = muon::bf16_bits_to_float(static_cast<const uint16_t*>(G)[e]);
        }
        float m = M[e], v = V[e];
        w = adamw_elem(p, w, g, m, v);
        M[e] = m;
        V[e] = v;
        if (F32) static_cast<float*>(W)[e] = w;
        else static_cast<uint16_t*>(W)[e] = muon::float_to_bf16_bits(w);
      }
    }
  }
}

}  // namespace

extern "C" muon_status muon_adamw_step(void* const* W, const void* const* G, float* const* m, float* const* v,
                                       const long long* numel, int count, int dtype,
                                       const muon_adamw_hparams* hp, void* stream) {
  if (!W || !G || !m || !v || !numel || !hp || count < 1 || count > MUON_MAX_BATCH) return MUON_ERR_INVALID_ARG;
  if (dtype != MUON_BF16 && dtype != MUON_F32) return MUON_ERR_DTYPE;
  if (!std::isfinite(hp->lr) || !std::isfinite(hp->beta1) || !std::isfinite(hp->beta2) ||
      !std::isfinite(hp->eps) || !std::isfinite(hp->weight_decay) || hp->step < 1 || hp->beta1 >= 1.f ||
      hp->beta2 >= 1.f || hp->eps < 0.f)
    return MUON_ERR_INVALID_ARG;
  AdamWParams p;
  std::memset(static_cast<void*>(&p), 0, sizeof(p));
  long long chunks = 0;
  for (int t = 0; t < count; ++t) {
    if (!W[t] || !G[t] || !m[t] || !v[t] || numel[t] < 1) return MUON_ERR_INVALID_ARG;
    p.w[t] = W[t];
    p.g[t] = G[t];
    p.m[t] = m[t];
    p.v[t] = v[t];
    p.numel[t] = numel[t];
    p.vec[t] = (reinterpret_cast<uintptr_t>(W[t]) | reinterpret_cast<uintptr_t>(G[t]) |
                reinterpret_cast<uintptr_t>(m[t]) | reinterpret_cast<uintptr_t>(v[t])) % 16 == 0;
    p.chunk_prefix[t] = static_cast<int>(chunks);
    chunks += (numel[t] + kChunk - 1) / kChunk;
    if (chunks > (1ll << 30)) return MUON_ERR_UNSUPPORTED_SHAPE;
  }
  p.chunk_prefix[count] = static_cast<int>(chunks);
  p.count = count;
  p.beta1 = hp->beta1;
  p.beta2 = hp->beta2;
  p.eps = hp->eps;
  p.decay = 1.0f - hp->lr * hp->weight_decay;
  const double bc1 = 1.0 - std::pow(static_cast<double>(hp->beta1), hp->step);
  const double bc2 = 1.0 - std::pow(static_cast<double>(hp->beta2), hp->step);
  p.step_size = static_cast<float>(hp->lr / bc1);
  p.inv_sqrt_bc2 = static_cast<float>(1.0 / std::sqrt(bc2));
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = static_cast<int>(chunks < 8LL * sms ? chunks : 8LL * sms);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == MUON_F32) adamw_kernel<true><<<grid, kThreads, 0, s>>>(p);
  else adamw_kernel<false><<<grid, kThreads, 0, s>>>(p);
  if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;
  return MUON_OK;
}
