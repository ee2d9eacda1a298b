// Allocation-free momentum / Nesterov / Frobenius-norm pass.
//
// Some callers cannot call cudaMalloc at all: code running inside a
// pre-allocated memory pool or a framework that owns every device allocation,
// allocator-free inference or training runtimes, and hooks that run while a
// CUDA graph is being captured.  muon_momentum_norm_noalloc serves them: it
// does what the momentum pass at the start of muon_step does for M and for
// ||U||_F, without a context and without allocating anything.  It does not
// materialise U.
//
// Its scratch (one fp32 partial sum per block and one arrival counter per
// matrix) lives in a file-scope __device__ array of kScratchBytes; every GPU
// that loads the library holds that array until the process exits.  Every
// call shares it and it keeps the last call's contents, so the counters are
// cleared at the start of each call, and calls that overlap on the GPU (two
// streams, or two host threads) race on it.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "../../include/muon.h"
#include "device_utils.cuh"

namespace {

constexpr size_t kScratchBytes = MUON_NOALLOC_SCRATCH_BYTES;
constexpr size_t kCounterBytes = sizeof(unsigned) * MUON_MAX_BATCH;
constexpr size_t kPartialCapacity = (kScratchBytes - kCounterBytes) / sizeof(float);
constexpr int kThreads = 256;
constexpr long long kElemsPerBlock = 8192;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

struct NoAllocParams {
  const void* g[MUON_MAX_BATCH];
  float* m[MUON_MAX_BATCH];
  float* nu;              // [batch], caller's device buffer
  unsigned* counters;     // scratch: [batch]
  float* partials;        // scratch: [batch][nblk]
  long long elems;        // rows * cols
  int nblk;
  float beta;
  int nesterov;
};

template <bool F32>
__device__ __forceinline__ float load_g(const void* g, long long e) {
  if (F32) return static_cast<const float*>(g)[e];
  return muon::bf16_bits_to_float(static_cast<const uint16_t*>(g)[e]);
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

// 8 consecutive elements of G (16-byte aligned bf16, or 32-byte aligned fp32) as floats.
template <bool F32>
__device__ __forceinline__ void load_g8(const void* g, long long e, float (&v)[8]) {
  if (F32) {
    const float4* q = reinterpret_cast<const float4*>(static_cast<const float*>(g) + e);
    const float4 a = __ldcs(q), b = __ldcs(q + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    const uint4 q = __ldcs(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(g) + e));
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

// grid (nblk, batch): block b of matrix l updates elements
// [b*chunk, (b+1)*chunk) of M and sums U^2; the last block of the matrix adds
// the partials in a fixed order (fp64) and writes ||U||_F.  VEC: rows*cols is a
// multiple of 8 and every pointer is 16-byte aligned, so each thread step moves
// 8 elements with 16-byte loads and stores (chunks are whole vectors).
template <bool F32, bool VEC>
__global__ void __launch_bounds__(kThreads) momentum_norm_noalloc_kernel(const __grid_constant__ NoAllocParams p) {
  __shared__ float fs[kThreads / 32];
  __shared__ double ds[kThreads / 32];
  __shared__ int is_last;
  const int l = blockIdx.y;
  const void* g = p.g[l];
  float* m = p.m[l];
  float ss = 0.f;
  if (VEC) {
    const long long nv = p.elems / 8;
    const long long chunk = (nv + p.nblk - 1) / p.nblk;
    const long long beg = chunk * blockIdx.x;
    const long long end = min(nv, beg + chunk);
    for (long long v = beg + threadIdx.x; v < end; v += kThreads) {
      const long long e = v * 8;
      float gv[8], mv[8];
      load_g8<F32>(g, e, gv);
      const float4* mq = reinterpret_cast<const float4*>(m + e);
      const float4 a = __ldcs(mq), b = __ldcs(mq + 1);
      mv[0] = a.x; mv[1] = a.y; mv[2] = a.z; mv[3] = a.w; mv[4] = b.x; mv[5] = b.y; mv[6] = b.z; mv[7] = b.w;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        mv[t] = fmaf(p.beta, mv[t], gv[t]);
        const float u = p.nesterov ? fmaf(p.beta, mv[t], gv[t]) : mv[t];
        ss = fmaf(u, u, ss);
      }
      float4* mo = reinterpret_cast<float4*>(m + e);
      __stcs(mo, make_float4(mv[0], mv[1], mv[2], mv[3]));
      __stcs(mo + 1, make_float4(mv[4], mv[5], mv[6], mv[7]));
    }
  } else {
    const long long chunk = (p.elems + p.nblk - 1) / p.nblk;
    const long long beg = chunk * blockIdx.x;
    const long long end = min(p.elems, beg + chunk);
    for (long long e = beg + threadIdx.x; e < end; e += kThreads) {
      const float gv = load_g<F32>(g, e);
      const float mn = fmaf(p.beta, m[e], gv);
      m[e] = mn;
      const float u = p.nesterov ? fmaf(p.beta, mn, gv) : mn;
      ss = fmaf(u, u, ss);
    }
  }
  const float blk = block_sum<float>(ss, fs);
  if (threadIdx.x == 0) {
    p.partials[static_cast<long long>(l) * p.nblk + blockIdx.x] = blk;
    __threadfence();
    is_last = atomicAdd(&p.counters[l], 1u) == static_cast<unsigned>(p.nblk) - 1u;
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  double acc = 0.0;
  for (int b = threadIdx.x; b < p.nblk; b += kThreads)
    acc += static_cast<double>(__ldcg(&p.partials[static_cast<long long>(l) * p.nblk + b]));
  const double tot = block_sum<double>(acc, ds);
  if (threadIdx.x == 0) p.nu[l] = static_cast<float>(sqrt(tot));
}

// Device address of the scratch array, looked up once per device and kept for the life of the
// process: it belongs to the device's context as it was at the lookup, so it must not be used
// after that context is destroyed (cudaDeviceReset).
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

cudaError_t scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" muon_status muon_momentum_norm_noalloc(const void* const* G, float* const* M, float* nu, int batch,
                                                  int rows, int cols, int dtype, float beta, int nesterov,
                                                  void* stream) {
  if (!G || !M || !nu || batch < 1 || batch > MUON_MAX_BATCH || rows < 1 || cols < 1) return MUON_ERR_INVALID_ARG;
  if (dtype != MUON_BF16 && dtype != MUON_F32) return MUON_ERR_DTYPE;
  if (!std::isfinite(beta)) return MUON_ERR_INVALID_ARG;
  for (int l = 0; l < batch; ++l)
    if (!G[l] || !M[l]) return MUON_ERR_INVALID_ARG;
  const long long elems = static_cast<long long>(rows) * cols;
  const long long nblk = (elems + kElemsPerBlock - 1) / kElemsPerBlock;
  if (nblk > 65535 || static_cast<unsigned long long>(nblk) * batch > kPartialCapacity)
    return MUON_ERR_UNSUPPORTED_SHAPE;  // the partial sums would not fit in the scratch array
  void* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess) {
    cudaGetLastError();
    return MUON_ERR_CUDA;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  NoAllocParams p;
  std::memset(static_cast<void*>(&p), 0, sizeof(p));
  for (int l = 0; l < batch; ++l) {
    p.g[l] = G[l];
    p.m[l] = M[l];
  }
  p.nu = nu;
  p.counters = static_cast<unsigned*>(scratch);
  p.partials = reinterpret_cast<float*>(static_cast<unsigned char*>(scratch) + kCounterBytes);
  p.elems = elems;
  p.nblk = static_cast<int>(nblk);
  p.beta = beta;
  p.nesterov = nesterov ? 1 : 0;
  // the previous call left its counters behind (or aborted midway): start from zero
  if (cudaMemsetAsync(p.counters, 0, sizeof(unsigned) * batch, s) != cudaSuccess) {
    cudaGetLastError();
    return MUON_ERR_CUDA;
  }
  bool vec = elems % 8 == 0;
  for (int l = 0; l < batch && vec; ++l)
    vec = reinterpret_cast<uintptr_t>(G[l]) % 16 == 0 && reinterpret_cast<uintptr_t>(M[l]) % 16 == 0;
  const dim3 grid(p.nblk, batch);
  if (dtype == MUON_F32) {
    if (vec) momentum_norm_noalloc_kernel<true, true><<<grid, kThreads, 0, s>>>(p);
    else momentum_norm_noalloc_kernel<true, false><<<grid, kThreads, 0, s>>>(p);
  } else {
    if (vec) momentum_norm_noalloc_kernel<false, true><<<grid, kThreads, 0, s>>>(p);
    else momentum_norm_noalloc_kernel<false, false><<<grid, kThreads, 0, s>>>(p);
  }
  if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;
  return MUON_OK;
}
