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
__device__ __forceinline__ void load_raw_smem(const uint8_t* row, int c, Raw8w<F32>& r) {
  const uint4* q = reinterpret_cast<const uint4*>(row + static_cast<size_t>(c) * (F32 ? 4 : 2));
#pragma unroll
  for (int i = 0; i < (F32 ? 2 : 1); ++i) r.q[i] = q[i];
}

// Where column c of v sits in the streaming pass's shared copy: within each 256-column chunk,
// the first four of every eight columns come first (128 values), the last four after them.
// Lane k's columns 8k..8k+7 of a chunk are then two 16-byte reads at 4k and 128 + 4k, which
// fall in distinct banks across each quarter warp.  The copy holds cols rounded up to 256.
__device__ __forceinline__ int vs_index(int c) {
  return (c & ~255) | ((c & 4) << 5) | (((c & 255) >> 3) << 2) | (c & 3);
}

// Packed pairs of fp32 values and the sm_100a two-lane FMA (each lane an ordinary fp32 fma,
// rounded to nearest): the streaming pass's dot products and z updates issue half the FMAs.
__device__ __forceinline__ uint64_t pack_f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ void unpack_f2(uint64_t r, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
}

__device__ __forceinline__ uint64_t fma_f2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// The 8 values of a packed 16-byte load as four (even, odd) column pairs.
template <bool F32>
__device__ __forceinline__ void raw_to_pairs(const Raw8w<F32>& r, uint64_t (&x)[4]) {
  if (F32) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      x[2 * i] = pack_f2(__uint_as_float(r.q[i].x), __uint_as_float(r.q[i].y));
      x[2 * i + 1] = pack_f2(__uint_as_float(r.q[i].z), __uint_as_float(r.q[i].w));
    }
  } else {
    const uint32_t w[4] = {r.q[0].x, r.q[0].y, r.q[0].z, r.q[0].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = pack_f2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
  }
}

// Two rows at once (the second when has1), both read from their shared-memory stage:
// t = W[r, :] . v for each, then z += t W[r, :], on (even, odd) column pairs.  Each dot product
// runs as two pair chains (the first and last four columns of every eight); the two rows' chains
// and shuffle trees interleave.  The z update reads the stage again rather than hold the rows'
// pairs across the trees (within the 96 registers two blocks per SM leave).  FULL: cols is
// exactly 256 * NV, so no column needs a bound check.
template <bool F32, int NV, bool FULL>
__device__ __forceinline__ void power_rows2(const uint8_t* row0, const uint8_t* row1, bool has1, const float* vs,
                                            int C, int lane, uint64_t (&z)[NV][4], float& t0, float& t1) {
  uint64_t a0 = 0, b0 = 0, a1 = 0, b1 = 0;  // (+0.0f, +0.0f) pairs
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = 8 * lane + 256 * i;
    if (FULL || c < C) {
      const ulonglong2 lo = *reinterpret_cast<const ulonglong2*>(vs + 256 * i + 4 * lane);
      const ulonglong2 hi = *reinterpret_cast<const ulonglong2*>(vs + 256 * i + 128 + 4 * lane);
      Raw8w<F32> w;
      uint64_t x[4];
      load_raw_smem<F32>(row0, c, w);
      raw_to_pairs<F32>(w, x);
      a0 = fma_f2(x[0], lo.x, a0);
      a0 = fma_f2(x[1], lo.y, a0);
      b0 = fma_f2(x[2], hi.x, b0);
      b0 = fma_f2(x[3], hi.y, b0);
      if (has1) {
        load_raw_smem<F32>(row1, c, w);
        raw_to_pairs<F32>(w, x);
        a1 = fma_f2(x[0], lo.x, a1);
        a1 = fma_f2(x[1], lo.y, a1);
        b1 = fma_f2(x[2], hi.x, b1);
        b1 = fma_f2(x[3], hi.y, b1);
      }
    }
  }
  float p, q, r, s;
  unpack_f2(a0, p, q);
  unpack_f2(b0, r, s);
  float d0 = (p + q) + (r + s);
  unpack_f2(a1, p, q);
  unpack_f2(b1, r, s);
  float d1 = (p + q) + (r + s);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    d0 += __shfl_xor_sync(0xffffffffu, d0, o);
    d1 += __shfl_xor_sync(0xffffffffu, d1, o);
  }
  const uint64_t dd0 = pack_f2(d0, d0), dd1 = pack_f2(d1, d1);
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = 8 * lane + 256 * i;
    if (FULL || c < C) {
      uint64_t x[4];
      Raw8w<F32> w;
      load_raw_smem<F32>(row0, c, w);
      raw_to_pairs<F32>(w, x);
#pragma unroll
      for (int k = 0; k < 4; ++k) z[i][k] = fma_f2(dd0, x[k], z[i][k]);
      if (has1) {
        load_raw_smem<F32>(row1, c, w);
        raw_to_pairs<F32>(w, x);
#pragma unroll
        for (int k = 0; k < 4; ++k) z[i][k] = fma_f2(dd1, x[k], z[i][k]);
      }
    }
  }
  t0 = d0;
  t1 = d1;
}

// z[k] = sum over b = 0, 1, ... (in that order) of part[b][c_k], c_k = tid + k * nthr (zero past
// cols; at most 8 columns per thread): every column of this thread at once, six partials per
// round, so the loads overlap.
__device__ __forceinline__ void sum_partials(const float* part, int nblk, int C, int tid, int nthr, float (&z)[8]) {
#pragma unroll
  for (int k = 0; k < 8; ++k) z[k] = 0.f;
  // partials in rounds of six (the loads of a round in flight together), added in block order
  constexpr int kRound = 6;
  for (int b = 0; b < nblk; b += kRound) {
    float q[8][kRound];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int c = tid + k * nthr;
#pragma unroll
      for (int j = 0; j < kRound; ++j)
        q[k][j] = c < C && b + j < nblk ? __ldcg(part + static_cast<long long>(b + j) * C + c) : 0.f;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k)
#pragma unroll
      for (int j = 0; j < kRound; ++j)
        if (b + j < nblk) z[k] += q[k][j];
  }
}

// Sum of squares of this thread's columns over the first nwarps warps, in a fixed order;
// every participating thread gets it.  `bar` synchronises exactly those warps.
template <typename Bar>
__device__ __forceinline__ double sum_squares(const float (&z)[8], double* scratch, int nwarps, Bar&& bar) {
  double ss = 0.0;
#pragma unroll
  for (int k = 0; k < 8; ++k) ss += static_cast<double>(z[k]) * z[k];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = ss;
  bar();
  double tot = 0.0;
  for (int k = 0; k < nwarps; ++k) tot += scratch[k];
  return tot;
}

// One pass over the rows of W per power iteration.  With t = W v, the next W^T u is
// W^T t / |t|, and W^T t = sum_r t_r W[r, :], so a row read once gives both its t_r and its
// share of z = W^T t.  A block owns rows_per_block consecutive rows of one matrix: a producer
// warp streams them through a ring of shared-memory stages (eight consecutive rows, one 1-D
// bulk copy, per stage), and each of the eight consumer warps takes one row of each of two
// stages at a time, forms t_r against v (staged in shared memory) and adds t_r W[r, :] to its
// running z.  The warps' z are summed in warp order into one partial per block, which also
// records its sum of t_r^2: where the final step's stages can hold all eight warps' z (two
// stages of bf16 rows, one of fp32 rows), the consumers keep those stages from the producer,
// each warp writes its z there and all consumer threads add them up at once; otherwise the
// warps add into one buffer one after another.
//
// One launch runs iterations it0 .. it1-1.  Iteration it > 0 starts from the previous
// iteration's partials, which every block sums in block order (z, then v = z / |z|); within a
// launch a block first waits (bounded) until all blocks of its matrix have written them (a
// per-matrix counter), which needs the launch's blocks co-resident (a cooperative launch).
// The producer does not wait: W does not change, so it streams the next iteration's rows while
// the consumers wait.  Iteration 0 takes the caller's v as it is (u and the next v do not depend
// on its scale).  After the last iteration, the last block of a matrix to finish writes
// v = z / |z|, u = t / |t| and sigma = |z| / |t| = |W^T u|.  A zero t leaves u, v at zero and
// sigma 0.  Requires cols % 8 == 0, 16-byte aligned W and cols <= 256 * NV <= 2048.
//
// With `shift` set (the smallest singular value of a tall W, whose wide view is X = W^T, so
// X X^T y = W^T W y = z), the same passes run the shifted iteration: pass 0 takes y = v / |v|,
// pass k > 0 takes y <- (s y - z) / |s y - z| with s = shift[l]^2 and z from pass k-1 (y, the
// previous pass's v, is still in every block's shared memory), and after the last pass the
// last block writes y to v and sigma[l] = |X^T y| = |W y| = |t|.  All passes of such a call run
// in one launch.
constexpr int kPowerWarps = 8;                         // consumer warps: a stage holds a row for each
constexpr int kPowerThreads = 32 * (kPowerWarps + 1);  // and one producer warp
constexpr int kPowerMaxBlocks = 64;                    // block partials per matrix
constexpr int kPowerCols = 8;                          // columns per thread in the partial sums
constexpr uint64_t kPowerDrainNs = 200000000ull;

struct PowerArgs {
  int rows_per_block, stages, nblk, iters;  // iters: of the whole call
  int it0, it1;                             // the iterations this launch runs
  const float* shift;  // [batch] sigma_max for the shifted iteration, or null for the power iteration
  float* part[2];      // [batch][nblk][cols] each: z partials of even / odd iterations
  float* tsq_partial;  // [batch][nblk]: each block's sum of t_r^2 (last iteration written)
  unsigned* sync;      // [batch]: partial sets written in this call (blocks x iterations)
  unsigned* done;      // [batch]: blocks through the final iteration
  float* sigma;        // [batch], written after the final iteration
  int* status;         // device status word (wait timeouts)
};

// Two blocks per SM where z's registers allow it (rows up to 1280 columns, bf16 up to 1536).
template <bool F32, int NV>
__global__ void __launch_bounds__(kPowerThreads, (NV <= 5 || (!F32 && NV <= 6)) ? 2 : 1) power_stream_kernel(
    const __grid_constant__ GemvParams p, const PowerArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float tq[kPowerWarps];
  __shared__ double sq[kPowerWarps + 1];
  __shared__ float s_tt;
  __shared__ int s_last;
  __shared__ volatile int abort_flag;
  constexpr int kConsumers = 32 * kPowerWarps;
  const int C = p.cols;
  const int Cr = (C + 255) & ~255;
  const uint32_t row_bytes = static_cast<uint32_t>(C) * (F32 ? 4u : 2u);
  const uint32_t stage_bytes = kPowerWarps * row_bytes;
  uint8_t* ring = smem;
  float* vs = reinterpret_cast<float*>(smem + static_cast<size_t>(a.stages) * stage_bytes);  // [Cr], permuted
  float* zs = vs + Cr;                                                                         // [C]
  const uint32_t bar0 = smem_addr(zs + C);  // full[stages], then empty[stages]
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (a.stages + s); };
  const int l = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r_beg = blockIdx.x * a.rows_per_block;
  const int r_end = min(p.rows, r_beg + a.rows_per_block);
  const int nst = (r_end - r_beg + kPowerWarps - 1) / kPowerWarps;
  // The final step (stages jl and jl + 1) holds the warps' z when its stages have room for them:
  // held_j is jl then, else -1.
  const int held_j = ((nst - 1) & ~1) + 1 < nst || F32 ? (nst - 1) & ~1 : -1;
  auto part_set = [&](int it) { return (it & 1) ? a.part[1] : a.part[0]; };
  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), kPowerWarps);
    }
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const int niter = a.it1 - a.it0;
  if (warp == kPowerWarps) {
    // ------------------------------------------------ producer (one thread): every iteration's rows
    if (lane == 0) {
      const uint8_t* src = static_cast<const uint8_t*>(p.w[l]) + static_cast<size_t>(r_beg) * row_bytes;
      const int total = niter * nst;
      int g = 0;
      for (; g < total; ++g) {
        const int s = g % a.stages;
        const int j = g % nst;
        if (g >= a.stages &&
            !mbar_wait_bounded(empty_bar(s), static_cast<uint32_t>((g / a.stages) - 1) & 1u, &abort_flag, a.status))
          break;
        const int nr = min(kPowerWarps, r_end - (r_beg + kPowerWarps * j));
        const uint32_t bytes = static_cast<uint32_t>(nr) * row_bytes;
        mbar_arrive_expect_tx(full_bar(s), bytes);
        bulk_load_1d(smem_addr(ring + static_cast<size_t>(s) * stage_bytes), src + static_cast<size_t>(j) * stage_bytes,
                     bytes, full_bar(s));
      }
      if (g < total) {
        // gave up: let the copies in flight land before the block exits
        const int n = min(g, a.stages);
        for (int k = g - n; k < g; ++k) {
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(full_bar(k % a.stages), static_cast<uint32_t>(k / a.stages) & 1u))
            if (global_timer_ns() - t0 > kPowerDrainNs) break;
        }
      }
    }
  } else {
    // ------------------------------------------------ consumers
    for (int it = a.it0; it < a.it1; ++it) {
      // v for this iteration
      if (it == 0 && a.shift == nullptr) {
        const float* x = p.x[l];
        for (int c = threadIdx.x; c < C; c += kConsumers) vs[vs_index(c)] = x[c];
      } else {
        if (it > a.it0) {
          // the previous iteration's partials of this matrix, written by this launch's blocks
          if (threadIdx.x == 0 && !abort_flag &&
              !wait_counter_bounded(a.sync + l, static_cast<unsigned>(a.nblk * (it - a.it0)), &abort_flag, a.status))
            abort_flag = 1;
          named_barrier_sync(1, kConsumers);
        }
        float zc[kPowerCols];
        if (it == 0) {
          // the shifted iteration starts from the caller's vector, normalised
          const float* x = p.x[l];
#pragma unroll
          for (int k = 0; k < kPowerCols; ++k) {
            const int c = threadIdx.x + k * kConsumers;
            zc[k] = c < C ? x[c] : 0.f;
          }
        } else {
          sum_partials(part_set(it - 1) + static_cast<long long>(l) * a.nblk * C, a.nblk, C, threadIdx.x,
                       kConsumers, zc);
          if (a.shift != nullptr) {
            // s y - z, y the previous pass's v (each thread reads and rewrites only its columns)
            const float s2 = a.shift[l] * a.shift[l];
#pragma unroll
            for (int k = 0; k < kPowerCols; ++k) {
              const int c = threadIdx.x + k * kConsumers;
              if (c < C) zc[k] = fmaf(s2, vs[vs_index(c)], -zc[k]);
            }
          }
        }
        const double ss = sum_squares(zc, sq, kPowerWarps, [] { named_barrier_sync(1, kConsumers); });
        const float nz = static_cast<float>(sqrt(ss));
        const float inv = nz > 0.f ? 1.0f / nz : 0.f;
#pragma unroll
        for (int k = 0; k < kPowerCols; ++k) {
          const int c = threadIdx.x + k * kConsumers;
          if (c < C) vs[vs_index(c)] = zc[k] * inv;
        }
      }
      named_barrier_sync(1, kConsumers);
      uint64_t z[NV][4];  // (even, odd) column pairs of this lane's running W^T t
#pragma unroll
      for (int i = 0; i < NV; ++i)
#pragma unroll
        for (int k = 0; k < 4; ++k) z[i][k] = 0;
      float tsq = 0.f;
      const int gbase = (it - a.it0) * nst;
      // After a failed wait (the status word says so) a warp skips the rest of its rows, but every
      // consumer warp still takes the same named barriers below, so none of them is left waiting.
      for (int j = 0; j < nst && !abort_flag; j += 2) {
        const bool two = j + 1 < nst;
        const int g0 = gbase + j, g1 = g0 + 1;
        const int s0 = g0 % a.stages, s1 = g1 % a.stages;
        if (!mbar_wait_bounded(full_bar(s0), static_cast<uint32_t>(g0 / a.stages) & 1u, &abort_flag, a.status) ||
            (two && !mbar_wait_bounded(full_bar(s1), static_cast<uint32_t>(g1 / a.stages) & 1u, &abort_flag,
                                       a.status)))
          break;
        const int r0 = r_beg + kPowerWarps * j + warp, r1 = r0 + kPowerWarps;
        const bool has1 = two && r1 < r_end;
        if (r0 < r_end) {
          const uint8_t* row0 = ring + static_cast<size_t>(s0) * stage_bytes + static_cast<size_t>(warp) * row_bytes;
          const uint8_t* row1 = ring + static_cast<size_t>(s1) * stage_bytes + static_cast<size_t>(warp) * row_bytes;
          float t0, t1;
          // rows of exactly 256 * NV columns up to 768 run without bound checks (measured faster
          // there; wider rows keep them, which measured faster for 1536 columns and leaves 1024
          // free of register spills)
          if (NV <= 3 && C == 256 * NV)
            power_rows2<F32, NV, true>(row0, row1, has1, vs, C, lane, z, t0, t1);
          else
            power_rows2<F32, NV, false>(row0, row1, has1, vs, C, lane, z, t0, t1);
          if (lane == 0) {
            p.y[l][r0] = t0;
            if (has1) p.y[l][r1] = t1;
          }
          tsq = fmaf(t0, t0, tsq);
          if (has1) tsq = fmaf(t1, t1, tsq);
        }
        __syncwarp();
        if (lane == 0 && j != held_j) {
          mbar_arrive(empty_bar(s0));
          if (two) mbar_arrive(empty_bar(s1));
        }
      }
      // the block's partial of this iteration: the warps' z added in warp order
      float* part = part_set(it) + (static_cast<long long>(l) * a.nblk + blockIdx.x) * C;
      if (held_j >= 0) {
        // once every warp has read its rows of the held stages, each warp's z goes there (warp w at
        // slot w % wps of stage held_j + w / wps) ...
        const int wps = F32 ? kPowerWarps : kPowerWarps / 2;  // warps' z per stage (8 C floats per two bf16 stages)
        const int gl = gbase + held_j;
        named_barrier_sync(1, kConsumers);
        const int sw = (warp < wps ? gl : gl + 1) % a.stages;
        float* zw = reinterpret_cast<float*>(ring + static_cast<size_t>(sw) * stage_bytes) + (warp % wps) * C;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
          const int c = 8 * lane + 256 * i;
          if (c < C) {
            ulonglong2* d = reinterpret_cast<ulonglong2*>(zw + c);
            d[0] = make_ulonglong2(z[i][0], z[i][1]);
            d[1] = make_ulonglong2(z[i][2], z[i][3]);
          }
        }
        if (lane == 0) tq[warp] = tsq;
        named_barrier_sync(1, kConsumers);
        // ... then every consumer thread adds eight columns of the eight warps' z
        const float* z0 = reinterpret_cast<const float*>(ring + static_cast<size_t>(gl % a.stages) * stage_bytes);
        const float* z1 = reinterpret_cast<const float*>(ring + static_cast<size_t>((gl + 1) % a.stages) * stage_bytes);
        for (int c = 8 * threadIdx.x; c < C; c += 8 * kConsumers) {
          float4 lo = *reinterpret_cast<const float4*>(z0 + c), hi = *reinterpret_cast<const float4*>(z0 + c + 4);
#pragma unroll
          for (int w = 1; w < kPowerWarps; ++w) {
            const float* src = (w < wps ? z0 : z1) + (w % wps) * C + c;
            const float4 e = *reinterpret_cast<const float4*>(src), f = *reinterpret_cast<const float4*>(src + 4);
            lo = make_float4(lo.x + e.x, lo.y + e.y, lo.z + e.z, lo.w + e.w);
            hi = make_float4(hi.x + f.x, hi.y + f.y, hi.z + f.z, hi.w + f.w);
          }
          *reinterpret_cast<float4*>(part + c) = lo;
          *reinterpret_cast<float4*>(part + c + 4) = hi;
        }
        // these generic accesses come before the producer's next bulk copies into the stages
        fence_proxy_async_smem();
      } else {
        // the warps' z added into zs one warp after another
        for (int w = 0; w < kPowerWarps; ++w) {
          if (warp == w) {
#pragma unroll
            for (int i = 0; i < NV; ++i) {
              const int c = 8 * lane + 256 * i;
              if (c < C) {
                ulonglong2* d = reinterpret_cast<ulonglong2*>(zs + c);
                if (w == 0) {
                  d[0] = make_ulonglong2(z[i][0], z[i][1]);
                  d[1] = make_ulonglong2(z[i][2], z[i][3]);
                } else {
                  const ulonglong2 e0 = d[0], e1 = d[1];
                  const uint64_t one = pack_f2(1.0f, 1.0f);
                  d[0] = make_ulonglong2(fma_f2(e0.x, one, z[i][0]), fma_f2(e0.y, one, z[i][1]));
                  d[1] = make_ulonglong2(fma_f2(e1.x, one, z[i][2]), fma_f2(e1.y, one, z[i][3]));
                }
              }
            }
            if (lane == 0) tq[w] = tsq;
          }
          named_barrier_sync(1, kConsumers);
        }
        for (int c = threadIdx.x; c < C; c += kConsumers) part[c] = zs[c];
      }
      if (threadIdx.x == 0) {
        float acc = 0.f;
#pragma unroll
        for (int k = 0; k < kPowerWarps; ++k) acc += tq[k];
        a.tsq_partial[static_cast<long long>(l) * a.nblk + blockIdx.x] = acc;
      }
      // Every store of the set is done (and zs or the held stages are free again).  Thread 0's
      // release after this barrier publishes the whole block's stores (release is cumulative).
      named_barrier_sync(1, kConsumers);
      if (held_j >= 0 && lane == 0) {
        const int gl = gbase + held_j;
        mbar_arrive(empty_bar(gl % a.stages));
        if (held_j + 1 < nst) mbar_arrive(empty_bar((gl + 1) % a.stages));
      }
      if (threadIdx.x == 0) red_release_gpu_add(a.sync + l, 1u);
    }
  }
  if (a.it1 < a.iters) return;
  // after the final iteration: the last block of this matrix to get here writes u, v and sigma
  // (thread 0's fence after the barrier orders the block's stores of u, the partials and t^2
  // before its count, for the last block's reads after its own count and fence)
  __syncthreads();
  if (abort_flag) return;
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(a.done + l, 1u) == static_cast<unsigned>(a.nblk - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (a.shift != nullptr) {
    // y is this block's v of the last pass (every block holds the same); sigma_min = |W y|
    float* y = const_cast<float*>(p.x[l]);
    for (int c = threadIdx.x; c < C; c += kPowerThreads) y[c] = vs[vs_index(c)];
    if (warp == 0) {
      const double tt = warp_sum_partials(a.tsq_partial + static_cast<long long>(l) * a.nblk, a.nblk, lane);
      if (lane == 0) a.sigma[l] = static_cast<float>(sqrt(tt));
    }
    return;
  }
  float zc[kPowerCols];
  sum_partials(part_set(a.iters - 1) + static_cast<long long>(l) * a.nblk * C, a.nblk, C, threadIdx.x,
               kPowerThreads, zc);
  if (warp == 0) {
    const double tt = warp_sum_partials(a.tsq_partial + static_cast<long long>(l) * a.nblk, a.nblk, lane);
    if (lane == 0) s_tt = static_cast<float>(sqrt(tt));
  }
  const double zz = sum_squares(zc, sq, kPowerWarps + 1, [] { __syncthreads(); });
  const float nz = static_cast<float>(sqrt(zz));
  const float inv_z = nz > 0.f ? 1.0f / nz : 0.f;
  float* v = const_cast<float*>(p.x[l]);
#pragma unroll
  for (int k = 0; k < kPowerCols; ++k) {
    const int c = threadIdx.x + k * kPowerThreads;
    if (c < C) v[c] = zc[k] * inv_z;
  }
  const float nt = s_tt;
  const float inv_t = nt > 0.f ? 1.0f / nt : 0.f;
  float* u = p.y[l];
  for (int r = threadIdx.x; r < p.rows; r += kPowerThreads) u[r] = __ldcg(u + r) * inv_t;
  if (threadIdx.x == 0) a.sigma[l] = nt > 0.f ? nz / nt : 0.f;
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
// A block takes kCapRows rows, kCapRowsPerWarp per warp at once; b is staged in shared memory
// once per block in the layout whose 16-byte reads of a lane's 8 columns are bank-conflict
// free (vs_index), and each lane reads 16-byte vectors of every plane of its warp's rows
// (the wide pitch is a multiple of 64 elements, so row starts are 128-byte aligned), two
// column chunks ahead, and the ragged tail element by element.  The block's partial is
// sum over its rows (in order) of a_i (O_i . b), the row dots by a fixed xor tree.
constexpr int kCapRowsPerWarp = 4;
constexpr int kCapRows = kCapRowsPerWarp * (kThreads / 32);

template <int PLANES>
__global__ void __launch_bounds__(kThreads) cap_alpha_partial_kernel(const __grid_constant__ CapParams p) {
  extern __shared__ __align__(16) float bs[];  // [round_up(n, 256)], vs_index layout
  __shared__ double wsum[kThreads / 32];
  const int l = blockIdx.y;
  const float* a = p.a[l];
  const float* b = p.b[l];
  const int n = p.n;
  const int nr = (n + 255) & ~255;
  for (int c = threadIdx.x; c < nr; c += kThreads) bs[vs_index(c)] = c < n ? b[c] : 0.f;
  __syncthreads();
  const uint16_t* o = p.o + static_cast<long long>(l) * p.o_mat;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = blockIdx.x * kCapRows + warp * kCapRowsPerWarp;
  const int nv = n & ~7;  // whole 8-column chunks
  float s[kCapRowsPerWarp];
#pragma unroll
  for (int k = 0; k < kCapRowsPerWarp; ++k) s[k] = 0.f;
  auto chunk = [&](int j, float (&acc)[kCapRowsPerWarp]) {
    // this lane's 8 columns j..j+7 of the warp's rows, every plane summed, against b; all the
    // rows' and planes' 16-byte loads are issued before any is used
    uint4 w[kCapRowsPerWarp][PLANES];
#pragma unroll
    for (int k = 0; k < kCapRowsPerWarp; ++k)
#pragma unroll
      for (int q = 0; q < PLANES; ++q)
        w[k][q] = r0 + k < p.m ? __ldcs(reinterpret_cast<const uint4*>(o + q * p.o_plane +
                                                                      static_cast<long long>(r0 + k) * p.pitch + j))
                               : make_uint4(0u, 0u, 0u, 0u);
    const int i = j >> 8, ln = (j & 255) >> 3;
    const float4 lo = *reinterpret_cast<const float4*>(bs + 256 * i + 4 * ln);
    const float4 hi = *reinterpret_cast<const float4*>(bs + 256 * i + 128 + 4 * ln);
    const float bb[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
    for (int k = 0; k < kCapRowsPerWarp; ++k) {
      float v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
      for (int q = 0; q < PLANES; ++q) {
        const uint32_t u[4] = {w[k][q].x, w[k][q].y, w[k][q].z, w[k][q].w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          v[2 * t] += __uint_as_float(u[t] << 16);
          v[2 * t + 1] += __uint_as_float(u[t] & 0xFFFF0000u);
        }
      }
#pragma unroll
      for (int t = 0; t < 8; ++t) acc[k] = fmaf(v[t], bb[t], acc[k]);
    }
  };
  int j = lane * 8;
  for (; j + 256 < nv; j += 512) {
    chunk(j, s);
    chunk(j + 256, s);
  }
  for (; j < nv; j += 256) chunk(j, s);
  for (int jj = nv + lane; jj < n; jj += 32) {
#pragma unroll
    for (int k = 0; k < kCapRowsPerWarp; ++k) {
      const int r = r0 + k;
      if (r >= p.m) continue;
      float v = 0.f;
#pragma unroll
      for (int q = 0; q < PLANES; ++q)
        v += bf16_bits_to_float(o[q * p.o_plane + static_cast<long long>(r) * p.pitch + jj]);
      s[k] = fmaf(v, bs[vs_index(jj)], s[k]);
    }
  }
  double acc = 0.0;
#pragma unroll
  for (int k = 0; k < kCapRowsPerWarp; ++k) {
    float d = s[k];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
    if (r0 + k < p.m) acc += static_cast<double>(d) * a[r0 + k];
  }
  if (lane == 0) wsum[warp] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) t += wsum[w];
    p.partial[static_cast<long long>(l) * gridDim.x + blockIdx.x] = t;
  }
}

__global__ void cap_alpha_reduce_kernel(const double* partial, int nblk, float* alpha) {
  if (threadIdx.x != 0) return;
  double s = 0.0;
  for (int k = 0; k < nblk; ++k) s += partial[static_cast<long long>(blockIdx.x) * nblk + k];
  alpha[blockIdx.x] = static_cast<float>(s);
}

// ------------------------------------------------------------------ shifted iteration, wide W
// For a wide W (rows <= cols) the wide view is X = W, so X X^T y = W (W^T y): a pass needs
// W^T y before W (W^T y).  A block owns a slab of S columns of one matrix (every row): phase 1
// streams the slab from HBM and forms d = W[:, slab]^T y (S values, lanes across the columns,
// a fixed xor tree over the rows a warp covers, then a warp-ordered sum) and |d|^2; phase 2
// reads the slab again (just read, so from L2) with a thread per row, adding W[r, slab] d into
// this slab's partial of z = W d.  The next pass's blocks sum the partials in slab order and take
// y <- (s y - z) / |s y - z| (s = shift[l]^2), once a per-matrix counter says every slab of the
// matrix has written them; the blocks wait on one another, so all passes run in one
// cooperative launch.  Pass 0 takes y = v / |v| from the caller's v.  The last pass skips
// phase 2, and the last block of a matrix to finish writes y to v and
// sigma[l] = |X^T y| = sqrt(sum over slabs of |d|^2).  Deterministic: every sum has a fixed order.
constexpr int kSlabRowsMax = 4096;  // y is kept in shared memory
constexpr int kSlabUnroll = 8;      // rows in flight per lane in phase 1

struct SlabArgs {
  int nslab, passes;
  const float* shift;  // [batch] sigma_max
  float* part[2];      // [batch][nslab][rows]: z partials of even / odd passes
  float* dsq;          // [batch][nslab]: |d|^2 of the last pass
  unsigned* sync;      // [batch]: slabs of this call that have written their partials
  unsigned* done;      // [batch]: slabs through the last pass
  float* sigma;        // [batch]
  int* status;
};

// Fixed-order sum of one value per thread over the whole block (every thread gets it).
__device__ __forceinline__ double block_total(double v, double* scratch) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = v;
  __syncthreads();
  double t = 0.0;
  for (int k = 0; k < kThreads / 32; ++k) t += scratch[k];
  return t;
}

template <bool F32, int S>
__global__ void __launch_bounds__(kThreads, 2) colslab_kernel(const __grid_constant__ GemvParams p, const SlabArgs a) {
  constexpr int LPR = S / 8;            // lanes per row in phase 1 (8 columns each)
  constexpr int RPW = 32 / LPR;         // rows a warp covers per load
  constexpr int kWarps = kThreads / 32;
  __shared__ float ys[kSlabRowsMax];
  __shared__ float dred[kWarps][S];
  __shared__ float ds[S];
  __shared__ double scratch[kWarps];
  __shared__ int s_last;
  __shared__ volatile int abort_flag;
  const int l = blockIdx.y, slab = blockIdx.x;
  const int R = p.rows, C = p.cols;
  const int c0 = slab * S;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rg = lane / LPR, k = lane % LPR;
  const char* W = static_cast<const char*>(p.w[l]);
  constexpr int ES = F32 ? 4 : 2;
  if (threadIdx.x == 0) abort_flag = 0;
  for (int pass = 0; pass < a.passes; ++pass) {
    // y for this pass
    {
      double ss = 0.0;
      if (pass == 0) {
        for (int r = threadIdx.x; r < R; r += kThreads) {
          const float v = p.x[l][r];
          ys[r] = v;
          ss += static_cast<double>(v) * v;
        }
      } else {
        if (threadIdx.x == 0 && !abort_flag &&
            !wait_counter_bounded(a.sync + l, static_cast<unsigned>(a.nslab * pass), &abort_flag, a.status))
          abort_flag = 1;
        __syncthreads();
        const float* pp = a.part[(pass - 1) & 1] + static_cast<long long>(l) * a.nslab * R;
        const float s2 = a.shift[l] * a.shift[l];
        for (int r = threadIdx.x; r < R; r += kThreads) {
          // the slabs' partials in slab order, eight loads in flight at a time
          float z = 0.f;
          for (int b = 0; b < a.nslab; b += 8) {
            float q[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) q[j] = b + j < a.nslab ? __ldcg(pp + static_cast<long long>(b + j) * R + r) : 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j)
              if (b + j < a.nslab) z += q[j];
          }
          const float v = fmaf(s2, ys[r], -z);
          ys[r] = v;
          ss += static_cast<double>(v) * v;
        }
      }
      const double tot = block_total(ss, scratch);
      const float nrm = static_cast<float>(sqrt(tot));
      const float inv = nrm > 0.f ? 1.0f / nrm : 0.f;
      for (int r = threadIdx.x; r < R; r += kThreads) ys[r] *= inv;
      __syncthreads();
    }
    // phase 1: d = W[:, slab]^T y, rows in strides of (warps x RPW), kSlabUnroll loads in flight
    float acc[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) acc[t] = 0.f;
    const int rstride = kWarps * RPW;
    for (int r0 = warp * RPW + rg; r0 < R && !abort_flag; r0 += rstride * kSlabUnroll) {
      uint4 raw[kSlabUnroll][F32 ? 2 : 1];
#pragma unroll
      for (int u = 0; u < kSlabUnroll; ++u) {
        const int r = r0 + u * rstride;
        if (r < R) {
          const uint4* src = reinterpret_cast<const uint4*>(W + (static_cast<long long>(r) * C + c0 + 8 * k) * ES);
#pragma unroll
          for (int h = 0; h < (F32 ? 2 : 1); ++h) raw[u][h] = __ldcs(src + h);
        }
      }
#pragma unroll
      for (int u = 0; u < kSlabUnroll; ++u) {
        const int r = r0 + u * rstride;
        if (r < R) {
          const float yr = ys[r];
          float x[8];
          if (F32) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              x[4 * h] = __uint_as_float(raw[u][h].x);
              x[4 * h + 1] = __uint_as_float(raw[u][h].y);
              x[4 * h + 2] = __uint_as_float(raw[u][h].z);
              x[4 * h + 3] = __uint_as_float(raw[u][h].w);
            }
          } else {
            const uint32_t w4[4] = {raw[u][0].x, raw[u][0].y, raw[u][0].z, raw[u][0].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              x[2 * i] = __uint_as_float(w4[i] << 16);
              x[2 * i + 1] = __uint_as_float(w4[i] & 0xFFFF0000u);
            }
          }
#pragma unroll
          for (int t = 0; t < 8; ++t) acc[t] = fmaf(x[t], yr, acc[t]);
        }
      }
    }
    // the rows this warp covered: xor tree over the row groups, then warps in order
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
      for (int t = 0; t < 8; ++t) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
    if (rg == 0)
#pragma unroll
      for (int t = 0; t < 8; ++t) dred[warp][8 * k + t] = acc[t];
    __syncthreads();
    double dd = 0.0;
    for (int j = threadIdx.x; j < S; j += kThreads) {
      float d = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) d += dred[w][j];
      ds[j] = d;
      dd += static_cast<double>(d) * d;
    }
    const double dtot = block_total(dd, scratch);  // also orders ds before phase 2
    if (pass == a.passes - 1) {
      if (threadIdx.x == 0) a.dsq[static_cast<long long>(l) * a.nslab + slab] = static_cast<float>(dtot);
      break;
    }
    // phase 2: this slab's share of z = W d, laid out like phase 1 (a row's columns over LPR
    // lanes, 8 each, coalesced 16-byte loads, U2 rows in flight per lane: half as many for fp32
    // rows, whose 8 columns take two loads); each row's lane products are added by an xor tree
    // inside its row group.  The loop runs warp-uniform (rows past R contribute zeros) so that
    // every lane takes part in the shuffles.
    constexpr int U2 = F32 ? kSlabUnroll / 2 : kSlabUnroll;
    float* part = a.part[pass & 1] + (static_cast<long long>(l) * a.nslab + slab) * R;
    float dk[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) dk[t] = ds[8 * k + t];
    for (int rb = warp * RPW; rb < R && !abort_flag; rb += rstride * U2) {
      uint4 raw[U2][F32 ? 2 : 1];
#pragma unroll
      for (int u = 0; u < U2; ++u) {
        const int r = rb + rg + u * rstride;
        if (r < R) {
          const uint4* src = reinterpret_cast<const uint4*>(W + (static_cast<long long>(r) * C + c0 + 8 * k) * ES);
#pragma unroll
          for (int h = 0; h < (F32 ? 2 : 1); ++h) raw[u][h] = __ldcg(src + h);
        } else {
#pragma unroll
          for (int h = 0; h < (F32 ? 2 : 1); ++h) raw[u][h] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
#pragma unroll
      for (int u = 0; u < U2; ++u) {
        float x[8];
        if (F32) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            x[4 * h] = __uint_as_float(raw[u][h].x);
            x[4 * h + 1] = __uint_as_float(raw[u][h].y);
            x[4 * h + 2] = __uint_as_float(raw[u][h].z);
            x[4 * h + 3] = __uint_as_float(raw[u][h].w);
          }
        } else {
          const uint32_t w4[4] = {raw[u][0].x, raw[u][0].y, raw[u][0].z, raw[u][0].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            x[2 * i] = __uint_as_float(w4[i] << 16);
            x[2 * i + 1] = __uint_as_float(w4[i] & 0xFFFF0000u);
          }
        }
        float zz = 0.f;
#pragma unroll
        for (int t = 0; t < 8; ++t) zz = fmaf(x[t], dk[t], zz);
#pragma unroll
        for (int o = 1; o < LPR; o <<= 1) zz += __shfl_xor_sync(0xffffffffu, zz, o);
        const int r = rb + rg + u * rstride;
        if (k == 0 && r < R) part[r] = zz;
      }
    }
    // thread 0's release after the barrier publishes the whole block's partial (cumulative)
    __syncthreads();
    if (threadIdx.x == 0) red_release_gpu_add(a.sync + l, 1u);
  }
  // after the last pass: the last slab of this matrix to get here writes y and sigma_min
  __syncthreads();
  if (abort_flag) return;
  __threadfence();
  if (threadIdx.x == 0) s_last = atomicAdd(a.done + l, 1u) == static_cast<unsigned>(a.nslab - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  float* y = const_cast<float*>(p.x[l]);
  for (int r = threadIdx.x; r < R; r += kThreads) y[r] = ys[r];
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int b = 0; b < a.nslab; ++b) t += __ldcg(a.dsq + static_cast<long long>(l) * a.nslab + b);
    a.sigma[l] = static_cast<float>(sqrt(t));
  }
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

namespace {

template <bool F32, int NV>
cudaError_t power_launch(const GemvParams& p, const PowerArgs& a, dim3 grid, size_t smem, bool cooperative,
                         cudaStream_t s) {
  auto kern = power_stream_kernel<F32, NV>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  if (!cooperative) {
    kern<<<grid, kPowerThreads, smem, s>>>(p, a);
    return cudaGetLastError();
  }
  void* args[] = {const_cast<GemvParams*>(&p), const_cast<PowerArgs*>(&a)};
  return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kern), grid, dim3(kPowerThreads), args, smem, s);
}

template <bool F32, int NV>
int power_blocks_per_sm(size_t smem) {
  auto kern = power_stream_kernel<F32, NV>;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
    return 0;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kPowerThreads, smem) != cudaSuccess) return 0;
  return n;
}

size_t power_smem_bytes(int cols, bool f32, int& stages) {
  const size_t stage_bytes = kPowerWarps * static_cast<size_t>(cols) * (f32 ? 4 : 2);
  // ~96 KB of rows in flight per block (two blocks per SM), two to eight stages (the consumers
  // work on two at a time)
  stages = static_cast<int>(std::max<size_t>(2, std::min<size_t>(8, (96 * 1024) / stage_bytes)));
  return stages * stage_bytes + sizeof(float) * (((cols + 255) & ~255) + cols) + 16 * stages;
}

int power_occupancy(int cols, bool f32) {
  int stages = 0;
  const size_t smem = power_smem_bytes(cols, f32, stages);
  switch ((cols + 255) / 256) {
#define MUON_POWER_OCC(NVV) \
  case NVV:                 \
    return f32 ? power_blocks_per_sm<true, NVV>(smem) : power_blocks_per_sm<false, NVV>(smem);
    MUON_POWER_OCC(1)
    MUON_POWER_OCC(2)
    MUON_POWER_OCC(3)
    MUON_POWER_OCC(4)
    MUON_POWER_OCC(5)
    MUON_POWER_OCC(6)
    MUON_POWER_OCC(7)
    MUON_POWER_OCC(8)
#undef MUON_POWER_OCC
  }
  return 0;
}

}  // namespace

int power_pass_blocks(int rows, int cols, int batch, bool f32, int sm_count) {
  // as many blocks as fit on the GPU at once (all of them resident, for the cooperative launch),
  // at most 64 per matrix and one stage of rows each
  const int per_sm = std::max(1, power_occupancy(cols, f32));
  const int want = std::max(1, std::min(kPowerMaxBlocks, per_sm * sm_count / batch));
  const int rpb = ((rows + want - 1) / want + kPowerWarps - 1) / kPowerWarps * kPowerWarps;
  return (rows + rpb - 1) / rpb;
}

bool power_pass_together(int cols, bool f32, int nblk, int batch, int sm_count) {
  return static_cast<long long>(nblk) * batch <= static_cast<long long>(power_occupancy(cols, f32)) * sm_count;
}

cudaError_t launch_power_iteration_stream(GemvParams& p, int batch, bool f32, int nblk, int iters,
                                          float* tsq_partial, unsigned* counters, float* sigma, int* status,
                                          int sm_count, cudaStream_t s, const float* shift) {
  const int nv = (p.cols + 255) / 256;
  if (p.cols % 8 != 0 || nv < 1 || nv > 8 || iters < 1 || nblk < 1 || nblk > kPowerMaxBlocks)
    return cudaErrorInvalidValue;
  const int rpb = ((p.rows + nblk - 1) / nblk + kPowerWarps - 1) / kPowerWarps * kPowerWarps;
  if ((p.rows + rpb - 1) / rpb != nblk) return cudaErrorInvalidValue;
  int stages = 0;
  const size_t smem = power_smem_bytes(p.cols, f32, stages);
  // all iterations in one cooperative launch when every block fits on the GPU at once
  bool together = iters > 1 && power_pass_together(p.cols, f32, nblk, batch, sm_count);
  // the shifted iteration keeps y in shared memory from pass to pass: one launch for all passes
  if (shift != nullptr && iters > 1 && !together) return cudaErrorInvalidValue;
  cudaError_t e = cudaMemsetAsync(counters, 0, 2 * sizeof(unsigned) * batch, s);
  if (e != cudaSuccess) return e;
  PowerArgs a;
  a.rows_per_block = rpb;
  a.stages = stages;
  a.nblk = nblk;
  a.iters = iters;
  a.shift = shift;
  a.part[0] = p.partial;
  a.part[1] = p.partial + static_cast<long long>(batch) * nblk * p.cols;
  a.tsq_partial = tsq_partial;
  a.sync = counters;
  a.done = counters + batch;
  a.sigma = sigma;
  a.status = status;
  const dim3 grid(nblk, batch);
  for (int it = 0; it < iters; it = a.it1) {
    a.it0 = it;
    a.it1 = together ? iters : it + 1;
    switch (nv) {
#define MUON_POWER_CASE(NVV)                                                                               \
  case NVV:                                                                                               \
    e = f32 ? power_launch<true, NVV>(p, a, grid, smem, together, s)                                      \
            : power_launch<false, NVV>(p, a, grid, smem, together, s);                                    \
    break;
      MUON_POWER_CASE(1)
      MUON_POWER_CASE(2)
      MUON_POWER_CASE(3)
      MUON_POWER_CASE(4)
      MUON_POWER_CASE(5)
      MUON_POWER_CASE(6)
      MUON_POWER_CASE(7)
      MUON_POWER_CASE(8)
#undef MUON_POWER_CASE
    }
    if (e == cudaErrorCooperativeLaunchTooLarge && together && shift == nullptr) {
      // the device had less room than its occupancy promised (another client on it): the power
      // iteration runs as one launch per iteration instead, from the start
      (void)cudaGetLastError();
      together = false;
      a.it1 = 0;
      continue;
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

namespace {

template <bool F32, int S>
int slab_blocks_per_sm() {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, colslab_kernel<F32, S>, kThreads, 0) != cudaSuccess) return 0;
  return n;
}

int slab_capacity(bool f32, int S, int sm_count) {
  int per_sm = 0;
  if (S == 64) per_sm = f32 ? slab_blocks_per_sm<true, 64>() : slab_blocks_per_sm<false, 64>();
  if (S == 128) per_sm = f32 ? slab_blocks_per_sm<true, 128>() : slab_blocks_per_sm<false, 128>();
  if (S == 256) per_sm = f32 ? slab_blocks_per_sm<true, 256>() : slab_blocks_per_sm<false, 256>();
  return per_sm * sm_count;
}

}  // namespace

int colslab_width(int rows, int cols, int batch, bool f32, int sm_count) {
  if (rows > kSlabRowsMax || rows > cols) return 0;
  // the narrowest slab whose grid still fits on the GPU at once (more blocks, shorter rows)
  for (int S : {64, 128, 256}) {
    if (cols % S != 0) continue;
    const long long blocks = static_cast<long long>(cols / S) * batch;
    if (cols / S <= 1024 && blocks <= slab_capacity(f32, S, sm_count)) return S;
  }
  return 0;
}

cudaError_t launch_min_singular_slabs(GemvParams& p, int batch, bool f32, int S, int iters, const float* shift,
                                      float* dsq, unsigned* counters, float* sigma, int* status, cudaStream_t s) {
  if (S != 64 && S != 128 && S != 256) return cudaErrorInvalidValue;
  if (p.cols % S != 0 || p.rows > kSlabRowsMax || iters < 0) return cudaErrorInvalidValue;
  SlabArgs a;
  a.nslab = p.cols / S;
  a.passes = iters + 1;
  a.shift = shift;
  a.part[0] = p.partial;
  a.part[1] = p.partial + static_cast<long long>(batch) * a.nslab * p.rows;
  a.dsq = dsq;
  a.sync = counters;
  a.done = counters + batch;
  a.sigma = sigma;
  a.status = status;
  cudaError_t e = cudaMemsetAsync(counters, 0, 2 * sizeof(unsigned) * batch, s);
  if (e != cudaSuccess) return e;
  const dim3 grid(a.nslab, batch);
  void* args[] = {&p, &a};
  const void* kern = nullptr;
  if (S == 64) kern = f32 ? reinterpret_cast<const void*>(colslab_kernel<true, 64>)
                          : reinterpret_cast<const void*>(colslab_kernel<false, 64>);
  if (S == 128) kern = f32 ? reinterpret_cast<const void*>(colslab_kernel<true, 128>)
                           : reinterpret_cast<const void*>(colslab_kernel<false, 128>);
  if (S == 256) kern = f32 ? reinterpret_cast<const void*>(colslab_kernel<true, 256>)
                           : reinterpret_cast<const void*>(colslab_kernel<false, 256>);
  return cudaLaunchCooperativeKernel(kern, grid, dim3(kThreads), args, 0, s);
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
  const int nblk = (p.m + kCapRows - 1) / kCapRows;
  const size_t smem = sizeof(float) * ((p.n + 255) & ~255);
  if (p.planes != 1 && p.planes != 3) return cudaErrorInvalidValue;
  auto kern = p.planes == 1 ? cap_alpha_partial_kernel<1> : cap_alpha_partial_kernel<3>;
  if (smem > 48 * 1024) {
    const cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  kern<<<dim3(nblk, batch), kThreads, smem, s>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  cap_alpha_reduce_kernel<<<batch, 32, 0, s>>>(p.partial, nblk, alpha);
  return cudaGetLastError();
}

}  // namespace muon
