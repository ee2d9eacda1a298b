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
// One launch covers every group of a call (blocks cut into per-group ranges).
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
#include "rowpos.cuh"

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

// The current W at dst[0..8) (16-byte aligned bf16, 32-byte fp32), when the pass applies a decay.
template <bool F32>
__device__ __forceinline__ void load8_w(const void* dst, int apply, float (&c)[8]) {
  if (!apply) {
#pragma unroll
    for (int t = 0; t < 8; ++t) c[t] = 0.f;
    return;
  }
  if (F32) {
    const float4* p = reinterpret_cast<const float4*>(dst);
    const float4 a = p[0], b = p[1];
    c[0] = a.x; c[1] = a.y; c[2] = a.z; c[3] = a.w; c[4] = b.x; c[5] = b.y; c[6] = b.z; c[7] = b.w;
  } else {
    const uint4 q = *reinterpret_cast<const uint4*>(dst);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      c[2 * i] = __uint_as_float(w[i] << 16);
      c[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

// dst[0..8) <- decay * c - lrs * v (apply) or v, in W's dtype.
template <bool F32>
__device__ __forceinline__ void store8_w(void* dst, const float (&v)[8], const float (&c)[8], int apply, float decay,
                                         float lrs) {
  float o[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) o[t] = apply ? fmaf(decay, c[t], -lrs * v[t]) : v[t];
  if (F32) {
    float4* p = reinterpret_cast<float4*>(dst);
    p[0] = make_float4(o[0], o[1], o[2], o[3]);
    p[1] = make_float4(o[4], o[5], o[6], o[7]);
  } else {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      w[i] = static_cast<uint32_t>(float_to_bf16_bits(o[2 * i])) |
             (static_cast<uint32_t>(float_to_bf16_bits(o[2 * i + 1])) << 16);
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// 16 bytes global -> this thread's shared memory, asynchronously (no registers held).
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// O - au v^T on 8 columns c..c+7 (c % 8 == 0): two 16-byte reads of v when the cap's
// vectors are aligned and the 8 columns exist, else element by element (columns < C).
__device__ __forceinline__ void cap_term8(float (&ov)[8], float au, const float* v, int c, int C, bool vec) {
  if (vec && c + 8 <= C) {
    const float4 x = *reinterpret_cast<const float4*>(v + c);
    const float4 y = *reinterpret_cast<const float4*>(v + c + 4);
    const float vv[8] = {x.x, x.y, x.z, x.w, y.x, y.y, y.z, y.w};
#pragma unroll
    for (int t = 0; t < 8; ++t) ov[t] = fmaf(-au, vv[t], ov[t]);
  } else {
#pragma unroll
    for (int t = 0; t < 8; ++t)
      if (c + t < C) ov[t] = fmaf(-au, v[c + t], ov[t]);
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
// A bf16 W takes two 8-element steps per iteration, both steps' loads issued as packed
// 16-byte vectors before either is unpacked (within the 40-register budget that keeps six
// blocks per SM); an fp32 W (three-plane iterate) or the capped pass, which would not fit
// that budget, one step.
template <bool F32, bool CAP>
__device__ __forceinline__ void wide_body(const ApplyParams& p, const ApplyGroup& q, int l, int b) {
  void* w = p.w[q.mat0 + l];
  const uint16_t* o = q.o + static_cast<long long>(l) * q.o_mat;
  const int C = q.cols;
  const bool cap = CAP && q.alpha != nullptr;
  if (q.vec) {
    const int per_row = C / 8;
    const long long total = static_cast<long long>(q.rows) * per_row;
    const long long chunk = (total + q.nblk - 1) / q.nblk;
    const long long beg = chunk * b;
    const long long end = min(total, beg + chunk);
    const RowStep one = rowstep_of(kThreads, per_row), two_steps = rowstep_of(2 * kThreads, per_row);
    if (F32 || CAP) {
      RowPos pos = rowpos_at(beg + threadIdx.x, per_row);
      for (long long v = beg + threadIdx.x; v < end; v += kThreads, pos = rowpos_add(pos, one, per_row)) {
        const long long i = pos.i;
        const int j = pos.j * 8;
        char* dst = static_cast<char*>(w) + (i * C + j) * (F32 ? 4 : 2);
        float ov[8], cw[8];
        load8_planes(o + i * q.pitch + j, q.o_plane, p.planes, ov);
        load8_w<F32>(dst, p.apply, cw);
        if (cap) cap_term8(ov, q.alpha[l] * p.cu[q.mat0 + l][i], p.cv[q.mat0 + l], j, C, q.cvec);
        store8_w<F32>(dst, ov, cw, p.apply, p.decay, q.lrs);
      }
    } else {
      RowPos pa = rowpos_at(beg + threadIdx.x, per_row);
      for (long long v0 = beg + threadIdx.x; v0 < end; v0 += 2 * kThreads, pa = rowpos_add(pa, two_steps, per_row)) {
        const long long v1 = v0 + kThreads;
        const bool two = v1 < end;
        const RowPos pb = rowpos_add(pa, one, per_row);
        const long long i0 = pa.i, i1 = pb.i;
        const int j0 = pa.j * 8, j1 = pb.j * 8;
        char* d0 = static_cast<char*>(w) + (i0 * C + j0) * (F32 ? 4 : 2);
        char* d1 = static_cast<char*>(w) + (i1 * C + j1) * (F32 ? 4 : 2);
        // both steps' loads as packed 16-byte vectors before either is unpacked
        uint4 oa[F32 ? 3 : 1], ob[F32 ? 3 : 1], wa[F32 ? 2 : 1], wb[F32 ? 2 : 1];
  #pragma unroll
        for (int pl = 0; pl < (F32 ? 3 : 1); ++pl) {
          oa[pl] = __ldcs(reinterpret_cast<const uint4*>(o + pl * q.o_plane + i0 * q.pitch + j0));
          if (two) ob[pl] = __ldcs(reinterpret_cast<const uint4*>(o + pl * q.o_plane + i1 * q.pitch + j1));
        }
        if (p.apply) {
  #pragma unroll
          for (int k = 0; k < (F32 ? 2 : 1); ++k) {
            wa[k] = reinterpret_cast<const uint4*>(d0)[k];
            if (two) wb[k] = reinterpret_cast<const uint4*>(d1)[k];
          }
        }
  #pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (h == 1 && !two) break;
          const uint4* ov4 = h ? ob : oa;
          float ov[8], cw[8];
  #pragma unroll
          for (int t = 0; t < 8; ++t) ov[t] = 0.f;
  #pragma unroll
          for (int pl = 0; pl < (F32 ? 3 : 1); ++pl) {
            const uint32_t u[4] = {ov4[pl].x, ov4[pl].y, ov4[pl].z, ov4[pl].w};
  #pragma unroll
            for (int k = 0; k < 4; ++k) {
              ov[2 * k] += __uint_as_float(u[k] << 16);
              ov[2 * k + 1] += __uint_as_float(u[k] & 0xFFFF0000u);
            }
          }
          load8_w<F32>(h ? wb : wa, p.apply, cw);
          const long long ii = h ? i1 : i0;
          const int jj = h ? j1 : j0;
          if (cap) cap_term8(ov, q.alpha[l] * p.cu[q.mat0 + l][ii], p.cv[q.mat0 + l], jj, C, q.cvec);
          store8_w<F32>(h ? d1 : d0, ov, cw, p.apply, p.decay, q.lrs);
        }
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
      float ov = load1_planes(o + i * q.pitch + j, q.o_plane, p.planes);
      if (cap) ov = fmaf(-q.alpha[l] * p.cu[q.mat0 + l][i], p.cv[q.mat0 + l][j], ov);
      rmw1<F32>(w, e, ov, p.apply, p.decay, q.lrs);
    }
  }
}

// Tall W (rows > cols): W(r, c) with O(c, r), through a 64 x 64 tile.  Each thread's share of
// the tile's W is copied into shared memory (cp.async) while O is read and transposed, so the two
// reads' latencies overlap; the thread reads back only what it copied itself.
template <bool F32, bool CAP>
__device__ __forceinline__ void tall_body(const ApplyParams& p, const ApplyGroup& q, int l, int b) {
  __shared__ float tile[64][65];
  __shared__ __align__(16) uint8_t wtile[64][64 * (F32 ? 4 : 2)];
  void* w = p.w[q.mat0 + l];
  const uint16_t* o = q.o + static_cast<long long>(l) * q.o_mat;
  const int R = q.rows, C = q.cols;
  const bool cap = CAP && q.alpha != nullptr;
  const int tiles_c = (C + 63) / 64;
  const int ntiles = ((R + 63) / 64) * tiles_c;
  const int rr = threadIdx.x >> 3;       // 0..31
  const int cc = (threadIdx.x & 7) * 8;  // 0..56
  // tile tt = (row tile, column tile) walked in strides of nblk without a division per tile
  const RowStep tstep = rowstep_of(q.nblk, tiles_c);
  RowPos tp = rowpos_at(b, tiles_c);
  for (int tt = b; tt < ntiles; tt += q.nblk, tp = rowpos_add(tp, tstep, tiles_c)) {
    const int r0 = tp.i * 64, c0 = tp.j * 64;
    const bool wvec = q.vec && c0 + cc < C;
    if (wvec && p.apply) {
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {
        const int r = r0 + rr + 32 * pass;
        if (r < R) {
          const char* src = static_cast<const char*>(w) + (static_cast<long long>(r) * C + c0 + cc) * (F32 ? 4 : 2);
#pragma unroll
          for (int k = 0; k < (F32 ? 2 : 1); ++k) cp_async16(&wtile[rr + 32 * pass][cc * (F32 ? 4 : 2) + 16 * k], src + 16 * k);
        }
      }
    }
    // O rows c (= W columns), 8 consecutive W rows r per thread: O(c, r..r+7); the wide pitch is
    // >= round_up(R, 8) and r % 8 == 0, so the 8-wide read stays in the row.  A bf16 W comes with
    // a one-plane iterate: both passes' 16-byte vectors are read before either is unpacked.
    if (!F32) {
      uint4 oq[2];
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {
        const int c = c0 + rr + 32 * pass;
        const int r = r0 + cc;
        oq[pass] = c < C && r < R ? __ldcs(reinterpret_cast<const uint4*>(o + static_cast<long long>(c) * q.pitch + r))
                                  : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {
        const uint32_t u[4] = {oq[pass].x, oq[pass].y, oq[pass].z, oq[pass].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          tile[cc + 2 * k][rr + 32 * pass] = __uint_as_float(u[k] << 16);
          tile[cc + 2 * k + 1][rr + 32 * pass] = __uint_as_float(u[k] & 0xFFFF0000u);
        }
      }
    } else {
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {
        const int c = c0 + rr + 32 * pass;
        const int r = r0 + cc;
        float ov[8];
        if (c < C && r < R) {
          load8_planes(o + static_cast<long long>(c) * q.pitch + r, q.o_plane, p.planes, ov);
        } else {
#pragma unroll
          for (int t = 0; t < 8; ++t) ov[t] = 0.f;
        }
#pragma unroll
        for (int t = 0; t < 8; ++t) tile[cc + t][rr + 32 * pass] = ov[t];
      }
    }
    if (wvec && p.apply) cp_async_wait_all();
    __syncthreads();
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
      const int rl = rr + 32 * pass;
      const int r = r0 + rl;
      const int c = c0 + cc;
      if (r < R) {
        float v[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) v[t] = tile[rl][cc + t];
        if (cap) cap_term8(v, q.alpha[l] * p.cu[q.mat0 + l][r], p.cv[q.mat0 + l], c, C, q.cvec);
        if (wvec) {
          char* dst = static_cast<char*>(w) + (static_cast<long long>(r) * C + c) * (F32 ? 4 : 2);
          float cw[8];
          load8_w<F32>(&wtile[rl][cc * (F32 ? 4 : 2)], p.apply, cw);
          store8_w<F32>(dst, v, cw, p.apply, p.decay, q.lrs);
        } else {
#pragma unroll
          for (int t = 0; t < 8; ++t)
            if (c + t < C) rmw1<F32>(w, static_cast<long long>(r) * C + c + t, v[t], p.apply, p.decay, q.lrs);
        }
      }
    }
    __syncthreads();
  }
}

// Six blocks per SM (40 registers) for the plain pass; the capped instantiation, which also
// carries the rank-one term, four (64 registers) so that it does not spill.
template <bool F32, bool CAP>
__global__ void __launch_bounds__(kThreads, CAP ? 4 : 6) apply_kernel(const __grid_constant__ ApplyParams p) {
  int gi = 0;
  while (gi + 1 < p.ngroups && static_cast<int>(blockIdx.x) >= p.grp[gi + 1].block0) ++gi;
  const ApplyGroup& q = p.grp[gi];
  const int local = static_cast<int>(blockIdx.x) - q.block0;
  const int lr = local / q.nblk;
  const int b = local - lr * q.nblk;
  // matrices last to first: the Newton-Schulz launch wrote the last matrix last
  const int l = q.batch - 1 - lr;
  if (q.flags != nullptr && q.flags[l] != 0) return;
  if (p.status != nullptr && (*p.status & kStatusTimeout)) return;  // the iterate is incomplete
  if (q.rows > q.cols) tall_body<F32, CAP>(p, q, l, b);
  else wide_body<F32, CAP>(p, q, l, b);
}

}  // namespace

cudaError_t launch_apply(ApplyParams& p, bool w_f32, cudaStream_t stream) {
  if (p.ngroups < 1 || p.ngroups > MUON_MAX_GROUPS) return cudaErrorInvalidValue;
  long long blocks = 0;
  bool cap = false;
  for (int gi = 0; gi < p.ngroups; ++gi) {
    ApplyGroup& q = p.grp[gi];
    q.block0 = static_cast<int>(blocks);
    q.vec = q.cols % 8 == 0;
    for (int l = 0; l < q.batch && q.vec; ++l)
      if (reinterpret_cast<uintptr_t>(p.w[q.mat0 + l]) % 16) q.vec = 0;
    q.cvec = q.alpha != nullptr;
    for (int l = 0; l < q.batch && q.cvec; ++l)
      if (reinterpret_cast<uintptr_t>(p.cv[q.mat0 + l]) % 16) q.cvec = 0;
    cap = cap || q.alpha != nullptr;
    blocks += static_cast<long long>(q.batch) * q.nblk;
  }
  if (blocks < 1 || blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(blocks));
  // the cap term is its own instantiation: the plain pass keeps its register allocation
  if (cap) {
    if (w_f32) apply_kernel<true, true><<<grid, kThreads, 0, stream>>>(p);
    else apply_kernel<false, true><<<grid, kThreads, 0, stream>>>(p);
  } else {
    if (w_f32) apply_kernel<true, false><<<grid, kThreads, 0, stream>>>(p);
    else apply_kernel<false, false><<<grid, kThreads, 0, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace muon
