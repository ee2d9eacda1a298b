// The three matrix products of a Newton-Schulz iteration on the tensor cores
// of sm_100a (tcgen05 + TMEM, operands staged by TMA):
//
//   Gram     A = X X^T            M = N = m, K = n, symmetric output
//   poly     B = b A + c A A      M = N = K = m,   symmetric output
//   update   X' = a X + B X       M = m, N = n, K = m (B operand MN-major)
//
// (MuonSSM: Orthogonalizing State Space Models, section on the lightweight
// Newton-Schulz step: the orthogonalisation is matrix products only, no SVD;
// Muon Meets Mamba, abstract: one orthogonalised update per weight matrix.)
//
// One persistent kernel serves all three: a launch carries every (group,
// iteration, phase) problem of a step, a CTA owns a 128-row M tile and up to
// 256 N columns, walks a static round-robin list of tiles (group by group,
// phase by phase, matrix by matrix), and runs
//   warp 0      TMA producer (one thread) into a 4-stage ring of 48 KB stages;
//               before a tile it waits for the previous phase of that tile's
//               matrix (per-(problem, matrix) completion counters),
//   warp 1      TMEM allocation + UMMA issuer (one thread),
//   warps 2..9  epilogue: TMEM -> registers -> fused arithmetic -> 32 x 32
//               swizzled shared-memory tiles -> TMA tensor stores; each warp
//               hands the accumulator back after its last TMEM read and counts
//               the tile done once its stores have landed.
// Two TMEM accumulators (2 x 256 fp32 columns) let the epilogue of one tile
// overlap the main loop of the next.  Symmetric outputs are computed on the
// upper 128 x 128 blocks only (tiles start at the diagonal block, and such a
// tile reads its A operand from the first rows of its B stage); the lower
// blocks are written by transposing the staged tile (a second TMA store).
// The update's aX term is folded into the polynomial (B' = aI + bA + cA^2),
// so the update epilogue only scales, converts and stores.
// The fp32 path passes three bf16 planes per operand; six plane products
// (small terms first) are accumulated in the same TMEM tile.
//
// Every wait is bounded; a CTA that runs out sets the device status word and
// unwinds after draining its own copies and MMAs, then frees its TMEM.
#include <cuda_bf16.h>

#include "device_utils.cuh"
#include "gemm.h"

namespace muon {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int BN = 256;
constexpr int STAGES = 4;
constexpr uint32_t A_BYTES = BM * BK * 2;     // 16 KB
constexpr uint32_t B_BYTES = BN * BK * 2;     // 32 KB
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t KMAJ_BOX_BYTES = 128 * BK * 2;  // box {64 K, 128 rows}
constexpr uint32_t MNMAJ_BOX_BYTES = 64 * BK * 2;  // box {64 N, 64 K rows}
constexpr int EPI_WARPS = kEpilogueWarps;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr uint32_t STAGING_BYTES_PER_WARP = 2 * 2048;  // two 32 x 32 bf16 store tiles
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COLS = 256;
constexpr int NUM_BARS = 2 * STAGES + 5;
constexpr uint32_t BAR_BYTES = 8 * NUM_BARS + 16;
constexpr uint64_t kDrainLimitNs = 200000000ull;

struct Tile {
  int pi, l, m0, n0, nw;
};

// What decoding a tile index needs of each problem, copied into shared memory at launch: the
// parameter block (up to 30 problems of four tensor maps each) is far larger than the constant
// cache, and every role decodes every tile.
struct TileMeta {
  int tile_base, tiles_per_matrix, L, M, N, sym, reverse, pad;
};
constexpr uint32_t META_BYTES = kMaxProblems * sizeof(TileMeta);

__device__ __forceinline__ void load_meta(const GemmParams& P, TileMeta* meta) {
  for (int i = threadIdx.x; i < P.nprob; i += blockDim.x) {
    const GemmProblem& q = P.prob[i];
    meta[i] = TileMeta{q.tile_base, q.tiles_per_matrix, q.L, q.M, q.N, q.sym, q.reverse, 0};
  }
}

// Tile t of the launch: problem, matrix, first row (multiple of TM), first
// column and width (a multiple of NG, at most BN).  Symmetric outputs start
// each TM-row block at its diagonal block.
template <int TM, int NG>
__device__ __forceinline__ Tile decode_tile(const TileMeta* meta, int nprob, int t) {
  Tile ti;
  int lo = 0, hi = nprob - 1;  // last problem whose first tile is <= t
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (meta[mid].tile_base <= t) lo = mid;
    else hi = mid - 1;
  }
  ti.pi = lo;
  const TileMeta q = meta[ti.pi];
  const int local = t - q.tile_base;
  const int lm = local / q.tiles_per_matrix;
  int r = local - lm * q.tiles_per_matrix;
  ti.l = q.reverse ? q.L - 1 - lm : lm;
  if (q.sym) {
    int mb = 0;
    for (;;) {
      const int cnt = (q.M - TM * mb + BN - 1) / BN;
      if (r < cnt) break;
      r -= cnt;
      ++mb;
    }
    ti.m0 = TM * mb;
    ti.n0 = TM * mb + BN * r;
  } else {
    const int tn = (q.N + BN - 1) / BN;
    const int mb = r / tn;
    ti.m0 = TM * mb;
    ti.n0 = (r - mb * tn) * BN;
  }
  const int nw = ((q.N - ti.n0 + NG - 1) / NG) * NG;
  ti.nw = nw < BN ? nw : BN;
  return ti;
}

// Plane pairs of the split products, smallest first: mid*mid, hi*lo, lo*hi,
// hi*mid, mid*hi, hi*hi (plane 0 = hi, 1 = mid, 2 = lo).
__device__ __forceinline__ void segment_planes(int nseg, int seg, int& pa, int& pb) {
  if (nseg == 1) {
    pa = 0;
    pb = 0;
    return;
  }
  // nibble seg of each constant: a planes {1,0,2,0,1,0}, b planes {1,2,0,1,0,0}
  pa = (0x10201 >> (4 * seg)) & 0xF;
  pb = (0x01021 >> (4 * seg)) & 0xF;
}

__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kDrainLimitNs) return false;
  }
  return true;
}

// ------------------------------------------------------------------ epilogue
__device__ __forceinline__ void unpack_bf16x8(uint4 q, float* v) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// v[t] += beta * sum_p cin_p(row, j0 + t) for t < nv (caller guarantees row < M, j0 < N)
__device__ __forceinline__ void add_cin(const GemmProblem& q, int l, int row, int j0, int nv,
                                        float (&v)[32]) {
  float c[32];
#pragma unroll
  for (int t = 0; t < 32; ++t) c[t] = 0.f;
  for (int p = 0; p < q.planes; ++p) {
    const uint16_t* src = q.cin + p * q.cin_plane + l * q.cin_mat +
                          static_cast<long long>(row) * q.cin_pitch + j0;
    if (nv == 32) {
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        float f[8];
        unpack_bf16x8(__ldcg(reinterpret_cast<const uint4*>(src) + h), f);
#pragma unroll
        for (int t = 0; t < 8; ++t) c[8 * h + t] += f[t];
      }
    } else {
#pragma unroll
      for (int t = 0; t < 32; ++t)
        if (t < nv) c[t] += bf16_bits_to_float(__ldcg(src + t));
    }
  }
#pragma unroll
  for (int t = 0; t < 32; ++t) v[t] = fmaf(q.beta, c[t], v[t]);
}

// Staging tile for one TMA store: 32 rows x 32 bf16 (64-byte rows) in the
// 64-byte swizzle the tensor map declares: 16-byte chunk c of row r sits at
// chunk c ^ ((r >> 1) & 3), which also keeps the row-per-lane writes free of
// bank conflicts.
__device__ __forceinline__ uint32_t stage_offset(int r, int chunk16) {
  return static_cast<uint32_t>(r * 64 + ((chunk16 ^ ((r >> 1) & 3)) << 4));
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

__device__ __forceinline__ void st_shared_u16(uint32_t addr, uint16_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

// This lane's 32 values become row `lane` of the staging tile.
__device__ __forceinline__ void stage_as_row(uint32_t buf, int lane, const uint16_t (&b)[32]) {
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    const int o = 8 * h;
    st_shared_v4(buf + stage_offset(lane, h),
                 static_cast<uint32_t>(b[o + 0]) | (static_cast<uint32_t>(b[o + 1]) << 16),
                 static_cast<uint32_t>(b[o + 2]) | (static_cast<uint32_t>(b[o + 3]) << 16),
                 static_cast<uint32_t>(b[o + 4]) | (static_cast<uint32_t>(b[o + 5]) << 16),
                 static_cast<uint32_t>(b[o + 6]) | (static_cast<uint32_t>(b[o + 7]) << 16));
  }
}

// This lane's 32 values become column `lane` of the staging tile (the mirror).
__device__ __forceinline__ void stage_as_col(uint32_t buf, int lane, const uint16_t (&b)[32]) {
#pragma unroll
  for (int t = 0; t < 32; ++t) st_shared_u16(buf + stage_offset(t, lane >> 3) + 2 * (lane & 7), b[t]);
}

// This lane's 32 values, already packed as 16 bf16 pairs, become row `lane` of the staging tile.
__device__ __forceinline__ void stage_packed_row(uint32_t buf, int lane, const uint32_t (&w)[16]) {
#pragma unroll
  for (int h = 0; h < 4; ++h)
    st_shared_v4(buf + stage_offset(lane, h), w[4 * h], w[4 * h + 1], w[4 * h + 2], w[4 * h + 3]);
}

__device__ __forceinline__ void st_shared_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// This lane's 32 values (packed pairs) become column `lane` of the staging tile (the mirror).
// Lanes 2k and 2k+1 trade their pairs, so each writes whole 32-bit words holding columns 2k and
// 2k+1: the even lane rows 2i, the odd lane rows 2i+1.  Each store then fills two adjacent 64-byte
// rows (one shared-memory wavefront) instead of one 2-byte slot per lane and row.
__device__ __forceinline__ void stage_packed_col(uint32_t buf, int lane, const uint32_t (&w)[16]) {
  const bool odd = lane & 1;
  const int col = lane & ~1;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t other = __shfl_xor_sync(0xffffffffu, w[i], 1);
    // even lane: (own low, other low) = row 2i; odd lane: (other high, own high) = row 2i + 1
    const uint32_t word = odd ? __byte_perm(other, w[i], 0x7632) : __byte_perm(w[i], other, 0x5410);
    st_shared_u32(buf + stage_offset(2 * i + (odd ? 1 : 0), col >> 3) + 2 * (col & 7), word);
  }
}

// A chunk and its mirror: both staging buffers filled, one proxy fence, two TMA stores.
// Lane 0 first makes sure every earlier store of this warp has finished reading its buffer.
template <typename StageA, typename StageB>
__device__ __forceinline__ void store_chunk_pair(const CUtensorMap* map, uint32_t stage_base, int& sb, int lane,
                                                 StageA&& sa, StageB&& sbf, int x, int y, int l, int p) {
  sb = 2;
  if (lane == 0) bulk_wait_group_read<0>();
  __syncwarp();
  sa(stage_base);
  sbf(stage_base + 2048u);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_4d(map, stage_base, x, y, l, p);
    tma_store_4d(map, stage_base + 2048u, y, x, l, p);
    bulk_commit_group();
  }
}

// One 32 x 32 TMA store from the warp's next staging buffer.  Lane 0 first
// makes sure the store that last read this buffer has finished reading it.
// `sb` is the next buffer (0 or 1), or 2 after a chunk pair, whose one store group reads both
// buffers: then the next store waits for every earlier group and starts again at buffer 0.
template <typename Stage>
__device__ __forceinline__ void store_chunk(const CUtensorMap* map, uint32_t stage_base, int& sb, int lane,
                                            Stage&& stage, int x, int y, int l, int p) {
  if (lane == 0) {
    if (sb == 2) bulk_wait_group_read<0>();
    else bulk_wait_group_read<1>();
  }
  if (sb == 2) sb = 0;
  const uint32_t buf = stage_base + static_cast<uint32_t>(sb) * 2048u;
  __syncwarp();
  stage(buf);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_4d(map, buf, x, y, l, p);
    bulk_commit_group();
  }
  sb ^= 1;
}

// One warp's share of a finished accumulator tile: TMEM rows row0..row0+31
// (this warp's lane quarter), 32-column chunks c_first, c_first + 64, ...
// v = alpha s_l acc + beta cin + diag on the diagonal, split into planes and
// stored through TMA; columns from `mirror_from` on are also stored transposed.
// `release()` hands the accumulator back to the MMA issuer: it runs once, right after this
// warp's last TMEM read of the tile (the stores that follow work from registers).
template <class Release>
__device__ __forceinline__ void epilogue_warp_tile(const GemmProblem& q, const Tile& ti, uint32_t tbase,
                                                   int row0, int lane, int c_first, int mirror_from,
                                                   uint32_t my_stage, int& sb, Release&& release) {
  if (row0 >= q.M) {
    release();
    return;
  }
  bool released = false;
  const int row = row0 + lane;
  const float scale = q.alpha * (q.mat_scale != nullptr ? q.mat_scale[ti.l] : 1.0f);
  for (int c = c_first; c < ti.nw; c += 64) {
    const int j0 = ti.n0 + c;
    if (j0 >= q.N) break;
    const int nv = min(32, q.N - j0);
    uint32_t r[32];
    __syncwarp();  // tcgen05.ld is warp-collective
    tmem_load_32cols(tbase + c, r);
    tmem_load_wait();
    if (c + 64 >= ti.nw || j0 + 64 >= q.N) {  // this warp's last chunk of the tile
      release();
      released = true;
    }
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = scale * __uint_as_float(r[i]);
    if (q.cin != nullptr && row < q.M) add_cin(q, ti.l, row, j0, nv, v);
    if (q.diag != 0.f) {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (j0 + i == row) v[i] += q.diag;
    }
    const bool mirror = q.sym && (j0 >= mirror_from);
    if (q.planes == 1) {
      // one bf16 plane: round to nearest even two values at a time, already packed for the stores
      uint32_t w[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t*>(&h);
      }
      if (mirror) {
        store_chunk_pair(
            &q.tmOut, my_stage, sb, lane, [&](uint32_t buf) { stage_packed_row(buf, lane, w); },
            [&](uint32_t buf) { stage_packed_col(buf, lane, w); }, j0, row0, ti.l, 0);
      } else {
        store_chunk(&q.tmOut, my_stage, sb, lane, [&](uint32_t buf) { stage_packed_row(buf, lane, w); }, j0, row0,
                    ti.l, 0);
      }
    } else {
      for (int p = 0; p < q.planes; ++p) {
        uint16_t b[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          b[i] = float_to_bf16_bits(v[i]);
          v[i] -= bf16_bits_to_float(b[i]);  // residual for the next plane
        }
        store_chunk(&q.tmOut, my_stage, sb, lane, [&](uint32_t buf) { stage_as_row(buf, lane, b); }, j0, row0,
                    ti.l, p);
        if (mirror)
          store_chunk(&q.tmOut, my_stage, sb, lane, [&](uint32_t buf) { stage_as_col(buf, lane, b); }, row0, j0,
                      ti.l, p);
      }
    }
  }
  if (!released) release();
}

// ------------------------------------------------------------------ kernel
__global__ void __launch_bounds__(THREADS, 1) ns_gemm_kernel(const __grid_constant__ GemmParams P) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t stage_area = base + STAGES * STAGE_BYTES;
  const uint32_t bar0 = stage_area + EPI_WARPS * STAGING_BYTES_PER_WARP;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(gbase + (bar0 - base) + 8 * NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  TileMeta* meta = reinterpret_cast<TileMeta*>(gbase + (bar0 - base) + BAR_BYTES);
  load_meta(P, meta);

  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 32 * EPI_WARPS);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < P.nprob; ++i) {
      tma_prefetch_map(&P.prob[i].tmA);
      tma_prefetch_map(&P.prob[i].tmB);
      tma_prefetch_map(&P.prob[i].tmOut);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      // counter of the next tile's dependency, read early (relaxed) so its
      // latency hides behind the current tile's loads
      unsigned dep_seen = 0;
      if (blockIdx.x < P.total_tiles) {
        const Tile t0 = decode_tile<BM, 64>(meta, P.nprob, blockIdx.x);
        if (P.prob[t0.pi].done_dep != nullptr) dep_seen = ld_relaxed_gpu(P.prob[t0.pi].done_dep + t0.l);
      }
      for (int t = blockIdx.x; ok && t < P.total_tiles; t += gridDim.x) {
        const Tile ti = decode_tile<BM, 64>(meta, P.nprob, t);
        const GemmProblem& q = P.prob[ti.pi];
        if (q.done_dep != nullptr) {
          // the previous phase of this matrix must have landed before it is read
          if (dep_seen >= q.dep_target) {
            __threadfence();  // acquire: pairs with the writers' release increments
          } else if (!wait_counter_bounded(q.done_dep + ti.l, q.dep_target, abort_flag, P.status)) {
            ok = false;
            break;
          }
          fence_proxy_async_global();
        }
        const int tn = t + gridDim.x;
        if (tn < P.total_tiles) {
          const Tile tin = decode_tile<BM, 64>(meta, P.nprob, tn);
          dep_seen = P.prob[tin.pi].done_dep != nullptr ? ld_relaxed_gpu(P.prob[tin.pi].done_dep + tin.l) : 0u;
        }
        const int nk = q.k_tiles * q.nseg;
        const bool narrow = !q.b_mn_major && ti.nw <= 128;
        const uint32_t bbytes = q.b_mn_major ? 4u * MNMAJ_BOX_BYTES : (narrow ? KMAJ_BOX_BYTES : 2u * KMAJ_BOX_BYTES);
        // a symmetric tile that starts on the diagonal has A = the first 128 rows of B
        const bool diag_tile = q.sym && ti.m0 == ti.n0;
        for (int kk = 0; kk < nk; ++kk, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait_bounded(empty_bar(s), ph ^ 1u, abort_flag, P.status)) {
            ok = false;
            break;
          }
          const int seg = kk / q.k_tiles;
          const int kb = kk - seg * q.k_tiles;
          int pa, pb;
          segment_planes(q.nseg, seg, pa, pb);
          const uint32_t sa = base + s * STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
          const bool a_in_b = diag_tile && pa == pb;  // the MMA reads A from B's first rows
          mbar_arrive_expect_tx(full_bar(s), (a_in_b ? 0u : A_BYTES) + bbytes);
          if (!a_in_b) tma_load_4d(sa, &q.tmA, full_bar(s), kb * BK, ti.m0, ti.l, pa);
          if (q.b_mn_major)
            tma_load_5d(sb, &q.tmB, full_bar(s), 0, kb * BK, ti.n0 / 64, ti.l, pb);
          else
            tma_load_4d(sb, narrow ? &q.tmB2 : &q.tmB, full_bar(s), kb * BK, ti.n0, ti.l, pb);
        }
      }
      if (!ok) {
        // Let the copies this thread started land before the CTA exits.
        const uint32_t n = it < STAGES ? it : STAGES;
        for (uint32_t j = it - n; j < it; ++j) wait_drain(full_bar(j % STAGES), (j / STAGES) & 1u);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ UMMA issuer
    if (lane == 0) {
      uint32_t it = 0;
      int local = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < P.total_tiles; t += gridDim.x, ++local) {
        const Tile ti = decode_tile<BM, 64>(meta, P.nprob, t);
        const GemmProblem& q = P.prob[ti.pi];
        const int acc = local & 1;
        const uint32_t aph = (local >> 1) & 1;
        if (!mbar_wait_bounded(tempty_bar(acc), aph ^ 1u, abort_flag, P.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
        const uint32_t idesc = instr_desc_bf16(BM, ti.nw, q.b_mn_major != 0);
        const int nk = q.k_tiles * q.nseg;
        const bool diag_tile = q.sym && ti.m0 == ti.n0;
        // Descriptors of stage 0, k-step 0; a stage or k-step only moves the start address (the
        // low 14 bits, in 16-byte units, which never carry: shared addresses are below 256 KB).
        // K-major operands advance 32 bytes per 16-deep k-step, the MN-major B 16 rows of 128 bytes.
        const uint64_t a_desc0 = smem_desc_sw128(base, 16u, 1024u);
        const uint64_t b_desc0 = q.b_mn_major ? smem_desc_sw128(base + A_BYTES, MNMAJ_BOX_BYTES, 1024u)
                                              : smem_desc_sw128(base + A_BYTES, 16u, 1024u);
        const uint32_t b_step = q.b_mn_major ? (2048u >> 4) : (32u >> 4);
        for (int kk = 0; kk < nk; ++kk, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait_bounded(full_bar(s), ph, abort_flag, P.status)) {
            ok = false;
            break;
          }
          int pa, pb;
          segment_planes(q.nseg, kk / q.k_tiles, pa, pb);
          const uint32_t stage_off = static_cast<uint32_t>(s) * (STAGE_BYTES >> 4);
          // K-major, 128-byte swizzle: B's rows 0..127 are laid out exactly as an A tile
          const uint64_t ad = a_desc0 + stage_off + (diag_tile && pa == pb ? (A_BYTES >> 4) : 0u);
          const uint64_t bd = b_desc0 + stage_off;
#pragma unroll
          for (int k4 = 0; k4 < BK / 16; ++k4)
            tc_mma_bf16(d_tmem, ad + 2u * k4, bd + b_step * k4, idesc, (kk | k4) != 0 ? 1u : 0u);
          tc_commit(empty_bar(s));
        }
        if (ok) tc_commit(tfull_bar(acc));
      }
      if (!ok) {
        tc_commit(drain_bar);
        wait_drain(drain_bar, 0);
      }
    }
  } else {
    // ------------------------------------------------ epilogue (warps 2 .. 2+EPI_WARPS-1)
    // Two warps share each TMEM lane quarter and split its 32-column chunks.
    const int e = warp - 2;
    const int quarter = warp & 3;
    const int half = e >> 2;
    const uint32_t my_stage = stage_area + static_cast<uint32_t>(e) * STAGING_BYTES_PER_WARP;
    int sb = 0;
    int local = 0;
    for (int t = blockIdx.x; t < P.total_tiles; t += gridDim.x, ++local) {
      const Tile ti = decode_tile<BM, 64>(meta, P.nprob, t);
      const GemmProblem& q = P.prob[ti.pi];
      const int acc = local & 1;
      const uint32_t aph = (local >> 1) & 1;
      if (!mbar_wait_bounded(tfull_bar(acc), aph, abort_flag, P.status)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(32 * quarter) << 16) + acc * ACC_COLS;
      if (q.cin != nullptr && q.done_dep != nullptr) {
        // cin was written earlier in this launch: acquire it for this warp's plain loads
        if (!wait_counter_bounded(q.done_dep + ti.l, q.dep_target, abort_flag, P.status)) break;
      }
      epilogue_warp_tile(q, ti, tbase, ti.m0 + 32 * quarter, lane, 32 * half, ti.m0 + BM, my_stage, sb, [&] {
        tc_fence_before();
        mbar_arrive(tempty_bar(acc));
      });
      if (q.done_self != nullptr) {
        // this warp's stores of the tile are complete and visible: count it done
        if (lane == 0) {
          bulk_wait_group_all();
          fence_proxy_async_global();
          if (!(P.drop_signal && blockIdx.x == 0 && e == 0 && local == 0))
            red_release_gpu_add(q.done_self + ti.l, 1u);
        }
        __syncwarp();
      }
    }
    if (lane == 0) bulk_wait_group_all();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}


}  // namespace

size_t gemm_smem_bytes() { return STAGES * STAGE_BYTES + EPI_WARPS * STAGING_BYTES_PER_WARP + BAR_BYTES + META_BYTES + 1024; }

int gemm_tiles_per_matrix(int M, int N, int sym) {
  if (sym) {
    int n = 0;
    for (int mb = 0; mb * BM < M; ++mb) n += (M - BM * mb + BN - 1) / BN;
    return n;
  }
  return ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
}

cudaError_t launch_gemm(const GemmParams& p, int ctas, cudaStream_t stream) {
  static int configured_device = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const int smem = static_cast<int>(gemm_smem_bytes());
  if (configured_device != dev) {
    e = cudaFuncSetAttribute(ns_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  ns_gemm_kernel<<<ctas, THREADS, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace muon
