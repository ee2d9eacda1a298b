// C-ABI of libmuon: argument checks, workspace, tensor maps and the launch
// sequence of one Muon step (momentum pass, k Newton-Schulz iterations of
// three tensor-core products each, the last one applying the update).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/muon.h"
#include "device_utils.cuh"
#include "internal.h"

using namespace muon;

namespace {

// ------------------------------------------------------------------ errors
char g_cuda_error[256] = "";
std::mutex g_err_mu;

muon_status cuda_fail(cudaError_t e, const char* what) {
  std::lock_guard<std::mutex> lk(g_err_mu);
  std::snprintf(g_cuda_error, sizeof(g_cuda_error), "%s: %s", what, cudaGetErrorString(e));
  return MUON_ERR_CUDA;
}

#define MUON_CUDA(call, what)                          \
  do {                                                 \
    cudaError_t _e = (call);                           \
    if (_e != cudaSuccess) return cuda_fail(_e, what); \
  } while (0)

// Capture state of `s`: 0 not capturing, 1 capturing into a CUDA graph, -1 unreadable.
int capture_state(cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  return cs == cudaStreamCaptureStatusNone ? 0 : 1;
}

muon_status refuse_growth(const char* what, const char* why) {
  std::lock_guard<std::mutex> lk(g_err_mu);
  std::snprintf(g_cuda_error, sizeof(g_cuda_error), "%s must grow, but %s", what, why);
  return MUON_ERR_ALLOC;
}

// Records why a device allocation failed (and clears the error) for muon_last_cuda_error.
void note_alloc_failure() {
  const cudaError_t e = cudaGetLastError();
  std::lock_guard<std::mutex> lk(g_err_mu);
  std::snprintf(g_cuda_error, sizeof(g_cuda_error), "device allocation: %s", cudaGetErrorString(e));
}

// ------------------------------------------------------------------ tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 buffer [planes][L][rows][pitch] viewed as 4-D {cols, rows, L, planes};
// box {box_cols, box_rows}.  Operand maps use the 128-byte swizzle the UMMA
// descriptors expect; store maps use the 64-byte swizzle of the epilogue's
// 32 x 32 staging tiles.  Out-of-range reads give zeros, stores are clipped.
bool encode_map(CUtensorMap* map, const void* base, int cols, int rows, int L, int planes,
                int pitch, int box_cols, int box_rows,
                CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(planes)};
  const cuuint64_t row_bytes = static_cast<cuuint64_t>(pitch) * 2;
  cuuint64_t strides[3] = {row_bytes, row_bytes * rows, row_bytes * rows * L};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

constexpr float kQuintic[3] = {3.4445f, -4.7750f, 2.0315f};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int round8(int x) { return (x + 7) / 8 * 8; }
int round64(int x) { return (x + 63) / 64 * 64; }

// MN-major operand [planes][L][rows][pitch] as the 5-D view {64, rows, pitch/64, L, planes}:
// one box {64, 64, 4, 1, 1} brings 64 rows of four 64-column chunks, chunk after chunk
// (the layout the UMMA descriptor walks with an 8 KB leading-dimension offset).
bool encode_chunked_map(CUtensorMap* map, const void* base, int rows, int L, int planes, int pitch,
                        int chunks = 4) {
  EncodeTiledFn enc = get_encoder();
  if (!enc || pitch % 64) return false;
  cuuint64_t dims[5] = {64, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(pitch / 64),
                        static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(planes)};
  const cuuint64_t row_bytes = static_cast<cuuint64_t>(pitch) * 2;
  cuuint64_t strides[4] = {row_bytes, 128, row_bytes * rows, row_bytes * rows * L};
  cuuint32_t box[5] = {64, 64, static_cast<cuuint32_t>(chunks), 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// One group as the kernels see it.
struct GroupPlan {
  const void* const* g;  // device pointers (G or X)
  float* const* m;       // null for orthogonalise-only
  void* const* w;        // W (step) or Out (orthogonalise)
  int batch, rows, cols, f32, planes;
  int m_rows, n_cols, transposed, pitch_n, pitch_m, nblk;
  long long x_mat, x_plane, a_mat, a_plane;  // elements
  size_t off_x[2], off_a, off_b;             // bytes into the workspace
  int mat_off, part_off;
};

}  // namespace

struct muon_ctx {
  int device = 0;
  int sm_count = 148;
  float coeffs[3 * MUON_MAX_ITERS];
  int k = 5;
  void* ws = nullptr;
  size_t ws_bytes = 0;
  // per-matrix arrays
  int cap_mats = 0;
  size_t cap_parts = 0;
  float* d_nu = nullptr;
  float* d_s1 = nullptr;
  float* d_s2 = nullptr;
  int* d_flags = nullptr;
  unsigned* d_counters = nullptr;
  float* d_partials = nullptr;
  int* d_status = nullptr;
  unsigned* d_done = nullptr;  // [kMaxProblems][MUON_MAX_BATCH] phase-completion counters
  // MUON_OVERLAP=1: momentum passes of later groups and applies of earlier groups run on a side
  // stream beside the Newton-Schulz launches of other groups.  Off by default: on B200 the
  // co-running elementwise passes slow the GEMM by as much time as they hide (both draw on the
  // same L2 -> SM bandwidth), and one persistent launch for all groups has no gap between them.
  bool overlap = false;
  // MUON_TEST_DROP_SIGNAL=1 at creation: the next persistent Newton-Schulz launch drops one
  // completion signal (test of the bounded waits; used once, then cleared)
  bool drop_signal_once = false;
  cudaStream_t side = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  cudaEvent_t ev_k1[MUON_MAX_GROUPS] = {};
  cudaEvent_t ev_gemm[MUON_MAX_GROUPS] = {};
  bool per_phase = false;       // MUON_LAUNCH=phase: one launch per phase (same work; per-phase timing)
  int last_count = 0;
  cudaStream_t last_stream = nullptr;
  bool pending = false;
  bool captured = false;        // a call was captured into a CUDA graph: the buffers never move again
  // device staging for gradients that arrive from host memory
  void* d_stage = nullptr;
  size_t stage_bytes = 0;
  // scratch of the spectral passes (GEMV partials, norms, cap partials)
  void* d_aux = nullptr;
  size_t aux_bytes = 0;
  // results of the last call as muon_get_status / muon_get_norms report them: the per-matrix
  // arrays of the last run, or the gathered copies of a slab-pipelined host call
  const float* out_nu = nullptr;
  const int* out_flags = nullptr;
  float* d_nu_all = nullptr;
  int* d_flags_all = nullptr;
  int cap_all = 0;
  std::vector<cudaEvent_t> copy_events;  // one per slab of a host call
  // per-launch timing
  bool profiling = false;
  std::vector<cudaEvent_t> events;  // pool, two per recorded launch
  std::vector<int> rec_kind;        // kind of recorded launch i (events 2i, 2i+1)
};

namespace {

// Record the start event of a profiled launch; returns the slot or -1.
int prof_begin(muon_ctx* c, int kind, cudaStream_t s) {
  if (!c->profiling) return -1;
  const size_t slot = c->rec_kind.size();
  while (c->events.size() < 2 * (slot + 1)) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return -1;
    c->events.push_back(e);
  }
  c->rec_kind.push_back(kind);
  cudaEventRecord(c->events[2 * slot], s);
  return static_cast<int>(slot);
}

void prof_end(muon_ctx* c, int slot, cudaStream_t s) {
  if (slot >= 0) cudaEventRecord(c->events[2 * slot + 1], s);
}

struct DeviceGuard {
  int prev = -1;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    if (prev != dev) cudaSetDevice(dev);
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

bool finite(float x) { return std::isfinite(x); }

muon_status check_hparams(const muon_hparams* hp) {
  if (!hp) return MUON_ERR_INVALID_ARG;
  if (!finite(hp->lr) || !finite(hp->beta) || !finite(hp->weight_decay) || !finite(hp->eps))
    return MUON_ERR_INVALID_ARG;
  if (hp->eps < 0.f) return MUON_ERR_INVALID_ARG;
  if (!finite(hp->grad_scale) || !(hp->grad_scale > 0.f)) return MUON_ERR_INVALID_ARG;
  if (hp->scale_mode < MUON_SCALE_SQRT_RATIO || hp->scale_mode > MUON_SCALE_RMS_MATCH)
    return MUON_ERR_INVALID_ARG;
  return MUON_OK;
}

muon_status check_group(const muon_group& g, bool need_m) {
  if (g.dtype != MUON_BF16 && g.dtype != MUON_F32) return MUON_ERR_DTYPE;
  if (g.batch < 1 || g.batch > MUON_MAX_BATCH) return MUON_ERR_INVALID_ARG;
  if (g.rows < 1 || g.cols < 1) return MUON_ERR_INVALID_ARG;
  if (g.rows > 32768 || g.cols > 32768 || std::min(g.rows, g.cols) > 8192)
    return MUON_ERR_UNSUPPORTED_SHAPE;
  if (!g.W || !g.G || (need_m && !g.M)) return MUON_ERR_INVALID_ARG;
  for (int l = 0; l < g.batch; ++l) {
    if (!g.W[l] || !g.G[l] || (need_m && !g.M[l])) return MUON_ERR_INVALID_ARG;
  }
  return MUON_OK;
}

float shape_scale(int rows, int cols, int mode) {
  switch (mode) {
    case MUON_SCALE_NONE: return 1.0f;
    case MUON_SCALE_RMS_MATCH: return 0.2f * std::sqrt(static_cast<float>(std::max(rows, cols)));
    default: return std::sqrt(std::max(1.0f, static_cast<float>(rows) / static_cast<float>(cols)));
  }
}

// Make sure the workspace and the per-matrix arrays can hold `plans`.
// Growing a context buffer synchronises the device and allocates; neither is allowed while the
// call's stream is being captured into a CUDA graph, and either would invalidate the capture.  A
// graph captured earlier keeps the buffers' addresses, so once a call has been captured the
// buffers never move again.  In both cases the call is refused before anything is queued (a
// capture in progress stays usable).  A stream whose capture state cannot be read counts as
// capturing: growth would fail on it too.
muon_status may_grow(muon_ctx* c, cudaStream_t s, const char* what) {
  if (capture_state(s) != 0)
    return refuse_growth(what, "the stream is capturing a CUDA graph: make the same call once before capture");
  if (c->captured)
    return refuse_growth(what, "a CUDA graph captured from this context holds its buffers: use another context");
  return MUON_OK;
}

// Called before any work of a call is queued on `s`: remembers that the context's buffers now
// sit in a captured graph.
void note_capture(muon_ctx* c, cudaStream_t s) {
  if (capture_state(s) == 1) c->captured = true;
}

muon_status reserve(muon_ctx* c, std::vector<GroupPlan>& plans, cudaStream_t s) {
  size_t bytes = 0;
  int mats = 0;
  size_t parts = 0;
  for (auto& p : plans) {
    const size_t xb = static_cast<size_t>(p.x_plane) * p.planes * 2;
    const size_t ab = static_cast<size_t>(p.a_plane) * p.planes * 2;
    p.off_x[0] = bytes; bytes = align_up(bytes + xb, 256);
    p.off_x[1] = bytes; bytes = align_up(bytes + xb, 256);
    p.off_a = bytes; bytes = align_up(bytes + ab, 256);
    p.off_b = bytes; bytes = align_up(bytes + ab, 256);
    p.mat_off = mats;
    mats += p.batch;
    p.part_off = static_cast<int>(parts);
    parts += static_cast<size_t>(p.batch) * p.nblk;
  }
  const bool grow_ws = bytes > c->ws_bytes;
  const bool grow_arrays = mats > c->cap_mats || parts > c->cap_parts;
  if (grow_ws || grow_arrays) {
    const muon_status st = may_grow(c, s, "the workspace");
    if (st != MUON_OK) return st;
  }
  note_capture(c, s);
  if (grow_ws) {
    MUON_CUDA(cudaDeviceSynchronize(), "sync before workspace growth");
    if (c->ws) cudaFree(c->ws);
    c->ws = nullptr;
    c->ws_bytes = 0;
    if (cudaMalloc(&c->ws, bytes) != cudaSuccess) {
      note_alloc_failure();
      return MUON_ERR_ALLOC;
    }
    c->ws_bytes = bytes;
  }
  if (grow_arrays) {
    MUON_CUDA(cudaDeviceSynchronize(), "sync before array growth");
    cudaFree(c->d_nu); cudaFree(c->d_s1); cudaFree(c->d_s2); cudaFree(c->d_flags);
    cudaFree(c->d_counters); cudaFree(c->d_partials);
    c->d_nu = c->d_s1 = c->d_s2 = c->d_partials = nullptr;
    c->d_flags = nullptr;
    c->d_counters = nullptr;
    const int cm = std::max(mats, c->cap_mats);
    const size_t cp = std::max(parts, c->cap_parts);
    bool ok = cudaMalloc(&c->d_nu, cm * sizeof(float)) == cudaSuccess &&
              cudaMalloc(&c->d_s1, cm * sizeof(float)) == cudaSuccess &&
              cudaMalloc(&c->d_s2, cm * sizeof(float)) == cudaSuccess &&
              cudaMalloc(&c->d_flags, cm * sizeof(int)) == cudaSuccess &&
              cudaMalloc(&c->d_counters, cm * sizeof(unsigned)) == cudaSuccess &&
              cudaMalloc(&c->d_partials, cp * sizeof(float)) == cudaSuccess;
    if (!ok) {
      note_alloc_failure();
      c->cap_mats = 0;
      c->cap_parts = 0;
      return MUON_ERR_ALLOC;
    }
    MUON_CUDA(cudaMemset(c->d_counters, 0, cm * sizeof(unsigned)), "clear counters");
    MUON_CUDA(cudaMemset(c->d_flags, 0, cm * sizeof(int)), "clear flags");
    c->cap_mats = cm;
    c->cap_parts = cp;
  }
  return MUON_OK;
}

GroupPlan plan_group(const muon_group& g) {
  GroupPlan p{};
  p.g = g.G;
  p.m = g.M;
  p.w = g.W;
  p.batch = g.batch;
  p.rows = g.rows;
  p.cols = g.cols;
  p.f32 = g.dtype == MUON_F32;
  p.planes = p.f32 ? 3 : 1;
  p.transposed = g.rows > g.cols;
  p.m_rows = std::min(g.rows, g.cols);
  p.n_cols = std::max(g.rows, g.cols);
  p.pitch_n = round64(p.n_cols);  // the chunked MN-major view never leaves a row
  p.pitch_m = round8(p.m_rows);
  p.nblk = momentum_blocks_per_matrix(g.rows, g.cols);
  p.x_mat = static_cast<long long>(p.m_rows) * p.pitch_n;
  p.x_plane = p.x_mat * p.batch;
  p.a_mat = static_cast<long long>(p.m_rows) * p.pitch_m;
  p.a_plane = p.a_mat * p.batch;
  return p;
}

uint16_t* ws_at(muon_ctx* c, size_t off) {
  return reinterpret_cast<uint16_t*>(static_cast<char*>(c->ws) + off);
}

enum Phase { PH_GRAM, PH_POLY, PH_UPDATE };

// Fill one GEMM problem for group p, phase ph of iteration `it`.
bool fill_problem(muon_ctx* c, const GroupPlan& p, Phase ph, int it, GemmProblem& q) {
  std::memset(static_cast<void*>(&q), 0, sizeof(q));
  const float a = c->coeffs[3 * it], b = c->coeffs[3 * it + 1], cc = c->coeffs[3 * it + 2];
  const int src = it & 1, dst = (it + 1) & 1;
  (void)dst;
  uint16_t* X = ws_at(c, p.off_x[src]);
  uint16_t* Xn = ws_at(c, p.off_x[dst]);
  uint16_t* A = ws_at(c, p.off_a);
  uint16_t* B = ws_at(c, p.off_b);
  const int m = p.m_rows, n = p.n_cols;
  q.L = p.batch;
  q.nseg = p.planes == 3 ? 6 : 1;
  q.planes = p.planes;
  const bool have_poly = cc != 0.f;
  const CUtensorMapSwizzle sw64 = CU_TENSOR_MAP_SWIZZLE_64B;
  // K-major B operand box height: the tile's N (256, or 128 for narrow tiles)
  const int kb_rows = 256;
  switch (ph) {
    case PH_GRAM:
      // A = s2 * X X^T; with c = 0 the polynomial is linear and the Gram
      // epilogue writes B' = b A + a I directly.
      if (!encode_map(&q.tmA, X, n, m, p.batch, p.planes, p.pitch_n, 64, 128)) return false;
      if (!encode_map(&q.tmB, X, n, m, p.batch, p.planes, p.pitch_n, 64, kb_rows)) return false;
      if (!encode_map(&q.tmB2, X, n, m, p.batch, p.planes, p.pitch_n, 64, kb_rows / 2)) return false;
      if (!encode_map(&q.tmOut, have_poly ? A : B, m, m, p.batch, p.planes, p.pitch_m, 32, 32, sw64))
        return false;
      q.M = m; q.N = m; q.K = n;
      q.b_mn_major = 0; q.sym = 1;
      q.alpha = have_poly ? 1.f : b;
      q.beta = 0.f;
      q.diag = have_poly ? 0.f : a;
      q.mat_scale = it == 0 ? c->d_s2 + p.mat_off : nullptr;
      break;
    case PH_POLY:
      // B' = c A A + b A + a I
      if (!encode_map(&q.tmA, A, m, m, p.batch, p.planes, p.pitch_m, 64, 128)) return false;
      if (!encode_map(&q.tmB, A, m, m, p.batch, p.planes, p.pitch_m, 64, kb_rows)) return false;
      if (!encode_map(&q.tmB2, A, m, m, p.batch, p.planes, p.pitch_m, 64, kb_rows / 2)) return false;
      if (!encode_map(&q.tmOut, B, m, m, p.batch, p.planes, p.pitch_m, 32, 32, sw64)) return false;
      q.M = m; q.N = m; q.K = m;
      q.b_mn_major = 0; q.sym = 1;
      q.alpha = cc; q.beta = b; q.diag = a;
      q.cin = A; q.cin_plane = p.a_plane; q.cin_mat = p.a_mat; q.cin_pitch = p.pitch_m;
      break;
    case PH_UPDATE: {
      // X' = s1 * B' X   (s1 = 1/(nu+eps) on the first iteration, X = U unnormalised)
      if (!encode_map(&q.tmA, B, m, m, p.batch, p.planes, p.pitch_m, 64, 128)) return false;
      // chunked MN-major view: 4 chunks of 64 columns per load
      if (!encode_chunked_map(&q.tmB, X, m, p.batch, p.planes, p.pitch_n, 4)) return false;
      q.M = m; q.N = n; q.K = m;
      q.b_mn_major = 1; q.sym = 0;
      q.alpha = 1.f; q.beta = 0.f; q.diag = 0.f;
      q.mat_scale = it == 0 ? c->d_s1 + p.mat_off : nullptr;
      if (!encode_map(&q.tmOut, Xn, n, m, p.batch, p.planes, p.pitch_n, 32, 32, sw64)) return false;
      break;
    }
  }
  q.tiles_per_matrix = gemm_tiles_per_matrix(q.M, q.N, q.sym);
  q.k_tiles = (q.K + 63) / 64;
  return true;
}

// Spectral cap of one group: per-matrix top singular vectors of the pre-step W
// (u: length rows, v: length cols) and where the coefficients go.
struct CapSpec {
  const float* const* u;
  const float* const* v;
  float* alpha;  // device [batch]
};

muon_status ensure_aux(muon_ctx* c, size_t bytes, cudaStream_t s) {
  if (bytes <= c->aux_bytes) {
    note_capture(c, s);
    return MUON_OK;
  }
  const muon_status st = may_grow(c, s, "the scratch");
  if (st != MUON_OK) return st;
  MUON_CUDA(cudaDeviceSynchronize(), "sync before scratch growth");
  cudaFree(c->d_aux);
  c->d_aux = nullptr;
  c->aux_bytes = 0;
  if (cudaMalloc(&c->d_aux, bytes) != cudaSuccess) {
    note_alloc_failure();
    return MUON_ERR_ALLOC;
  }
  c->aux_bytes = bytes;
  return MUON_OK;
}

muon_status run(muon_ctx* c, std::vector<GroupPlan>& plans, const muon_hparams* hp, bool step,
                float eps, cudaStream_t s, const CapSpec* cap = nullptr, bool clear_status = true) {
  muon_status st = reserve(c, plans, s);
  if (st != MUON_OK) return st;
  if (cap != nullptr) {  // per-block partials of the cap coefficients, sized before any launch
    st = ensure_aux(c, sizeof(double) * plans[0].batch * cap_alpha_blocks(plans[0].m_rows), s);
    if (st != MUON_OK) return st;
  }
  int total = 0;
  for (auto& p : plans) total += p.batch;
  if (clear_status) MUON_CUDA(cudaMemsetAsync(c->d_status, 0, sizeof(int), s), "clear status");

  // K1: momentum / look-ahead / norm over the groups `gs` (one launch per run of groups that share
  // a dtype and fit the launch's pointer tables).
  auto k1 = [&](const std::vector<int>& gs, cudaStream_t strm) -> muon_status {
    size_t i = 0;
    while (i < gs.size()) {
      MomentumParams mp;
      std::memset(static_cast<void*>(&mp), 0, sizeof(mp));
      mp.beta = step ? hp->beta : 0.f;
      mp.gscale = step ? hp->grad_scale : 1.f;
      mp.nesterov = step ? hp->nesterov : 0;
      mp.eps = eps;
      const int f32 = plans[gs[i]].f32;
      int mats = 0;
      for (; i < gs.size() && mp.ngroups < MUON_MAX_GROUPS; ++i) {
        const GroupPlan& p = plans[gs[i]];
        if (p.f32 != f32 || mats + p.batch > MUON_MAX_BATCH) break;
        MomentumGroup& q = mp.grp[mp.ngroups++];
        q.mat0 = mats;
        for (int l = 0; l < p.batch; ++l) {
          mp.g[mats + l] = p.g[l];
          mp.m[mats + l] = step ? p.m[l] : nullptr;
        }
        mats += p.batch;
        q.batch = p.batch;
        q.rows = p.rows;
        q.cols = p.cols;
        q.nblk = p.nblk;
        q.pitch = p.pitch_n;
        q.x = ws_at(c, p.off_x[0]);
        q.x_plane = p.x_plane;
        q.x_mat = p.x_mat;
        q.partials = c->d_partials + p.part_off;
        q.counters = c->d_counters + p.mat_off;
        q.nu = c->d_nu + p.mat_off;
        q.scale1 = c->d_s1 + p.mat_off;
        q.scale2 = c->d_s2 + p.mat_off;
        q.flags = c->d_flags + p.mat_off;
      }
      const int slot = prof_begin(c, MUON_KERNEL_MOMENTUM, strm);
      MUON_CUDA(launch_momentum(mp, f32 != 0, step, f32 ? 3 : 1, strm), "momentum kernel");
      prof_end(c, slot, strm);
    }
    return MUON_OK;
  };
  // Both elementwise launches take the groups last to first (and, inside each launch, the
  // matrices last to first): the momentum pass then writes last the U the Newton-Schulz launch
  // reads first (group 0, matrix 0), and the apply reads first the iterates that launch wrote
  // last, while they are still in L2.
  std::vector<int> all_groups;
  for (int g = static_cast<int>(plans.size()) - 1; g >= 0; --g) all_groups.push_back(g);
  // k Newton-Schulz iterations.  One persistent launch runs every phase of
  // every group (as many as fit in one parameter block), ordered phase by phase;
  // per-(phase, matrix) counters let a tile start as soon as the previous phase
  // of its own matrix has landed.  MUON_LAUNCH=phase runs one launch per phase.
  std::vector<Phase> seq_ph;
  std::vector<int> seq_it;
  for (int it = 0; it < c->k; ++it) {
    for (int ph = PH_GRAM; ph <= PH_UPDATE; ++ph) {
      if (ph == PH_POLY && c->coeffs[3 * it + 2] == 0.f) continue;
      seq_ph.push_back(static_cast<Phase>(ph));
      seq_it.push_back(it);
    }
  }
  const bool persistent = !c->per_phase;
  const int signals_per_tile = kEpilogueWarps;
  const int ng = static_cast<int>(plans.size());
  const int nph = static_cast<int>(seq_ph.size());
  // Launch order of (group, phase) problems.  Persistent launches go group by
  // group: one group's X stays (mostly) L2-resident across its phases, and the
  // next group starts while the last phases of the previous one drain.  (Each
  // phase keeps the matrix order of the previous one, so a matrix's next phase
  // is dispatched a whole phase after its previous one; reversing the order for
  // L2 reuse measured slower because of those dependency waits.)  The per-phase
  // mode runs one launch per phase covering every group.
  struct Item { int g, pi; };
  std::vector<std::vector<Item>> launches;
  // Pipelined schedule (two or more groups, persistent kernel): one launch per group on the
  // caller's stream; the momentum pass of group g+1 and the apply of group g run on the side
  // stream beside them.  Groups whose momentum pass is transposed (tall W, shared-memory
  // tiles that cannot sit beside a GEMM CTA) go first, so the passes that overlap are the
  // ones that fit.
  const bool pipelined = c->overlap && persistent && ng >= 2 && cap == nullptr && c->side != nullptr;
  std::vector<int> order;
  for (int g = 0; g < ng; ++g)
    if (plans[g].transposed) order.push_back(g);
  for (int g = 0; g < ng; ++g)
    if (!plans[g].transposed) order.push_back(g);
  if (pipelined) {
    for (int g : order) {
      std::vector<Item> cur;
      for (int pi = 0; pi < nph; ++pi) cur.push_back({g, pi});
      launches.push_back(cur);
    }
  } else if (persistent) {
    std::vector<Item> cur;
    for (int g = 0; g < ng; ++g) {
      for (int pi = 0; pi < nph; ++pi) {
        if (static_cast<int>(cur.size()) == kMaxProblems) {
          launches.push_back(cur);
          cur.clear();
        }
        cur.push_back({g, pi});
      }
    }
    if (!cur.empty()) launches.push_back(cur);
  } else {
    for (int pi = 0; pi < nph; ++pi) {
      std::vector<Item> cur;
      for (int g = 0; g < ng; ++g) cur.push_back({g, pi});
      launches.push_back(cur);
    }
  }
  GemmParams gp;
  auto run_launch = [&](const std::vector<Item>& items, cudaStream_t strm) -> muon_status {
    std::memset(static_cast<void*>(&gp), 0, sizeof(gp));
    gp.status = c->d_status;
    int tiles = 0;
    int last_of_group[MUON_MAX_GROUPS];
    for (int g = 0; g < ng; ++g) last_of_group[g] = -1;
    for (const Item& itm : items) {
      GemmProblem& q = gp.prob[gp.nprob];
      if (!fill_problem(c, plans[itm.g], seq_ph[itm.pi], seq_it[itm.pi], q))
        return cuda_fail(cudaErrorInvalidValue, "tensor map encoding");
      q.tile_base = tiles;
      tiles += q.tiles_per_matrix * q.L;
      if (persistent) {
        q.done_self = c->d_done + static_cast<size_t>(gp.nprob) * MUON_MAX_BATCH;
        const int prev = last_of_group[itm.g];
        if (prev >= 0) {  // the previous phase of this group is in the same launch
          q.done_dep = gp.prob[prev].done_self;
          q.dep_target = static_cast<unsigned>(signals_per_tile * gp.prob[prev].tiles_per_matrix);
        }
        last_of_group[itm.g] = gp.nprob;
      }
      ++gp.nprob;
    }
    gp.total_tiles = tiles;
    if (persistent && c->drop_signal_once && gp.nprob > 1) {
      gp.drop_signal = 1;
      c->drop_signal_once = false;
    }
    if (persistent)
      MUON_CUDA(cudaMemsetAsync(c->d_done, 0, sizeof(unsigned) * gp.nprob * MUON_MAX_BATCH, strm), "clear counters");
    const int units = std::min(tiles, c->sm_count);
    const int kind = items.size() > static_cast<size_t>(ng) || persistent
                         ? MUON_KERNEL_NS_FUSED
                         : MUON_KERNEL_GRAM + (seq_ph[items[0].pi] - PH_GRAM);
    const int slot = prof_begin(c, kind, strm);
    MUON_CUDA(launch_gemm(gp, units, strm), "newton-schulz gemm");
    prof_end(c, slot, strm);
    return MUON_OK;
  };

  // K5: scale + decoupled decay applied to W (or the plain copy to Out) over the groups `gs`.
  auto k5 = [&](const std::vector<int>& gs, cudaStream_t strm) -> muon_status {
    size_t i = 0;
    while (i < gs.size()) {
      ApplyParams ap;
      std::memset(static_cast<void*>(&ap), 0, sizeof(ap));
      const int f32 = plans[gs[i]].f32;
      ap.planes = plans[gs[i]].planes;
      ap.apply = step ? 1 : 0;
      ap.decay = step ? 1.0f - hp->lr * hp->weight_decay : 1.0f;
      ap.status = c->d_status;
      int mats = 0;
      for (; i < gs.size() && ap.ngroups < MUON_MAX_GROUPS; ++i) {
        const GroupPlan& p = plans[gs[i]];
        if (p.f32 != f32 || mats + p.batch > MUON_MAX_BATCH) break;
        ApplyGroup& q = ap.grp[ap.ngroups++];
        q.mat0 = mats;
        for (int l = 0; l < p.batch; ++l) {
          ap.w[mats + l] = p.w[l];
          if (cap != nullptr) {
            ap.cu[mats + l] = cap->u[l];
            ap.cv[mats + l] = cap->v[l];
          }
        }
        mats += p.batch;
        q.batch = p.batch;
        q.rows = p.rows;
        q.cols = p.cols;
        q.nblk = momentum_blocks_per_matrix(p.rows, p.cols);
        q.o = ws_at(c, p.off_x[c->k & 1]);
        q.o_plane = p.x_plane;
        q.o_mat = p.x_mat;
        q.pitch = p.pitch_n;
        q.lrs = step ? hp->lr * shape_scale(p.rows, p.cols, hp->scale_mode) : 0.f;
        q.flags = step ? c->d_flags + p.mat_off : nullptr;
        q.alpha = cap != nullptr ? cap->alpha : nullptr;
      }
      const int slot = prof_begin(c, MUON_KERNEL_APPLY, strm);
      MUON_CUDA(launch_apply(ap, f32 != 0, strm), "apply kernel");
      prof_end(c, slot, strm);
    }
    return MUON_OK;
  };

  if (pipelined) {
    // caller's stream: K1(first), GEMM(first), GEMM(second) ..., K5(last)
    // side stream:     K1(second) ..., K5(first) ...
    st = k1({order[0]}, s);
    if (st != MUON_OK) return st;
    MUON_CUDA(cudaEventRecord(c->ev_fork, s), "fork");
    MUON_CUDA(cudaStreamWaitEvent(c->side, c->ev_fork, 0), "fork");
    for (int i = 1; i < ng; ++i) {
      st = k1({order[i]}, c->side);
      if (st != MUON_OK) return st;
      MUON_CUDA(cudaEventRecord(c->ev_k1[i], c->side), "momentum done");
    }
    for (int i = 0; i < ng; ++i) {
      if (i > 0) MUON_CUDA(cudaStreamWaitEvent(s, c->ev_k1[i], 0), "wait momentum");
      st = run_launch(launches[i], s);
      if (st != MUON_OK) return st;
      if (i + 1 < ng) {
        MUON_CUDA(cudaEventRecord(c->ev_gemm[i], s), "gemm done");
        MUON_CUDA(cudaStreamWaitEvent(c->side, c->ev_gemm[i], 0), "wait gemm");
        st = k5({order[i]}, c->side);
        if (st != MUON_OK) return st;
      }
    }
    st = k5({order[ng - 1]}, s);
    if (st != MUON_OK) return st;
    MUON_CUDA(cudaEventRecord(c->ev_join, c->side), "join");
    MUON_CUDA(cudaStreamWaitEvent(s, c->ev_join, 0), "join");
  } else {
    st = k1(all_groups, s);
    if (st != MUON_OK) return st;
    for (const auto& items : launches) {
      st = run_launch(items, s);
      if (st != MUON_OK) return st;
    }
    // Spectral cap: alpha_l = u_l^T O_l v_l from the final iterate (one group).
    if (cap != nullptr) {
      const GroupPlan& p = plans[0];
      CapParams cp;
      std::memset(static_cast<void*>(&cp), 0, sizeof(cp));
      for (int l = 0; l < p.batch; ++l) {
        cp.a[l] = p.transposed ? cap->v[l] : cap->u[l];  // wide rows are W's columns when tall
        cp.b[l] = p.transposed ? cap->u[l] : cap->v[l];
      }
      cp.o = ws_at(c, p.off_x[c->k & 1]);
      cp.o_plane = p.x_plane;
      cp.o_mat = p.x_mat;
      cp.pitch = p.pitch_n;
      cp.m = p.m_rows;
      cp.n = p.n_cols;
      cp.planes = p.planes;
      cp.partial = static_cast<double*>(c->d_aux);
      MUON_CUDA(launch_cap_alpha(cp, p.batch, cap->alpha, s), "cap coefficient");
    }
    st = k5(all_groups, s);
    if (st != MUON_OK) return st;
  }
  c->last_count = total;
  c->last_stream = s;
  c->pending = true;
  c->out_nu = c->d_nu;
  c->out_flags = c->d_flags;
  return MUON_OK;
}

muon_status validate_and_plan(muon_ctx* c, const muon_group* groups, int ngroups, bool step,
                              std::vector<GroupPlan>& plans) {
  if (!c || !groups || ngroups < 1 || ngroups > MUON_MAX_GROUPS) return MUON_ERR_INVALID_ARG;
  plans.clear();
  for (int i = 0; i < ngroups; ++i) {
    muon_status st = check_group(groups[i], step);
    if (st != MUON_OK) return st;
    plans.push_back(plan_group(groups[i]));
  }
  return MUON_OK;
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

int muon_abi_version(void) { return MUON_ABI_VERSION; }

const char* muon_status_string(muon_status s) {
  switch (s) {
    case MUON_OK: return "MUON_OK";
    case MUON_ERR_INVALID_ARG: return "MUON_ERR_INVALID_ARG";
    case MUON_ERR_UNSUPPORTED_SHAPE: return "MUON_ERR_UNSUPPORTED_SHAPE";
    case MUON_ERR_DTYPE: return "MUON_ERR_DTYPE";
    case MUON_ERR_CUDA: return "MUON_ERR_CUDA";
    case MUON_ERR_NONFINITE: return "MUON_ERR_NONFINITE";
    case MUON_ERR_TIMEOUT: return "MUON_ERR_TIMEOUT";
    case MUON_ERR_NO_DEVICE: return "MUON_ERR_NO_DEVICE";
    case MUON_ERR_ALLOC: return "MUON_ERR_ALLOC";
  }
  return "MUON_ERR_UNKNOWN";
}

const char* muon_last_cuda_error(void) { return g_cuda_error; }

muon_status muon_create(muon_ctx** out, int device) {
  if (!out) return MUON_ERR_INVALID_ARG;
  *out = nullptr;
  int n = 0;
  if (cudaGetDeviceCount(&n) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return MUON_ERR_NO_DEVICE;
  }
  if (device < 0 || device >= n) return MUON_ERR_INVALID_ARG;
  cudaDeviceProp prop;
  MUON_CUDA(cudaGetDeviceProperties(&prop, device), "device properties");
  if (prop.major != 10) return MUON_ERR_NO_DEVICE;
  if (!get_encoder()) return MUON_ERR_NO_DEVICE;
  DeviceGuard guard(device);
  muon_ctx* c = new muon_ctx();
  c->device = device;
  c->sm_count = prop.multiProcessorCount;
  for (int i = 0; i < 5; ++i) std::memcpy(&c->coeffs[3 * i], kQuintic, sizeof(kQuintic));
  c->k = 5;

  if (const char* l = std::getenv("MUON_LAUNCH")) {
    if (std::strcmp(l, "phase") == 0) c->per_phase = true;
  }
  if (const char* d = std::getenv("MUON_TEST_DROP_SIGNAL")) {
    if (std::strcmp(d, "1") == 0) c->drop_signal_once = true;
  }
  if (const char* o = std::getenv("MUON_OVERLAP")) {
    if (std::strcmp(o, "1") == 0) c->overlap = true;
  }
  {
    int least = 0, greatest = 0;
    bool ok = cudaDeviceGetStreamPriorityRange(&least, &greatest) == cudaSuccess &&
              cudaStreamCreateWithPriority(&c->side, cudaStreamNonBlocking, least) == cudaSuccess &&
              cudaEventCreateWithFlags(&c->ev_fork, cudaEventDisableTiming) == cudaSuccess &&
              cudaEventCreateWithFlags(&c->ev_join, cudaEventDisableTiming) == cudaSuccess;
    for (int g = 0; ok && g < MUON_MAX_GROUPS; ++g)
      ok = cudaEventCreateWithFlags(&c->ev_k1[g], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&c->ev_gemm[g], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
      cudaGetLastError();
      if (c->side) cudaStreamDestroy(c->side);
      c->side = nullptr;  // everything runs on the caller's stream
    }
  }
  if (cudaMalloc(&c->d_status, sizeof(int)) != cudaSuccess) {
    note_alloc_failure();
    delete c;
    return MUON_ERR_ALLOC;
  }
  cudaMemset(c->d_status, 0, sizeof(int));
  if (cudaMalloc(&c->d_done, sizeof(unsigned) * kMaxProblems * MUON_MAX_BATCH) != cudaSuccess) {
    note_alloc_failure();
    cudaFree(c->d_status);
    delete c;
    return MUON_ERR_ALLOC;
  }
  *out = c;
  return MUON_OK;
}

muon_status muon_destroy(muon_ctx* c) {
  if (!c) return MUON_OK;
  DeviceGuard guard(c->device);
  cudaDeviceSynchronize();
  cudaFree(c->ws);
  cudaFree(c->d_nu);
  cudaFree(c->d_s1);
  cudaFree(c->d_s2);
  cudaFree(c->d_flags);
  cudaFree(c->d_counters);
  cudaFree(c->d_partials);
  cudaFree(c->d_status);
  cudaFree(c->d_done);
  cudaFree(c->d_stage);
  cudaFree(c->d_aux);
  cudaFree(c->d_nu_all);
  cudaFree(c->d_flags_all);
  for (cudaEvent_t e : c->copy_events) cudaEventDestroy(e);
  for (cudaEvent_t e : c->events) cudaEventDestroy(e);
  for (int g = 0; g < MUON_MAX_GROUPS; ++g) {
    if (c->ev_k1[g]) cudaEventDestroy(c->ev_k1[g]);
    if (c->ev_gemm[g]) cudaEventDestroy(c->ev_gemm[g]);
  }
  if (c->ev_fork) cudaEventDestroy(c->ev_fork);
  if (c->ev_join) cudaEventDestroy(c->ev_join);
  if (c->side) cudaStreamDestroy(c->side);
  delete c;
  return MUON_OK;
}

muon_status muon_set_coeffs(muon_ctx* c, const float* abc, int k) {
  if (!c || !abc || k < 1 || k > MUON_MAX_ITERS) return MUON_ERR_INVALID_ARG;
  for (int i = 0; i < 3 * k; ++i)
    if (!std::isfinite(abc[i])) return MUON_ERR_INVALID_ARG;
  std::memcpy(c->coeffs, abc, sizeof(float) * 3 * k);
  c->k = k;
  return MUON_OK;
}

muon_status muon_get_coeffs(const muon_ctx* c, float* abc, int* k) {
  if (!c || !abc || !k) return MUON_ERR_INVALID_ARG;
  std::memcpy(abc, c->coeffs, sizeof(float) * 3 * c->k);
  *k = c->k;
  return MUON_OK;
}

muon_status muon_step_groups(muon_ctx* c, const muon_group* groups, int ngroups,
                             const muon_hparams* hp, void* stream) {
  std::vector<GroupPlan> plans;
  muon_status st = validate_and_plan(c, groups, ngroups, true, plans);
  if (st != MUON_OK) return st;
  st = check_hparams(hp);
  if (st != MUON_OK) return st;
  DeviceGuard guard(c->device);
  return run(c, plans, hp, true, hp->eps, static_cast<cudaStream_t>(stream));
}

muon_status muon_step(muon_ctx* c, void* const* W, const void* const* G, float* const* M,
                      int batch, int rows, int cols, int dtype, const muon_hparams* hp,
                      void* stream) {
  muon_group g;
  g.W = W;
  g.G = G;
  g.M = M;
  g.batch = batch;
  g.rows = rows;
  g.cols = cols;
  g.dtype = dtype;
  return muon_step_groups(c, &g, 1, hp, stream);
}

muon_status muon_ns_orthogonalize(muon_ctx* c, const void* const* X, void* const* Out, int batch,
                                  int rows, int cols, int dtype, float eps, void* stream) {
  if (!std::isfinite(eps) || eps < 0.f) return MUON_ERR_INVALID_ARG;
  muon_group g;
  g.W = Out;
  g.G = X;
  g.M = nullptr;
  g.batch = batch;
  g.rows = rows;
  g.cols = cols;
  g.dtype = dtype;
  std::vector<GroupPlan> plans;
  muon_status st = validate_and_plan(c, &g, 1, false, plans);
  if (st != MUON_OK) return st;
  for (int l = 0; l < batch; ++l)
    if (Out[l] == X[l]) return MUON_ERR_INVALID_ARG;
  DeviceGuard guard(c->device);
  return run(c, plans, nullptr, false, eps, static_cast<cudaStream_t>(stream));
}

muon_status muon_get_status(muon_ctx* c, int* flags, int capacity, int* count) {
  if (!c || capacity < 0) return MUON_ERR_INVALID_ARG;
  DeviceGuard guard(c->device);
  if (count) *count = c->last_count;
  if (!c->pending) return MUON_OK;
  MUON_CUDA(cudaStreamSynchronize(c->last_stream), "stream synchronize");
  int status = 0;
  MUON_CUDA(cudaMemcpy(&status, c->d_status, sizeof(int), cudaMemcpyDeviceToHost), "read status");
  std::vector<int> f(c->last_count);
  if (c->last_count > 0)
    MUON_CUDA(cudaMemcpy(f.data(), c->out_flags, sizeof(int) * c->last_count, cudaMemcpyDeviceToHost),
              "read flags");
  if (flags) std::memcpy(flags, f.data(), sizeof(int) * std::min(capacity, c->last_count));
  if (status & kStatusTimeout) return MUON_ERR_TIMEOUT;
  for (int v : f)
    if (v & MUON_FLAG_NONFINITE) return MUON_ERR_NONFINITE;
  return MUON_OK;
}

muon_status muon_get_norms(muon_ctx* c, float* nu, int capacity, int* count) {
  if (!c || !nu || capacity < 0) return MUON_ERR_INVALID_ARG;
  DeviceGuard guard(c->device);
  if (count) *count = c->last_count;
  if (!c->pending || c->last_count == 0) return MUON_OK;
  MUON_CUDA(cudaStreamSynchronize(c->last_stream), "stream synchronize");
  MUON_CUDA(cudaMemcpy(nu, c->out_nu, sizeof(float) * std::min(capacity, c->last_count),
                       cudaMemcpyDeviceToHost),
            "read norms");
  return MUON_OK;
}

muon_status muon_step_groups_host(muon_ctx* c, const muon_group* groups, int ngroups,
                                  const muon_hparams* hp, float* nu_host, int* flags_host,
                                  void* stream) {
  if (!c || !groups || ngroups < 1 || ngroups > MUON_MAX_GROUPS) return MUON_ERR_INVALID_ARG;
  muon_status st = check_hparams(hp);
  if (st != MUON_OK) return st;
  size_t need = 0;
  for (int i = 0; i < ngroups; ++i) {
    st = check_group(groups[i], true);
    if (st != MUON_OK) return st;
    const size_t eb = groups[i].dtype == MUON_F32 ? 4 : 2;
    need += align_up(static_cast<size_t>(groups[i].rows) * groups[i].cols * eb, 256) * groups[i].batch;
  }
  DeviceGuard guard(c->device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (need > c->stage_bytes) {
    MUON_CUDA(cudaStreamSynchronize(s), "sync before staging growth");
    cudaFree(c->d_stage);
    c->d_stage = nullptr;
    c->stage_bytes = 0;
    if (cudaMalloc(&c->d_stage, need) != cudaSuccess) {
      note_alloc_failure();
      return MUON_ERR_ALLOC;
    }
    c->stage_bytes = need;
  }
  // Staging slot of every matrix (256-byte aligned, group after group).
  std::vector<std::vector<const void*>> gptr(ngroups);
  std::vector<std::vector<size_t>> gbytes(ngroups);
  size_t off = 0;
  int total = 0;
  for (int i = 0; i < ngroups; ++i) {
    const size_t eb = groups[i].dtype == MUON_F32 ? 4 : 2;
    const size_t bytes = static_cast<size_t>(groups[i].rows) * groups[i].cols * eb;
    gptr[i].resize(groups[i].batch);
    gbytes[i].assign(groups[i].batch, bytes);
    for (int l = 0; l < groups[i].batch; ++l) {
      gptr[i][l] = static_cast<char*>(c->d_stage) + off;
      off += align_up(bytes, 256);
    }
    total += groups[i].batch;
  }
  if (c->side == nullptr) {
    // one stream: every upload, then one step over all groups
    std::vector<muon_group> dev(groups, groups + ngroups);
    for (int i = 0; i < ngroups; ++i) {
      for (int l = 0; l < groups[i].batch; ++l)
        MUON_CUDA(cudaMemcpyAsync(const_cast<void*>(gptr[i][l]), groups[i].G[l], gbytes[i][l],
                                  cudaMemcpyHostToDevice, s),
                  "gradient upload");
      dev[i].G = gptr[i].data();
    }
    std::vector<GroupPlan> plans;
    st = validate_and_plan(c, dev.data(), ngroups, true, plans);
    if (st != MUON_OK) return st;
    st = run(c, plans, hp, true, hp->eps, s);
    if (st != MUON_OK) return st;
  } else {
    // Slab pipeline: the uploads run on the side stream (copy engine) slab after slab while the
    // caller's stream steps each slab as soon as its gradients have landed, so the PCIe transfer of
    // slab k+1 overlaps the step of slab k.  A slab is up to ~32 MB of one group's gradients.
    constexpr size_t kSlabBytes = size_t(32) << 20;
    struct Slab { int g, l0, n; };
    std::vector<Slab> slabs;
    for (int i = 0; i < ngroups; ++i) {
      const size_t mb = std::max<size_t>(gbytes[i][0], 1);
      const int per = static_cast<int>(std::max<size_t>(1, kSlabBytes / mb));
      for (int l0 = 0; l0 < groups[i].batch; l0 += per)
        slabs.push_back({i, l0, std::min(per, groups[i].batch - l0)});
    }
    while (c->copy_events.size() < slabs.size()) {
      cudaEvent_t e;
      MUON_CUDA(cudaEventCreateWithFlags(&e, cudaEventDisableTiming), "event");
      c->copy_events.push_back(e);
    }
    if (total > c->cap_all) {
      MUON_CUDA(cudaStreamSynchronize(s), "sync before result growth");
      cudaFree(c->d_nu_all);
      cudaFree(c->d_flags_all);
      c->d_nu_all = nullptr;
      c->d_flags_all = nullptr;
      c->cap_all = 0;
      if (cudaMalloc(&c->d_nu_all, sizeof(float) * total) != cudaSuccess ||
          cudaMalloc(&c->d_flags_all, sizeof(int) * total) != cudaSuccess) {
        note_alloc_failure();
        return MUON_ERR_ALLOC;
      }
      c->cap_all = total;
    }
    // the uploads start once everything queued on the caller's stream (e.g. the previous step
    // still reading the staging buffer) is done
    MUON_CUDA(cudaEventRecord(c->ev_fork, s), "fork");
    MUON_CUDA(cudaStreamWaitEvent(c->side, c->ev_fork, 0), "fork");
    for (size_t k = 0; k < slabs.size(); ++k) {
      const Slab& sl = slabs[k];
      for (int l = sl.l0; l < sl.l0 + sl.n; ++l)
        MUON_CUDA(cudaMemcpyAsync(const_cast<void*>(gptr[sl.g][l]), groups[sl.g].G[l], gbytes[sl.g][l],
                                  cudaMemcpyHostToDevice, c->side),
                  "gradient upload");
      MUON_CUDA(cudaEventRecord(c->copy_events[k], c->side), "upload done");
    }
    int first = 0;
    std::vector<int> first_of_group(ngroups, 0);
    for (int i = 1; i < ngroups; ++i) first_of_group[i] = first_of_group[i - 1] + groups[i - 1].batch;
    for (size_t k = 0; k < slabs.size(); ++k) {
      const Slab& sl = slabs[k];
      MUON_CUDA(cudaStreamWaitEvent(s, c->copy_events[k], 0), "wait upload");
      muon_group sg = groups[sl.g];
      sg.W = groups[sl.g].W + sl.l0;
      sg.G = gptr[sl.g].data() + sl.l0;
      sg.M = groups[sl.g].M + sl.l0;
      sg.batch = sl.n;
      std::vector<GroupPlan> plans;
      st = validate_and_plan(c, &sg, 1, true, plans);
      if (st != MUON_OK) return st;
      st = run(c, plans, hp, true, hp->eps, s, nullptr, /*clear_status=*/k == 0);
      if (st != MUON_OK) return st;
      first = first_of_group[sl.g] + sl.l0;
      MUON_CUDA(cudaMemcpyAsync(c->d_nu_all + first, c->d_nu, sizeof(float) * sl.n, cudaMemcpyDeviceToDevice, s),
                "gather norms");
      MUON_CUDA(cudaMemcpyAsync(c->d_flags_all + first, c->d_flags, sizeof(int) * sl.n, cudaMemcpyDeviceToDevice,
                                s),
                "gather flags");
    }
    c->last_count = total;
    c->out_nu = c->d_nu_all;
    c->out_flags = c->d_flags_all;
  }
  if (nu_host)
    MUON_CUDA(cudaMemcpyAsync(nu_host, c->out_nu, sizeof(float) * c->last_count, cudaMemcpyDeviceToHost, s),
              "norm download");
  if (flags_host)
    MUON_CUDA(cudaMemcpyAsync(flags_host, c->out_flags, sizeof(int) * c->last_count, cudaMemcpyDeviceToHost, s),
              "flag download");
  MUON_CUDA(cudaStreamSynchronize(s), "stream synchronize");
  return muon_get_status(c, nullptr, 0, nullptr);
}

muon_status muon_power_iteration(muon_ctx* c, const void* const* W, float* const* u, float* const* v,
                                 float* sigma, int batch, int rows, int cols, int dtype, int iters,
                                 void* stream) {
  if (!c || !W || !u || !v || !sigma || batch < 1 || batch > MUON_MAX_BATCH || iters < 1 || iters > 10000)
    return MUON_ERR_INVALID_ARG;
  if (rows < 1 || cols < 1) return MUON_ERR_INVALID_ARG;
  if (rows > 32768 || cols > 32768) return MUON_ERR_UNSUPPORTED_SHAPE;
  if (dtype != MUON_BF16 && dtype != MUON_F32) return MUON_ERR_DTYPE;
  for (int l = 0; l < batch; ++l)
    if (!W[l] || !u[l] || !v[l]) return MUON_ERR_INVALID_ARG;
  DeviceGuard guard(c->device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  GemvParams gp;
  std::memset(static_cast<void*>(&gp), 0, sizeof(gp));
  gp.rows = rows;
  gp.cols = cols;
  const bool f32 = dtype == MUON_F32;
  for (int l = 0; l < batch; ++l) gp.w[l] = W[l];
  bool fused = cols % 8 == 0 && cols <= power_pass_max_cols();
  for (int l = 0; l < batch && fused; ++l)
    if (reinterpret_cast<uintptr_t>(W[l]) % 16) fused = false;
  if (fused) {
    // one pass over W and one launch per iteration (power_stream_kernel)
    const int nblk = power_pass_blocks(rows, cols, batch, f32, c->sm_count);
    const size_t part_bytes = align_up(2 * sizeof(float) * batch * nblk * cols, 256);
    const size_t tsq_bytes = align_up(sizeof(float) * batch * nblk, 256);
    muon_status st = ensure_aux(c, part_bytes + tsq_bytes + 2 * sizeof(unsigned) * batch, s);
    if (st != MUON_OK) return st;
    gp.partial = static_cast<float*>(c->d_aux);
    float* tsq = reinterpret_cast<float*>(static_cast<char*>(c->d_aux) + part_bytes);
    unsigned* done = reinterpret_cast<unsigned*>(static_cast<char*>(c->d_aux) + part_bytes + tsq_bytes);
    for (int l = 0; l < batch; ++l) {
      gp.x[l] = v[l];
      gp.y[l] = u[l];
    }
    MUON_CUDA(launch_power_iteration_stream(gp, batch, f32, nblk, iters, tsq, done, sigma, c->d_status,
                                            c->sm_count, s),
              "power iteration");
    return MUON_OK;
  }
  gp.rows_per_chunk = 64;
  gp.row_chunks = (rows + 63) / 64;
  const size_t part_bytes = align_up(sizeof(float) * batch * gp.row_chunks * cols, 256);
  muon_status st = ensure_aux(c, part_bytes + sizeof(float) * MUON_MAX_BATCH, s);
  if (st != MUON_OK) return st;
  gp.partial = static_cast<float*>(c->d_aux);
  float* norms = reinterpret_cast<float*>(static_cast<char*>(c->d_aux) + part_bytes);
  MUON_CUDA(launch_normalize(v, batch, cols, norms, s), "normalise start vector");
  for (int i = 0; i < iters; ++i) {
    for (int l = 0; l < batch; ++l) {
      gp.x[l] = v[l];
      gp.y[l] = u[l];
    }
    MUON_CUDA(launch_gemv_rows(gp, batch, f32, s), "W v");
    MUON_CUDA(launch_normalize(u, batch, rows, norms, s), "normalise u");
    for (int l = 0; l < batch; ++l) {
      gp.x[l] = u[l];
      gp.y[l] = v[l];
    }
    MUON_CUDA(launch_gemv_cols(gp, batch, f32, s), "W^T u");
    MUON_CUDA(launch_normalize(v, batch, cols, sigma, s), "normalise v");
  }
  return MUON_OK;
}

muon_status muon_min_singular(muon_ctx* c, const void* const* W, float* const* y, const float* sigma_max,
                              float* sigma_min, int batch, int rows, int cols, int dtype, int iters, void* stream) {
  if (!c || !W || !y || !sigma_max || !sigma_min || batch < 1 || batch > MUON_MAX_BATCH || iters < 0 ||
      iters > 100000)
    return MUON_ERR_INVALID_ARG;
  if (rows < 1 || cols < 1) return MUON_ERR_INVALID_ARG;
  if (rows > 32768 || cols > 32768) return MUON_ERR_UNSUPPORTED_SHAPE;
  if (dtype != MUON_BF16 && dtype != MUON_F32) return MUON_ERR_DTYPE;
  for (int l = 0; l < batch; ++l)
    if (!W[l] || !y[l]) return MUON_ERR_INVALID_ARG;
  DeviceGuard guard(c->device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool tall = rows > cols;
  const int m = tall ? cols : rows, n = tall ? rows : cols;  // wide view X is m x n
  const bool f32 = dtype == MUON_F32;
  if (tall) {
    // X X^T y = W^T W y: one streaming pass over W per shifted step (power_stream_kernel with a
    // shift), all passes in one launch when its blocks fit on the GPU at once
    bool stream_ok = cols % 8 == 0 && cols <= power_pass_max_cols();
    for (int l = 0; l < batch && stream_ok; ++l)
      if (reinterpret_cast<uintptr_t>(W[l]) % 16) stream_ok = false;
    const int nblk = stream_ok ? power_pass_blocks(rows, cols, batch, f32, c->sm_count) : 0;
    if (stream_ok && (iters == 0 || power_pass_together(cols, f32, nblk, batch, c->sm_count))) {
      const size_t part_bytes = align_up(2 * sizeof(float) * batch * nblk * cols, 256);
      const size_t tsq_bytes = align_up(sizeof(float) * batch * nblk, 256);
      const size_t cnt_bytes = align_up(2 * sizeof(unsigned) * batch, 256);
      const size_t t_bytes = align_up(sizeof(float) * rows, 256);
      muon_status st = ensure_aux(c, part_bytes + tsq_bytes + cnt_bytes + batch * t_bytes, s);
      if (st != MUON_OK) return st;
      char* base = static_cast<char*>(c->d_aux);
      GemvParams sp;
      std::memset(static_cast<void*>(&sp), 0, sizeof(sp));
      sp.rows = rows;
      sp.cols = cols;
      sp.partial = reinterpret_cast<float*>(base);
      float* tsq = reinterpret_cast<float*>(base + part_bytes);
      unsigned* counters = reinterpret_cast<unsigned*>(base + part_bytes + tsq_bytes);
      for (int l = 0; l < batch; ++l) {
        sp.w[l] = W[l];
        sp.x[l] = y[l];
        sp.y[l] = reinterpret_cast<float*>(base + part_bytes + tsq_bytes + cnt_bytes + l * t_bytes);
      }
      const cudaError_t e = launch_power_iteration_stream(sp, batch, f32, nblk, iters + 1, tsq, counters,
                                                          sigma_min, c->d_status, c->sm_count, s, sigma_max);
      if (e == cudaSuccess) return MUON_OK;
      // no room for the cooperative launch after all (another client on the device): two GEMVs
      if (e != cudaErrorCooperativeLaunchTooLarge) return cuda_fail(e, "shifted iteration");
      (void)cudaGetLastError();
    }
  }
  if (!tall) {
    // X = W: one pass over W per shifted step, column slabs (colslab_kernel), one launch
    bool aligned = true;
    for (int l = 0; l < batch && aligned; ++l)
      if (reinterpret_cast<uintptr_t>(W[l]) % 16) aligned = false;
    const int S = aligned ? colslab_width(rows, cols, batch, f32, c->sm_count) : 0;
    if (S > 0) {
      const int nslab = cols / S;
      const size_t part_bytes = align_up(2 * sizeof(float) * batch * nslab * rows, 256);
      const size_t dsq_bytes = align_up(sizeof(float) * batch * nslab, 256);
      muon_status st = ensure_aux(c, part_bytes + dsq_bytes + 2 * sizeof(unsigned) * batch, s);
      if (st != MUON_OK) return st;
      char* base = static_cast<char*>(c->d_aux);
      GemvParams sp;
      std::memset(static_cast<void*>(&sp), 0, sizeof(sp));
      sp.rows = rows;
      sp.cols = cols;
      sp.partial = reinterpret_cast<float*>(base);
      for (int l = 0; l < batch; ++l) {
        sp.w[l] = W[l];
        sp.x[l] = y[l];
      }
      const cudaError_t e = launch_min_singular_slabs(sp, batch, f32, S, iters, sigma_max,
                                                      reinterpret_cast<float*>(base + part_bytes),
                                                      reinterpret_cast<unsigned*>(base + part_bytes + dsq_bytes),
                                                      sigma_min, c->d_status, s);
      if (e == cudaSuccess) return MUON_OK;
      // no room for the cooperative launch after all (another client on the device): two GEMVs
      if (e != cudaErrorCooperativeLaunchTooLarge) return cuda_fail(e, "shifted iteration (column slabs)");
      (void)cudaGetLastError();
    }
  }
  GemvParams gp;
  std::memset(static_cast<void*>(&gp), 0, sizeof(gp));
  gp.rows = rows;
  gp.cols = cols;
  gp.rows_per_chunk = 64;
  gp.row_chunks = (rows + 63) / 64;
  const size_t part_bytes = align_up(sizeof(float) * batch * gp.row_chunks * cols, 256);
  const size_t w_bytes = align_up(sizeof(float) * n, 256), z_bytes = align_up(sizeof(float) * m, 256);
  muon_status st = ensure_aux(c, part_bytes + batch * (w_bytes + z_bytes), s);
  if (st != MUON_OK) return st;
  char* base = static_cast<char*>(c->d_aux);
  gp.partial = reinterpret_cast<float*>(base);
  float* wv[MUON_MAX_BATCH];
  float* zv[MUON_MAX_BATCH];
  for (int l = 0; l < batch; ++l) {
    gp.w[l] = W[l];
    wv[l] = reinterpret_cast<float*>(base + part_bytes + l * w_bytes);
    zv[l] = reinterpret_cast<float*>(base + part_bytes + batch * w_bytes + l * z_bytes);
  }
  // out <- X^T in (length n) and out <- X in (length m), X the wide view of W
  auto apply_xt = [&](float* const* in, float* const* out) {
    for (int l = 0; l < batch; ++l) {
      gp.x[l] = in[l];
      gp.y[l] = out[l];
    }
    return tall ? launch_gemv_rows(gp, batch, f32, s) : launch_gemv_cols(gp, batch, f32, s);
  };
  auto apply_x = [&](float* const* in, float* const* out) {
    for (int l = 0; l < batch; ++l) {
      gp.x[l] = in[l];
      gp.y[l] = out[l];
    }
    return tall ? launch_gemv_cols(gp, batch, f32, s) : launch_gemv_rows(gp, batch, f32, s);
  };
  MUON_CUDA(launch_normalize(y, batch, m, nullptr, s), "normalise start vector");
  for (int i = 0; i < iters; ++i) {
    MUON_CUDA(apply_xt(y, wv), "X^T y");
    MUON_CUDA(apply_x(wv, zv), "X X^T y");
    MUON_CUDA(launch_shift_normalize(y, zv, batch, m, sigma_max, s), "shifted step");
  }
  MUON_CUDA(apply_xt(y, wv), "X^T y");
  MUON_CUDA(launch_normalize(wv, batch, n, sigma_min, s), "Rayleigh estimate");
  return MUON_OK;
}

muon_status muon_step_capped(muon_ctx* c, void* const* W, const void* const* G, float* const* M,
                             const float* const* u, const float* const* v, int batch, int rows, int cols,
                             int dtype, const muon_hparams* hp, float* alpha, void* stream) {
  if (!u || !v || !alpha) return MUON_ERR_INVALID_ARG;
  muon_group g;
  g.W = W;
  g.G = G;
  g.M = M;
  g.batch = batch;
  g.rows = rows;
  g.cols = cols;
  g.dtype = dtype;
  std::vector<GroupPlan> plans;
  muon_status st = validate_and_plan(c, &g, 1, true, plans);
  if (st != MUON_OK) return st;
  st = check_hparams(hp);
  if (st != MUON_OK) return st;
  for (int l = 0; l < batch; ++l)
    if (!u[l] || !v[l]) return MUON_ERR_INVALID_ARG;
  DeviceGuard guard(c->device);
  CapSpec cap{u, v, alpha};
  return run(c, plans, hp, true, hp->eps, static_cast<cudaStream_t>(stream), &cap);
}

size_t muon_workspace_bytes(const muon_ctx* c) {
  if (!c) return 0;
  return c->ws_bytes + c->stage_bytes + c->aux_bytes;
}

muon_status muon_profile_enable(muon_ctx* c, int on) {
  if (!c) return MUON_ERR_INVALID_ARG;
  c->profiling = on != 0;
  return MUON_OK;
}

muon_status muon_profile_read(muon_ctx* c, muon_profile* out, int reset) {
  if (!c || !out) return MUON_ERR_INVALID_ARG;
  DeviceGuard guard(c->device);
  std::memset(out, 0, sizeof(*out));
  for (size_t i = 0; i < c->rec_kind.size(); ++i) {
    MUON_CUDA(cudaEventSynchronize(c->events[2 * i + 1]), "profile event");
    float ms = 0.f;
    MUON_CUDA(cudaEventElapsedTime(&ms, c->events[2 * i], c->events[2 * i + 1]), "profile elapsed");
    out->launches[c->rec_kind[i]] += 1;
    out->ms[c->rec_kind[i]] += ms;
  }
  if (reset) c->rec_kind.clear();
  return MUON_OK;
}

}  // extern "C"
