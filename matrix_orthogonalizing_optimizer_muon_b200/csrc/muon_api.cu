// Host side of libmuon: the C ABI declared in include/muon.h.
//
// muon_init turns the list of parameter shapes into a plan: one device
// allocation that holds the Newton-Schulz workspace, the per-matrix
// descriptors, the tile schedules of every GEMM phase, the chunk schedule of
// the elementwise kernels and the TMA descriptors of every buffer.  A step is
// then a fixed sequence of launches on the caller's stream:
//   k1 (momentum, Nesterov input, Frobenius norm, bf16 split)
//   N x [Gram, polynomial, X update]   (tensor cores)
//   [Eq. 6 only: RMS(O) reduction]
//   the update pass (weight update, or O for muon_orthogonalize)
//   optional update-RMS finalisation.
// muon_step does not wait for the device except, rarely, to reuse the pinned
// staging of a pointer table; per-call device pointer tables are kept on the
// device (a few of them) and uploaded only when a call brings a new one.
#include "muon.h"
#include "muon_internal.cuh"

#include <cuda.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

using namespace muon;

namespace {

constexpr int kMaxDim = 65536;
constexpr int kMaxNsSteps = 32;
constexpr int kEventPool = 4096;
constexpr int kProfNs = 5;  // the Newton-Schulz phase of the profile (phases 1-3 together)

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D bf16 tensor map over a [rows, cols] array with row pitch `ld`
// elements; boxes of box_cols (contiguous) x box_rows, zero fill outside.
// 64-column boxes use the 128-byte swizzle (tensor-core operands), 32-column
// boxes the 64-byte swizzle (epilogue staging blocks).
bool encode_bf16_2d(CUtensorMap* tm, void* base, int rows, int cols, int ld, int box_cols, int box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle swz = box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swz, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 tensor map over two [rows, cols] arrays with the same pitch `ld`,
// the second `pair_bytes` after the first: boxes {32, 32, 2} move a 32 x 32
// block of both arrays at once; 64-byte swizzle.
bool encode_bf16_pair(CUtensorMap* tm, void* base, int rows, int cols, int ld, long long pair_bytes) {
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr || pair_bytes <= 0 || pair_bytes % 16 != 0) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows), 2};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld) * 2, static_cast<cuuint64_t>(pair_bytes)};
  const cuuint32_t box[3] = {32, 32, 2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D fp32 tensor map over `nparts` [rows, cols] arrays with row pitch `ld`,
// `part_bytes` apart: boxes {32, 32, 1}, 128-byte swizzle (the split-K parts).
bool encode_f32_parts(CUtensorMap* tm, void* base, int rows, int cols, int ld, long long part_bytes, int nparts) {
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr || part_bytes <= 0 || part_bytes % 16 != 0 || nparts < 1) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(nparts)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld) * 4, static_cast<cuuint64_t>(part_bytes)};
  const cuuint32_t box[3] = {32, 32, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool muon::pdl_enabled(unsigned cls) {
  static const unsigned mask = [] {
    const char* env = std::getenv("MUON_PDL");
    // default: the tensor-core launches only (on the elementwise passes the
    // attribute measured no faster on small plans and slower on large ones)
    return env != nullptr ? static_cast<unsigned>(std::atoi(env)) : static_cast<unsigned>(kPdlGemm);
  }();
  return (mask & cls) != 0;
}

// Operand maps (64 x 128 and 64 x 64 boxes) and epilogue store maps (32 x 32,
// hi and lo together) of one matrix's workspace arrays, in MapIndex order.
// lo must lie after hi0 and hi1 in memory.  Without split-K parts the part
// map repeats the A store map (it is never used then).
bool muon::encode_matrix_maps(void* maps, const MatInfo& mi, __nv_bfloat16* hi0, __nv_bfloat16* hi1,
                              __nv_bfloat16* lo, __nv_bfloat16* A, __nv_bfloat16* B, float* part,
                              int64_t part_stride, int nparts) {
  CUtensorMap* t = static_cast<CUtensorMap*>(maps);
  const int R = mi.rows, C = mi.cols, m = mi.m;
  const bool parts_ok = part != nullptr
                            ? encode_f32_parts(t + kMapStPart, part, m, m, mi.lda, part_stride * 4, nparts)
                            : encode_bf16_2d(t + kMapStPart, A, m, m, mi.lda, kEpiBoxCols, 32);
  return parts_ok && encode_bf16_2d(t + kMapHi0, hi0, R, C, mi.ld, kBoxInner, 128) &&
         encode_bf16_2d(t + kMapHi1, hi1, R, C, mi.ld, kBoxInner, 128) &&
         encode_bf16_2d(t + kMapA, A, m, m, mi.lda, kBoxInner, 128) &&
         encode_bf16_2d(t + kMapB, B, m, m, mi.lda, kBoxInner, 128) &&
         encode_bf16_2d(t + kMapHi0S, hi0, R, C, mi.ld, kBoxInner, 64) &&
         encode_bf16_2d(t + kMapHi1S, hi1, R, C, mi.ld, kBoxInner, 64) &&
         encode_bf16_2d(t + kMapAS, A, m, m, mi.lda, kBoxInner, 64) &&
         encode_bf16_2d(t + kMapBS, B, m, m, mi.lda, kBoxInner, 64) &&
         encode_bf16_pair(t + kMapStHiLo0, hi0, R, C, mi.ld, reinterpret_cast<char*>(lo) - reinterpret_cast<char*>(hi0)) &&
         encode_bf16_pair(t + kMapStHiLo1, hi1, R, C, mi.ld, reinterpret_cast<char*>(lo) - reinterpret_cast<char*>(hi1)) &&
         encode_bf16_2d(t + kMapStA, A, m, m, mi.lda, kEpiBoxCols, 32) &&
         encode_bf16_2d(t + kMapStB, B, m, m, mi.lda, kEpiBoxCols, 32);
}

namespace {

// The events of one profiled call: segment k lies between events
// first_event + k and first_event + k + 1 and its time goes to phase seg[k];
// launches[] counts the call's launches per phase.
struct ProfRec {
  int first_event = 0;
  std::vector<int> seg;
  int64_t launches[MUON_NUM_PHASES] = {};
};

// One wave of a plan: the matrices whose Newton-Schulz workspace is resident
// at the same time, and the ranges of the plan's schedules that cover them.
// A plan without a workspace cap has one wave holding every matrix.
struct Wave {
  int sym_off = 0, n_sym = 0;      // bf16 path, symmetric products
  int symg_off = 0, n_symg = 0;    // the Gram product's tiles with their split-K parts
  int red_off = 0, n_red = 0;      // split-K reduction blocks
  int full_off = 0, n_full = 0;    // bf16 path, X update
  int sym32_off = 0, n_sym32 = 0;  // fp32 path
  int full32_off = 0, n_full32 = 0;
  int chunk_off = 0, nchunks = 0;  // elementwise chunks
  int nmat = 0;
};

}  // namespace

struct muon_plan_s {
  int device = 0;
  int sm_count = 0;
  int npairs = 0;  // resident 2-CTA clusters of the tensor-core kernel
  int n = 0;
  uint32_t flags = 0;
  bool fp32_ws = false;
  std::vector<MatInfo> mats;
  // device memory
  uint8_t* dmem = nullptr;
  size_t dbytes = 0;
  Workspace ws{};
  MatInfo* mats_d = nullptr;
  TcTile* sym_d = nullptr;
  TcTile* full_d = nullptr;
  TileDesc* sym32_d = nullptr;
  TileDesc* full32_d = nullptr;
  int n_sym = 0, n_full = 0, n_sym32 = 0, n_full32 = 0;
  ChunkDesc* chunks_d = nullptr;
  int nchunks = 0;
  std::vector<Wave> waves;     // run one after another; their workspace is shared
  int split = 1;               // split-K parts of the Gram product (1: none)
  TcTile* symg_d = nullptr;    // the Gram tiles with their parts (split > 1)
  int4* reduce_d = nullptr;    // split-K reduction blocks, wave by wave
  uint64_t inject_wait_ns = 0; // failure-detection test: consumed by the next call's first GEMM launch
  void* tmaps_d = nullptr;
  // Per-call pointer tables, kept resident on the device: a call whose
  // pointers match a kept table uses it with no copy.  A caller that
  // alternates between buffer sets (double-buffered gradients) thus issues no
  // host-to-device copy per step; such a small copy would otherwise queue on
  // the copy engine behind the caller's own large input copies.
  struct PtrSlot {
    MatPtrs* dev = nullptr;     // device table
    MatPtrs* pinned = nullptr;  // staging of its last upload
    cudaEvent_t ev = nullptr;   // that upload has been read
    bool pending = false;
    bool valid = false;
    uint64_t last_use = 0;
    std::vector<MatPtrs> host;  // what the device table holds
  };
  static constexpr int kPtrSlots = 4;
  PtrSlot slots[kPtrSlots];
  MatPtrs* ptrs_d = nullptr;    // the table of the current call
  uint64_t use_clock = 0;
  cudaStream_t last_stream = nullptr;
  // profiling (0 off, MUON_PROFILE_LAUNCHES or MUON_PROFILE_SPANS)
  int prof = 0;
  std::vector<cudaEvent_t> events;
  int ev_next = 0;
  std::vector<ProfRec> recs;
  double prof_ms[MUON_NUM_PHASES] = {};
  int64_t prof_launches[MUON_NUM_PHASES] = {};
  int prof_calls = 0;
};

namespace {

muon_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? MUON_OK : MUON_ERR_CUDA; }

bool finite(float v) { return std::isfinite(v); }

// Make pl->ptrs_d a device table holding `t`: a kept table if one matches,
// else the least recently used slot, refilled by an asynchronous copy on `st`
// (stream order protects kernels of earlier calls still reading it).
muon_status_t upload_ptrs(muon_plan_s* pl, const std::vector<MatPtrs>& t, cudaStream_t st) {
  const size_t bytes = t.size() * sizeof(MatPtrs);
  muon_plan_s::PtrSlot* victim = nullptr;
  for (auto& sl : pl->slots) {
    if (sl.valid && std::memcmp(t.data(), sl.host.data(), bytes) == 0) {
      sl.last_use = ++pl->use_clock;
      pl->ptrs_d = sl.dev;
      return MUON_OK;
    }
    if (victim == nullptr || !sl.valid || (victim->valid && sl.last_use < victim->last_use)) victim = &sl;
  }
  if (victim->pending) {  // its staging buffer may still be read by the previous upload
    if (cudaEventSynchronize(victim->ev) != cudaSuccess) return MUON_ERR_CUDA;
    victim->pending = false;
  }
  std::memcpy(victim->pinned, t.data(), bytes);
  if (cudaMemcpyAsync(victim->dev, victim->pinned, bytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return MUON_ERR_CUDA;
  if (cudaEventRecord(victim->ev, st) != cudaSuccess) return MUON_ERR_CUDA;
  victim->pending = true;
  victim->host = t;
  victim->valid = true;
  victim->last_use = ++pl->use_clock;
  pl->ptrs_d = victim->dev;
  return MUON_OK;
}

// ------------------------------------------------------------ profiling
void prof_flush(muon_plan_s* pl) {
  for (const ProfRec& r : pl->recs) {
    const int nseg = static_cast<int>(r.seg.size());
    cudaEventSynchronize(pl->events[r.first_event + nseg]);
    for (int k = 0; k < nseg; ++k) {
      float ms = 0.0f;
      cudaEventElapsedTime(&ms, pl->events[r.first_event + k], pl->events[r.first_event + k + 1]);
      pl->prof_ms[r.seg[k]] += ms;
      if (r.seg[k] >= kPhaseGram + 1 && r.seg[k] <= kPhaseUpdate + 1) pl->prof_ms[kProfNs] += ms;
    }
    for (int p = 0; p < MUON_NUM_PHASES; ++p) pl->prof_launches[p] += r.launches[p];
    pl->prof_calls += 1;
  }
  pl->recs.clear();
  pl->ev_next = 0;
}

// Records a call's events.  mark(phase) follows every launch; in span mode a
// product launch records no event, and span_end() closes the products of a
// wave with one event whose segment goes to the Newton-Schulz phase.
struct Recorder {
  muon_plan_s* pl;
  cudaStream_t st;
  ProfRec rec{};
  bool on = false;
  bool spans = false;
  int open = 0;  // launches since the last event
  Recorder(muon_plan_s* p, cudaStream_t s, int max_launches) : pl(p), st(s) {
    if (pl->prof == 0) return;
    spans = pl->prof == MUON_PROFILE_SPANS;
    if (max_launches + 1 > static_cast<int>(pl->events.size())) pl->events.resize(max_launches + 1, nullptr);
    for (auto& ev : pl->events)
      if (ev == nullptr && cudaEventCreate(&ev) != cudaSuccess) return;
    if (pl->ev_next + max_launches + 1 > static_cast<int>(pl->events.size())) prof_flush(pl);
    rec.first_event = pl->ev_next;
    rec.seg.reserve(max_launches);
    cudaEventRecord(pl->events[pl->ev_next++], st);
    on = true;
  }
  void close(int phase) {
    rec.seg.push_back(phase);
    open = 0;
    cudaEventRecord(pl->events[pl->ev_next++], st);
  }
  void mark(int phase) {
    if (!on) return;
    rec.launches[phase] += 1;
    if (phase >= kPhaseGram + 1 && phase <= kPhaseUpdate + 1) rec.launches[kProfNs] += 1;
    ++open;
    if (spans && phase >= kPhaseGram + 1 && phase <= kPhaseUpdate + 1) return;
    close(phase);
  }
  void span_end() {
    if (on && spans && open > 0) close(kProfNs);
  }
  ~Recorder() {
    if (on) pl->recs.push_back(rec);
  }
};

// ------------------------------------------------------------ the launch sequence
// The launch sequence of one call: for each wave, k1 over its chunks, the
// Newton-Schulz launches over its tiles and the update pass over its chunks
// (every matrix's arithmetic is the same whichever wave holds it), then the
// RMS finalisation over all matrices.
muon_status_t run_ns(muon_plan_s* pl, const StepScalars& sc, int ns_steps, int precision, int final_mode,
                     int k1_mode, float* update_rms, cudaStream_t st) {
  const int nwave = static_cast<int>(pl->waves.size());
  Recorder rec(pl, st, nwave * (3 * ns_steps + 3) + 1);
  const int fp32 = precision == MUON_NS_FP32 ? 1 : 0;
  // The last iterate is in hi[cur]/lo (x32[cur]); O = s X when N = 0.  Eq. 6
  // needs RMS(O) before any weight changes, so it adds a reduction pass.
  const int mul_s = ns_steps == 0 ? 1 : 0;
  const bool norm_pass = (final_mode == kFinalWeight && sc.scale_mode == kScaleUpdateNorm);
  cudaError_t e = cudaSuccess;
  for (const Wave& w : pl->waves) {
    const ChunkDesc* chunks = pl->chunks_d + w.chunk_off;
    e = launch_k1(chunks, w.nchunks, pl->mats_d, pl->ptrs_d, pl->ws, sc, k1_mode, fp32, st);
    if (e != cudaSuccess) return MUON_ERR_CUDA;
    rec.mark(0);
    int cur = 0;
    for (int it = 0; it < ns_steps; ++it) {
      for (int ph = kPhaseGram; ph <= kPhaseUpdate; ++ph) {
        if (fp32) {
          Gemm32Args a{};
          a.tiles = (ph == kPhaseUpdate) ? pl->full32_d + w.full32_off : pl->sym32_d + w.sym32_off;
          a.ntiles = (ph == kPhaseUpdate) ? w.n_full32 : w.n_sym32;
          a.phase = ph;
          a.iter = it;
          a.cur = cur;
          a.mats = pl->mats_d;
          a.ptrs = pl->ptrs_d;
          a.ws = pl->ws;
          a.sc = sc;
          e = launch_gemm_f32(a, st);
        } else {
          GemmArgs a{};
          const bool gsplit = (ph == kPhaseGram && pl->split > 1);
          a.tiles = (ph == kPhaseUpdate) ? pl->full_d + w.full_off
                                         : (gsplit ? pl->symg_d + w.symg_off : pl->sym_d + w.sym_off);
          a.ntiles = (ph == kPhaseUpdate) ? w.n_full : (gsplit ? w.n_symg : w.n_sym);
          a.phase = ph;
          a.iter = it;
          a.cur = cur;
          a.mats = pl->mats_d;
          a.ptrs = pl->ptrs_d;
          a.tmaps = pl->tmaps_d;
          a.ws = pl->ws;
          a.sc = sc;
          a.test_wait_ns = pl->inject_wait_ns;
          a.split = gsplit ? pl->split : 1;
          pl->inject_wait_ns = 0;
          e = launch_gemm_tc(a, pl->npairs, st);
          if (e == cudaSuccess && a.split > 1)
            e = launch_split_reduce(pl->reduce_d + w.red_off, w.n_red, pl->mats_d, pl->ws, sc, ph, it, a.split, st);
        }
        if (e != cudaSuccess) return MUON_ERR_CUDA;
        rec.mark(1 + ph);
      }
      cur ^= 1;  // the X update wrote the other buffer
    }
    rec.span_end();
    if (norm_pass) {
      e = launch_update_norm(chunks, w.nchunks, pl->mats_d, pl->ws, sc, fp32, cur, mul_s, update_rms, st);
      if (e != cudaSuccess) return MUON_ERR_CUDA;
      rec.mark(4);
    }
    e = launch_apply_update(chunks, w.nchunks, pl->mats_d, pl->ptrs_d, pl->ws, sc, final_mode, fp32, cur, mul_s,
                            st);
    if (e != cudaSuccess) return MUON_ERR_CUDA;
    rec.mark(4);
  }
  if (update_rms != nullptr && !norm_pass) {
    e = launch_rms_finalize(pl->mats_d, pl->n, pl->ws.rms_part, update_rms, st);
    if (e != cudaSuccess) return MUON_ERR_CUDA;
    rec.mark(4);
  }
  return MUON_OK;
}

void free_plan(muon_plan_s* pl) {
  if (pl == nullptr) return;
  if (pl->dmem) cudaFree(pl->dmem);
  for (auto& sl : pl->slots) {
    if (sl.pinned) cudaFreeHost(sl.pinned);
    if (sl.ev) cudaEventDestroy(sl.ev);
  }
  for (cudaEvent_t ev : pl->events)
    if (ev != nullptr) cudaEventDestroy(ev);
  delete pl;
}

}  // namespace

extern "C" {

const char* muon_status_string(muon_status_t s) {
  switch (s) {
    case MUON_OK: return "ok";
    case MUON_ERR_INVALID_ARG: return "invalid argument";
    case MUON_ERR_SHAPE_MISMATCH: return "descriptor count or shape differs from the plan";
    case MUON_ERR_UNSUPPORTED: return "unsupported request for this plan or device";
    case MUON_ERR_NO_MEMORY: return "out of memory";
    case MUON_ERR_CUDA: return "CUDA error";
    case MUON_ERR_NONFINITE: return "non-finite Frobenius norm";
    case MUON_ERR_TIMEOUT: return "device-side wait timed out";
    case MUON_ERR_ALIAS: return "buffers overlap";
    case MUON_ERR_NOT_CONVERGED: return "eigenvalue iteration did not converge";
  }
  return "unknown status";
}

muon_status_t muon_hparams_default(muon_hparams_t* hp) {
  if (hp == nullptr) return MUON_ERR_INVALID_ARG;
  hp->lr = 4.2e-4f;
  hp->weight_decay = 0.1f;
  hp->momentum = 0.95f;
  hp->ns_steps = 5;
  hp->a = 3.4445f;
  hp->b = -4.7750f;
  hp->c = 2.0315f;
  hp->rms_scale = 0.2f;
  hp->nesterov = 1;
  hp->ns_precision = MUON_NS_BF16;
  hp->scale_mode = MUON_SCALE_MAX_DIM;
  hp->hidden_dim = 0.0f;
  return MUON_OK;
}

muon_status_t muon_init(muon_plan_t* out, const muon_param_t* params, int32_t n, uint32_t flags, void* stream) {
  if (out != nullptr) *out = nullptr;
  if (flags & MUON_INIT_MAX_WORKSPACE) return MUON_ERR_INVALID_ARG;  // the budget needs muon_init_ex
  return muon_init_ex(out, params, n, flags, 0, stream);
}

muon_status_t muon_init_ex(muon_plan_t* out, const muon_param_t* params, int32_t n, uint32_t flags,
                           size_t max_workspace_bytes, void* stream) {
  if (out == nullptr) return MUON_ERR_INVALID_ARG;
  *out = nullptr;
  if (params == nullptr || n < 1 || n > (1 << 20)) return MUON_ERR_INVALID_ARG;
  if (flags & ~(MUON_INIT_ZERO_MOMENTUM | MUON_INIT_FP32_NS | MUON_INIT_MAX_WORKSPACE)) return MUON_ERR_INVALID_ARG;
  const bool capped = (flags & MUON_INIT_MAX_WORKSPACE) != 0;
  if (capped != (max_workspace_bytes != 0)) return MUON_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    const muon_param_t& p = params[i];
    if (p.rows < 1 || p.cols < 1 || p.rows > kMaxDim || p.cols > kMaxDim || p.reserved != 0)
      return MUON_ERR_INVALID_ARG;
    if ((flags & MUON_INIT_ZERO_MOMENTUM) && p.M == nullptr) return MUON_ERR_INVALID_ARG;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MUON_ERR_CUDA;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MUON_ERR_CUDA;
  if (prop.major != 10 || prop.minor != 0) return MUON_ERR_UNSUPPORTED;
  if (get_encode_fn() == nullptr) return MUON_ERR_CUDA;

  muon_plan_s* pl = new (std::nothrow) muon_plan_s();
  if (pl == nullptr) return MUON_ERR_NO_MEMORY;
  pl->device = dev;
  pl->sm_count = prop.multiProcessorCount;
  // persistent grid of the tensor-core kernel: as many 2-CTA clusters as can be
  // resident (clusters never wait on each other, so more would only queue)
  pl->npairs = gemm_tc_max_pairs();
  if (pl->npairs < 1) pl->npairs = std::max(1, pl->sm_count / 2);
  if (const char* env = std::getenv("MUON_TC_PAIRS")) {  // diagnostic: cap the persistent grid
    const int v = std::atoi(env);
    if (v >= 1 && v < pl->npairs) pl->npairs = v;
  }
  pl->n = n;
  pl->flags = flags;
  pl->fp32_ws = (flags & MUON_INIT_FP32_NS) != 0;
  pl->mats.resize(n);

  // ---- per-matrix shapes and workspace sizes (elements of the [R, ld] and [m, lda] arrays)
  std::vector<size_t> xel(n), ael(n);
  for (int i = 0; i < n; ++i) {
    MatInfo& mi = pl->mats[i];
    const int R = static_cast<int>(params[i].rows), C = static_cast<int>(params[i].cols);
    mi.rows = R;
    mi.cols = C;
    mi.m = std::min(R, C);
    mi.n = std::max(R, C);
    mi.tall = R > C ? 1 : 0;
    mi.ld = static_cast<int>(round_up(C, 8));
    mi.lda = static_cast<int>(round_up(mi.m, 8));
    xel[i] = round_up(static_cast<size_t>(R) * mi.ld, 128);
    ael[i] = round_up(static_cast<size_t>(mi.m) * mi.lda, 128);
  }
  // bytes per element of the iterate arrays (hi0, hi1, lo; + x32[2]) and of the
  // symmetric arrays (A, B; + a32, b32)
  size_t bx = pl->fp32_ws ? 6 + 8 : 6, ba = pl->fp32_ws ? 4 + 8 : 4;
  // LPT order of matrices (largest Newton-Schulz work first): the order of the
  // GEMM schedules and of the wave packing
  std::vector<int> order(n);
  for (int i = 0; i < n; ++i) order[i] = i;
  auto work = [&](int i) {
    const double m = static_cast<double>(pl->mats[i].m), nn = static_cast<double>(pl->mats[i].n);
    return m * m * nn + m * m * m;
  };
  std::stable_sort(order.begin(), order.end(), [&](int x, int y) { return work(x) > work(y); });

  // ---- the small device structures every plan holds, whatever its waves
  std::vector<TcTile> sym, symg, full;
  std::vector<TileDesc> sym32, full32;
  std::vector<int4> red;
  std::vector<ChunkDesc> chunks;
  std::vector<int> wave_of(n, 0);
  auto fixed_bytes = [&](size_t ntile_sym, size_t ntile_full, size_t ntile_sym32, size_t ntile_full32,
                         size_t nchunk) {
    size_t b = 0;
    auto add = [&](size_t v) { b += round_up(v, 256); };
    add(n * sizeof(float));                          // s
    add(nchunk * sizeof(double));                    // norm partials
    add(n * sizeof(unsigned));                       // arrival counters
    add(nchunk * sizeof(float));                     // update partials
    add(sizeof(unsigned));                           // status
    add(n * sizeof(float));                          // Eq. 6 factors
    add(n * sizeof(MatInfo));
    add(muon_plan_s::kPtrSlots * n * sizeof(MatPtrs));
    add(std::max<size_t>(1, ntile_sym) * sizeof(TcTile));
    add(std::max<size_t>(1, ntile_full) * sizeof(TcTile));
    add(std::max<size_t>(1, ntile_sym32) * sizeof(TileDesc));
    add(std::max<size_t>(1, ntile_full32) * sizeof(TileDesc));
    add(nchunk * sizeof(ChunkDesc));
    add(static_cast<size_t>(n) * kMapsPerMat * sizeof(CUtensorMap));
    return b;
  };
  // tile and chunk counts do not depend on the waves
  size_t cnt_sym = 0, cnt_full = 0, cnt_sym32 = 0, cnt_full32 = 0, cnt_chunk = 0;
  for (int i = 0; i < n; ++i) {
    const MatInfo& mi = pl->mats[i];
    for_each_sym_tile(mi.m, [&](const TcTile&) { ++cnt_sym; });
    for_each_full_tile(mi.rows, mi.cols, [&](const TcTile&) { ++cnt_full; });
    if (pl->fp32_ws) {
      cnt_sym32 += static_cast<size_t>((mi.m + kT32 - 1) / kT32) * ((mi.m + kT32 - 1) / kT32);
      cnt_full32 += static_cast<size_t>((mi.rows + kT32 - 1) / kT32) * ((mi.cols + kT32 - 1) / kT32);
    }
    const int rows_per_chunk = std::max(1, kChunkElems / mi.cols);
    cnt_chunk += (mi.rows + rows_per_chunk - 1) / rows_per_chunk;
  }
  // ---- split K of the Gram product: a plan whose symmetric launches hold
  // too few tiles to fill the CTA pairs, and whose Gram products have a long
  // K (= n), splits each Gram tile's K range into 2 or 4 parts (fp32 partial
  // products, then a fixed-order reduction) while every part keeps at least
  // 32 stages; shorter parts measured no faster than the unsplit product.
  // The choice depends on the plan's shapes only, so every wave of a capped
  // plan makes the same one.
  {
    int nk_min = 1 << 30;
    for (int i = 0; i < n; ++i) nk_min = std::min(nk_min, (pl->mats[i].n + kBK - 1) / kBK);
    int split = 1;
    for (int sp : {4, 2})
      if (cnt_sym * sp * 5 <= static_cast<size_t>(pl->npairs) * 6 && nk_min >= 32 * sp) {
        split = sp;
        break;
      }
    if (const char* env = std::getenv("MUON_SPLITK")) {  // diagnostic: force the split (1, 2 or 4)
      const int v = std::atoi(env);
      if ((v == 1 || v == 2 || v == 4) && nk_min >= 4 * v) split = v;
    }
    pl->split = split;
  }
  const int split = pl->split;
  // ---- split N of the symmetric and X-update tiles: a plan whose launches
  // hold at most half as many tiles as CTA pairs halves its tiles along N
  // (256 -> 128 -> 64 columns) while the count still gives each pair at most
  // one, so that more pairs share a latency-bound launch.  The Gram product
  // of a K-split plan keeps its unsplit tiles.
  int nsplit_sym = 0, nsplit_full = 0;
  {
    auto levels = [&](size_t count) {
      int lv = 0;
      while (lv < 2 && count * 2 <= static_cast<size_t>(pl->npairs)) {
        ++lv;
        count *= 2;
      }
      return lv;
    };
    nsplit_sym = levels(cnt_sym);
    nsplit_full = levels(cnt_full);
    if (const char* env = std::getenv("MUON_NSPLIT")) {  // diagnostic: force the levels (0, 1 or 2)
      const int v = std::atoi(env);
      if (v >= 0 && v <= 2) nsplit_sym = nsplit_full = v;
    }
  }
  size_t cnt_sym_n = 0, cnt_full_n = 0;  // list sizes after the N split
  for (int i = 0; i < n; ++i) {
    const MatInfo& mi = pl->mats[i];
    for_each_sym_tile(mi.m, [&](const TcTile& t) {
      split_n(t, nsplit_sym, mi.m, [&](const TcTile&) { ++cnt_sym_n; });
    });
    for_each_full_tile(mi.rows, mi.cols, [&](const TcTile& t) {
      split_n(t, nsplit_full, mi.cols, [&](const TcTile&) { ++cnt_full_n; });
    });
  }
  size_t cnt_red = 0;  // 32 x 32 blocks on or below the diagonal of every symmetric product
  if (split > 1)
    for (int i = 0; i < n; ++i) {
      const size_t b = (pl->mats[i].m + 31) / 32;
      cnt_red += b * (b + 1) / 2;
    }
  const size_t fixed = fixed_bytes(cnt_sym_n, cnt_full_n, cnt_sym32, cnt_full32, cnt_chunk) +
                       round_up(cnt_red * sizeof(int4), 256) +
                       (split > 1 ? round_up(cnt_sym * split * sizeof(TcTile), 256) : 0);

  if (split > 1) ba += 4 * static_cast<size_t>(split);  // fp32 parts of the symmetric products
  // ---- waves: with a workspace cap, matrices are packed first-fit in LPT
  // order into waves whose iterate and symmetric arrays fit what the cap
  // leaves after the fixed structures.  The arrays are shared by all waves and
  // sized by the largest wave of each kind, so the packing is repeated with a
  // tighter capacity until the total fits.
  size_t X_total = 0, A_total = 0;
  int nwave = 1;
  if (!capped) {
    for (int i = 0; i < n; ++i) {
      X_total += xel[i];
      A_total += ael[i];
    }
  } else {
    const size_t slack = 6 * 256;  // alignment of the iterate and symmetric arrays
    if (max_workspace_bytes <= fixed + slack) {
      free_plan(pl);
      return MUON_ERR_NO_MEMORY;
    }
    size_t cap = max_workspace_bytes - fixed - slack;
    size_t biggest = 0;
    for (int i = 0; i < n; ++i) biggest = std::max(biggest, bx * xel[i] + ba * ael[i]);
    bool fits = false;
    for (int attempt = 0; attempt < 64 && cap >= biggest; ++attempt) {
      std::vector<size_t> wx, wa;
      for (int i : order) {
        const size_t need = bx * xel[i] + ba * ael[i];
        int w = 0;
        while (w < static_cast<int>(wx.size()) && bx * wx[w] + ba * wa[w] + need > cap) ++w;
        if (w == static_cast<int>(wx.size())) {
          wx.push_back(0);
          wa.push_back(0);
        }
        wx[w] += xel[i];
        wa[w] += ael[i];
        wave_of[i] = w;
      }
      X_total = *std::max_element(wx.begin(), wx.end());
      A_total = *std::max_element(wa.begin(), wa.end());
      nwave = static_cast<int>(wx.size());
      const size_t total = bx * X_total + ba * A_total;
      if (total <= max_workspace_bytes - fixed - slack) {
        fits = true;
        break;
      }
      const size_t over = total - (max_workspace_bytes - fixed - slack);
      cap = cap > over ? cap - over : 0;
    }
    if (!fits) {
      free_plan(pl);
      return MUON_ERR_NO_MEMORY;
    }
  }

  // ---- per-wave offsets, chunk lists and tile schedules (LPT order inside a wave)
  pl->waves.assign(nwave, Wave{});
  {
    std::vector<size_t> xoff(nwave, 0), aoff(nwave, 0);
    for (int i = 0; i < n; ++i) {  // descriptor order inside a wave
      MatInfo& mi = pl->mats[i];
      const int w = wave_of[i];
      mi.off_x = static_cast<int64_t>(xoff[w]);
      mi.off_a = static_cast<int64_t>(aoff[w]);
      xoff[w] += xel[i];
      aoff[w] += ael[i];
      pl->waves[w].nmat += 1;
    }
  }
  for (int w = 0; w < nwave; ++w) {
    Wave& wv = pl->waves[w];
    wv.chunk_off = static_cast<int>(chunks.size());
    for (int i = 0; i < n; ++i) {  // descriptor order inside a wave
      if (wave_of[i] != w) continue;
      MatInfo& mi = pl->mats[i];
      const int rows_per_chunk = std::max(1, kChunkElems / mi.cols);
      mi.chunk_base = static_cast<int>(chunks.size());
      for (int r = 0; r < mi.rows; r += rows_per_chunk)
        chunks.push_back(make_int4(i, r, std::min(rows_per_chunk, mi.rows - r), static_cast<int>(chunks.size())));
      mi.nchunks = static_cast<int>(chunks.size()) - mi.chunk_base;
    }
    wv.nchunks = static_cast<int>(chunks.size()) - wv.chunk_off;
    wv.sym_off = static_cast<int>(sym.size());
    wv.symg_off = static_cast<int>(symg.size());
    wv.full_off = static_cast<int>(full.size());
    wv.sym32_off = static_cast<int>(sym32.size());
    wv.full32_off = static_cast<int>(full32.size());
    for (int i : order) {
      if (wave_of[i] != w) continue;
      const MatInfo& mi = pl->mats[i];
      for_each_sym_tile(mi.m, [&](TcTile t) {
        t.p = i;
        split_n(t, nsplit_sym, mi.m, [&](const TcTile& piece) { sym.push_back(piece); });
        if (split > 1)
          for (int kp = 0; kp < split; ++kp) {  // the parts of a tile side by side
            t.kpart = kp;
            symg.push_back(t);
          }
      });
      for_each_full_tile(mi.rows, mi.cols, [&](TcTile t) {
        t.p = i;
        split_n(t, nsplit_full, mi.cols, [&](const TcTile& piece) { full.push_back(piece); });
      });
      if (pl->fp32_ws) {
        for (int r0 = 0; r0 < mi.m; r0 += kT32)
          for (int c0 = 0; c0 < mi.m; c0 += kT32) sym32.push_back(make_int4(i, r0, c0, 0));
        for (int r0 = 0; r0 < mi.rows; r0 += kT32)
          for (int c0 = 0; c0 < mi.cols; c0 += kT32) full32.push_back(make_int4(i, r0, c0, 0));
      }
    }
    wv.n_sym = static_cast<int>(sym.size()) - wv.sym_off;
    wv.n_symg = static_cast<int>(symg.size()) - wv.symg_off;
    wv.red_off = static_cast<int>(red.size());
    if (split > 1)
      for (int i : order) {
        if (wave_of[i] != w) continue;
        const int m = pl->mats[i].m;
        for (int i0 = 0; i0 < m; i0 += 32)
          for (int j0 = 0; j0 <= i0; j0 += 32) red.push_back(make_int4(i, i0, j0, 0));
      }
    wv.n_red = static_cast<int>(red.size()) - wv.red_off;
    wv.n_full = static_cast<int>(full.size()) - wv.full_off;
    wv.n_sym32 = static_cast<int>(sym32.size()) - wv.sym32_off;
    wv.n_full32 = static_cast<int>(full32.size()) - wv.full32_off;
  }
  pl->n_sym = static_cast<int>(sym.size());
  pl->n_full = static_cast<int>(full.size());
  pl->n_sym32 = static_cast<int>(sym32.size());
  pl->n_full32 = static_cast<int>(full32.size());
  pl->nchunks = static_cast<int>(chunks.size());
  const size_t total_x = X_total, total_a = A_total;

  // ---- carve one device allocation
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = round_up(off + bytes, 256);
    return o;
  };
  const size_t o_hi0 = take(total_x * 2), o_hi1 = take(total_x * 2), o_lo = take(total_x * 2);
  const size_t o_A = take(total_a * 2), o_B = take(total_a * 2);
  const size_t o_part = split > 1 ? take(total_a * 4 * static_cast<size_t>(split)) : 0;
  size_t o_x0 = 0, o_x1 = 0, o_a32 = 0, o_b32 = 0;
  if (pl->fp32_ws) {
    o_x0 = take(total_x * 4);
    o_x1 = take(total_x * 4);
    o_a32 = take(total_a * 4);
    o_b32 = take(total_a * 4);
  }
  const size_t n_rms = static_cast<size_t>(pl->nchunks);
  const size_t o_s = take(n * sizeof(float));
  const size_t o_np = take(pl->nchunks * sizeof(double));
  const size_t o_nc = take(n * sizeof(unsigned));
  const size_t o_rms = take(n_rms * sizeof(float));
  const size_t o_status = take(sizeof(unsigned));
  const size_t o_unorm = take(n * sizeof(float));
  const size_t o_mats = take(n * sizeof(MatInfo));
  const size_t o_ptrs = take(muon_plan_s::kPtrSlots * n * sizeof(MatPtrs));
  const size_t o_sym = take(std::max<size_t>(1, sym.size()) * sizeof(TcTile));
  const size_t o_full = take(std::max<size_t>(1, full.size()) * sizeof(TcTile));
  const size_t o_sym32 = take(std::max<size_t>(1, sym32.size()) * sizeof(TileDesc));
  const size_t o_full32 = take(std::max<size_t>(1, full32.size()) * sizeof(TileDesc));
  const size_t o_chunks = take(chunks.size() * sizeof(ChunkDesc));
  const size_t o_tmaps = take(static_cast<size_t>(n) * kMapsPerMat * sizeof(CUtensorMap));
  const size_t o_red = take(std::max<size_t>(1, red.size()) * sizeof(int4));
  const size_t o_symg = take(std::max<size_t>(1, symg.size()) * sizeof(TcTile));
  pl->dbytes = off;
  if (capped && pl->dbytes > max_workspace_bytes) {  // the packing above accounts for every byte
    free_plan(pl);
    return MUON_ERR_NO_MEMORY;
  }
  if (cudaMalloc(&pl->dmem, pl->dbytes) != cudaSuccess) {
    cudaGetLastError();
    free_plan(pl);
    return MUON_ERR_NO_MEMORY;
  }
  uint8_t* b = pl->dmem;
  Workspace& ws = pl->ws;
  ws.hi[0] = reinterpret_cast<__nv_bfloat16*>(b + o_hi0);
  ws.hi[1] = reinterpret_cast<__nv_bfloat16*>(b + o_hi1);
  ws.lo = reinterpret_cast<__nv_bfloat16*>(b + o_lo);
  ws.A = reinterpret_cast<__nv_bfloat16*>(b + o_A);
  ws.B = reinterpret_cast<__nv_bfloat16*>(b + o_B);
  if (pl->fp32_ws) {
    ws.x32[0] = reinterpret_cast<float*>(b + o_x0);
    ws.x32[1] = reinterpret_cast<float*>(b + o_x1);
    ws.a32 = reinterpret_cast<float*>(b + o_a32);
    ws.b32 = reinterpret_cast<float*>(b + o_b32);
  }
  ws.s = reinterpret_cast<float*>(b + o_s);
  ws.norm_part = reinterpret_cast<double*>(b + o_np);
  ws.norm_count = reinterpret_cast<unsigned*>(b + o_nc);
  ws.rms_part = reinterpret_cast<float*>(b + o_rms);
  ws.status = reinterpret_cast<unsigned*>(b + o_status);
  ws.unorm = reinterpret_cast<float*>(b + o_unorm);
  if (split > 1) {
    ws.part = reinterpret_cast<float*>(b + o_part);
    ws.part_stride = static_cast<int64_t>(total_a);
  }
  pl->reduce_d = reinterpret_cast<int4*>(b + o_red);
  pl->symg_d = reinterpret_cast<TcTile*>(b + o_symg);
  pl->mats_d = reinterpret_cast<MatInfo*>(b + o_mats);
  for (int k = 0; k < muon_plan_s::kPtrSlots; ++k) pl->slots[k].dev = reinterpret_cast<MatPtrs*>(b + o_ptrs) + k * n;
  pl->ptrs_d = pl->slots[0].dev;
  pl->sym_d = reinterpret_cast<TcTile*>(b + o_sym);
  pl->full_d = reinterpret_cast<TcTile*>(b + o_full);
  pl->sym32_d = reinterpret_cast<TileDesc*>(b + o_sym32);
  pl->full32_d = reinterpret_cast<TileDesc*>(b + o_full32);
  pl->chunks_d = reinterpret_cast<ChunkDesc*>(b + o_chunks);
  pl->tmaps_d = b + o_tmaps;

  // ---- TMA descriptors per matrix
  std::vector<CUtensorMap> tmaps(static_cast<size_t>(n) * kMapsPerMat);
  for (int i = 0; i < n; ++i) {
    const MatInfo& mi = pl->mats[i];
    if (!encode_matrix_maps(&tmaps[static_cast<size_t>(kMapsPerMat) * i], mi, ws.hi[0] + mi.off_x,
                            ws.hi[1] + mi.off_x, ws.lo + mi.off_x, ws.A + mi.off_a, ws.B + mi.off_a,
                            split > 1 ? ws.part + mi.off_a : nullptr, ws.part_stride, split)) {
      free_plan(pl);
      return MUON_ERR_CUDA;
    }
  }

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  bool ok = cudaMemcpy(pl->mats_d, pl->mats.data(), n * sizeof(MatInfo), cudaMemcpyHostToDevice) == cudaSuccess;
  ok = ok && (sym.empty() || cudaMemcpy(pl->sym_d, sym.data(), sym.size() * sizeof(TcTile),
                                        cudaMemcpyHostToDevice) == cudaSuccess);
  ok = ok && (full.empty() || cudaMemcpy(pl->full_d, full.data(), full.size() * sizeof(TcTile),
                                         cudaMemcpyHostToDevice) == cudaSuccess);
  ok = ok && (sym32.empty() || cudaMemcpy(pl->sym32_d, sym32.data(), sym32.size() * sizeof(TileDesc),
                                          cudaMemcpyHostToDevice) == cudaSuccess);
  ok = ok && (full32.empty() || cudaMemcpy(pl->full32_d, full32.data(), full32.size() * sizeof(TileDesc),
                                           cudaMemcpyHostToDevice) == cudaSuccess);
  ok = ok && cudaMemcpy(pl->chunks_d, chunks.data(), chunks.size() * sizeof(ChunkDesc), cudaMemcpyHostToDevice) ==
                 cudaSuccess;
  ok = ok && (red.empty() || cudaMemcpy(pl->reduce_d, red.data(), red.size() * sizeof(int4), cudaMemcpyHostToDevice) ==
                                 cudaSuccess);
  ok = ok && (symg.empty() || cudaMemcpy(pl->symg_d, symg.data(), symg.size() * sizeof(TcTile),
                                         cudaMemcpyHostToDevice) == cudaSuccess);
  ok = ok && cudaMemcpy(pl->tmaps_d, tmaps.data(), tmaps.size() * sizeof(CUtensorMap), cudaMemcpyHostToDevice) ==
                 cudaSuccess;
  ok = ok && cudaMemset(ws.norm_count, 0, n * sizeof(unsigned)) == cudaSuccess;
  ok = ok && cudaMemset(ws.status, 0, sizeof(unsigned)) == cudaSuccess;
  ok = ok && cudaMemset(ws.s, 0, n * sizeof(float)) == cudaSuccess;
  for (auto& sl : pl->slots) {
    ok = ok && cudaHostAlloc(reinterpret_cast<void**>(&sl.pinned), n * sizeof(MatPtrs), cudaHostAllocDefault) ==
                   cudaSuccess;
    ok = ok && cudaEventCreateWithFlags(&sl.ev, cudaEventDisableTiming) == cudaSuccess;
  }
  if (!ok) {
    cudaGetLastError();
    free_plan(pl);
    return MUON_ERR_CUDA;
  }
  if (flags & MUON_INIT_ZERO_MOMENTUM) {
    for (int i = 0; i < n; ++i) {
      if (cudaMemsetAsync(params[i].M, 0, static_cast<size_t>(params[i].rows) * params[i].cols * sizeof(float), st) !=
          cudaSuccess) {
        cudaGetLastError();
        free_plan(pl);
        return MUON_ERR_CUDA;
      }
    }
  }
  pl->last_stream = st;
  *out = pl;
  return MUON_OK;
}

muon_status_t muon_step(muon_plan_t pl, const muon_param_t* params, int32_t n, const muon_hparams_t* hp,
                        float* update_rms, void* stream) {
  if (pl == nullptr || params == nullptr || hp == nullptr) return MUON_ERR_INVALID_ARG;
  if (n != pl->n) return MUON_ERR_SHAPE_MISMATCH;
  if (!finite(hp->lr) || !finite(hp->weight_decay) || !finite(hp->momentum) || !finite(hp->a) || !finite(hp->b) ||
      !finite(hp->c) || !finite(hp->rms_scale))
    return MUON_ERR_INVALID_ARG;
  if (hp->ns_steps < 0 || hp->ns_steps > kMaxNsSteps) return MUON_ERR_INVALID_ARG;
  if (hp->nesterov != 0 && hp->nesterov != 1) return MUON_ERR_INVALID_ARG;
  if (hp->scale_mode != MUON_SCALE_MAX_DIM && hp->scale_mode != MUON_SCALE_HIDDEN &&
      hp->scale_mode != MUON_SCALE_UPDATE_NORM)
    return MUON_ERR_INVALID_ARG;
  if (hp->scale_mode == MUON_SCALE_HIDDEN && !(finite(hp->hidden_dim) && hp->hidden_dim > 0.0f))
    return MUON_ERR_INVALID_ARG;
  if (hp->ns_precision != MUON_NS_BF16 && hp->ns_precision != MUON_NS_FP32) return MUON_ERR_INVALID_ARG;
  if (hp->ns_precision == MUON_NS_FP32 && !pl->fp32_ws) return MUON_ERR_UNSUPPORTED;
  std::vector<MatPtrs> t(n);
  std::vector<ByteRange> iv;
  iv.reserve(3 * static_cast<size_t>(n) + 1);
  for (int i = 0; i < n; ++i) {
    const muon_param_t& p = params[i];
    const MatInfo& mi = pl->mats[i];
    if (p.rows != mi.rows || p.cols != mi.cols) return MUON_ERR_SHAPE_MISMATCH;
    if (p.W == nullptr || p.G == nullptr || p.M == nullptr || p.reserved != 0) return MUON_ERR_INVALID_ARG;
    if (p.g_dtype != MUON_DT_BF16 && p.g_dtype != MUON_DT_FP32) return MUON_ERR_INVALID_ARG;
    const size_t e = static_cast<size_t>(mi.rows) * mi.cols;
    const uintptr_t w = reinterpret_cast<uintptr_t>(p.W), g = reinterpret_cast<uintptr_t>(p.G),
                    m = reinterpret_cast<uintptr_t>(p.M);
    iv.push_back({w, w + e * 4});
    iv.push_back({g, g + e * (p.g_dtype == MUON_DT_BF16 ? 2 : 4)});
    iv.push_back({m, m + e * 4});
    t[i].W = p.W;
    t[i].G = p.G;
    t[i].M = p.M;
    t[i].g_dtype = p.g_dtype;
    t[i].vec_ok = ((w | g | m) % 16 == 0 && mi.cols % 8 == 0) ? 1 : 0;
  }
  if (update_rms != nullptr) {
    const uintptr_t r = reinterpret_cast<uintptr_t>(update_rms);
    iv.push_back({r, r + static_cast<size_t>(n) * 4});
  }
  if (any_overlap(iv)) return MUON_ERR_ALIAS;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int cur_dev = -1;
  if (cudaGetDevice(&cur_dev) != cudaSuccess || cur_dev != pl->device) return MUON_ERR_INVALID_ARG;
  muon_status_t s = upload_ptrs(pl, t, st);
  if (s != MUON_OK) return s;
  StepScalars sc{hp->lr, hp->weight_decay, hp->momentum, hp->a, hp->b, hp->c, hp->rms_scale, hp->nesterov,
                 hp->scale_mode, 0.0f};
  if (hp->scale_mode == MUON_SCALE_HIDDEN) sc.const_scale = hp->rms_scale * std::sqrt(hp->hidden_dim);
  return run_ns(pl, sc, hp->ns_steps, hp->ns_precision, kFinalWeight, kK1Momentum, update_rms, st);
}

muon_status_t muon_orthogonalize(muon_plan_t pl, const void* const* X_in, float* const* O_out, int32_t n,
                                 int32_t in_dtype, int32_t ns_steps, const float abc[3], int32_t ns_precision,
                                 void* stream) {
  if (pl == nullptr || X_in == nullptr || O_out == nullptr || abc == nullptr) return MUON_ERR_INVALID_ARG;
  if (n != pl->n) return MUON_ERR_SHAPE_MISMATCH;
  if (in_dtype != MUON_DT_BF16 && in_dtype != MUON_DT_FP32) return MUON_ERR_INVALID_ARG;
  if (ns_steps < 0 || ns_steps > kMaxNsSteps) return MUON_ERR_INVALID_ARG;
  if (!finite(abc[0]) || !finite(abc[1]) || !finite(abc[2])) return MUON_ERR_INVALID_ARG;
  if (ns_precision != MUON_NS_BF16 && ns_precision != MUON_NS_FP32) return MUON_ERR_INVALID_ARG;
  if (ns_precision == MUON_NS_FP32 && !pl->fp32_ws) return MUON_ERR_UNSUPPORTED;
  std::vector<MatPtrs> t(n);
  std::vector<ByteRange> iv;
  iv.reserve(2 * static_cast<size_t>(n));
  for (int i = 0; i < n; ++i) {
    const MatInfo& mi = pl->mats[i];
    if (X_in[i] == nullptr || O_out[i] == nullptr) return MUON_ERR_INVALID_ARG;
    const size_t e = static_cast<size_t>(mi.rows) * mi.cols;
    const uintptr_t x = reinterpret_cast<uintptr_t>(X_in[i]), o = reinterpret_cast<uintptr_t>(O_out[i]);
    iv.push_back({x, x + e * (in_dtype == MUON_DT_BF16 ? 2 : 4)});
    iv.push_back({o, o + e * 4});
    t[i].W = O_out[i];
    t[i].G = X_in[i];
    t[i].M = nullptr;
    t[i].g_dtype = in_dtype;
    t[i].vec_ok = ((x | o) % 16 == 0 && mi.cols % 8 == 0) ? 1 : 0;
  }
  if (any_overlap(iv)) return MUON_ERR_ALIAS;
  int cur_dev = -1;
  if (cudaGetDevice(&cur_dev) != cudaSuccess || cur_dev != pl->device) return MUON_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  muon_status_t s = upload_ptrs(pl, t, st);
  if (s != MUON_OK) return s;
  StepScalars sc{0.0f, 0.0f, 0.0f, abc[0], abc[1], abc[2], 0.0f, 0, kScaleMaxDim, 0.0f};
  return run_ns(pl, sc, ns_steps, ns_precision, kFinalOut, kK1Copy, nullptr, st);
}

size_t muon_workspace_bytes(muon_plan_t pl) { return pl == nullptr ? 0 : pl->dbytes; }

muon_status_t muon_inject_wait_timeout(muon_plan_t pl, uint32_t wait_ns) {
  if (pl == nullptr || wait_ns < 1 || wait_ns > 1000000000u) return MUON_ERR_INVALID_ARG;
  pl->inject_wait_ns = wait_ns;
  return MUON_OK;
}

int32_t muon_num_waves(muon_plan_t pl) { return pl == nullptr ? -1 : static_cast<int32_t>(pl->waves.size()); }

muon_status_t muon_get_status(muon_plan_t pl) {
  if (pl == nullptr) return MUON_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(pl->last_stream) != cudaSuccess) return MUON_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpy(&v, pl->ws.status, sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess) return MUON_ERR_CUDA;
  if (v != 0 && cudaMemset(pl->ws.status, 0, sizeof(unsigned)) != cudaSuccess) return MUON_ERR_CUDA;
  if (v & kStatusTimeout) return MUON_ERR_TIMEOUT;
  if (v & kStatusNonFinite) return MUON_ERR_NONFINITE;
  return MUON_OK;
}

void muon_destroy(muon_plan_t pl) {
  if (pl == nullptr) return;
  cudaStreamSynchronize(pl->last_stream);
  cudaGetLastError();
  free_plan(pl);
}

muon_status_t muon_profile_enable(muon_plan_t pl, int32_t enable) {
  if (pl == nullptr || enable < 0 || enable > MUON_PROFILE_SPANS) return MUON_ERR_INVALID_ARG;
  if (enable && pl->events.empty()) {
    pl->events.resize(kEventPool);
    for (auto& ev : pl->events)
      if (cudaEventCreate(&ev) != cudaSuccess) return MUON_ERR_CUDA;
  }
  pl->prof = enable;
  return MUON_OK;
}

muon_status_t muon_profile_read(muon_plan_t pl, double* phase_ms, int64_t* launches, int32_t* calls) {
  if (pl == nullptr || phase_ms == nullptr || launches == nullptr || calls == nullptr) return MUON_ERR_INVALID_ARG;
  prof_flush(pl);
  for (int k = 0; k < MUON_NUM_PHASES; ++k) {
    phase_ms[k] += pl->prof_ms[k];
    launches[k] += pl->prof_launches[k];
    pl->prof_ms[k] = 0.0;
    pl->prof_launches[k] = 0;
  }
  *calls = pl->prof_calls;
  pl->prof_calls = 0;
  return from_cuda(cudaGetLastError());
}

}  // extern "C"
