// muon_orthogonalize_noalloc: Newton-Schulz of one matrix with no device
// allocation at all.
//
// Some callers cannot call cudaMalloc: code whose device memory is owned by a
// framework allocator or a fixed budget, and latency-critical loops that must
// not allocate (cudaMalloc can synchronize the device) after start-up.  This
// entry point runs the same kernels as muon_orthogonalize on the bf16
// tensor-core path, but every byte of scratch it needs (iterate buffers,
// Gram and polynomial matrices, norms, schedules, TMA descriptors) lives in
// one file-scope device array of fixed size, which every GPU that loads the
// library holds until the process exits.  The caller passes the input and the
// output; the per-call descriptors are copied in from the host stack, so the
// call returns only once the driver has staged those (pageable) copies, and a
// stream that is being captured is refused.
#include "muon.h"
#include "muon_internal.cuh"

#include <cuda.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

using namespace muon;

namespace {

// Size limits of one call.
constexpr int64_t kNaMaxElems = int64_t(1) << 20;  // rows * cols
constexpr int kNaMaxDim = 8192;                    // rows and cols each
constexpr int kNaMaxM = 1024;                      // min(rows, cols)
constexpr int kNaMaxTiles = 256;                   // per tile list
constexpr int kNaMaxChunks = 512;

constexpr size_t align256(size_t v) { return (v + 255) / 256 * 256; }

// Scratch layout (byte offsets).
constexpr size_t kNaX = align256((kNaMaxElems + 8 * kNaMaxDim) * 2);       // one [R, ld] bf16 array
constexpr size_t kNaA = align256(size_t(kNaMaxM) * kNaMaxM * 2);            // one [m, lda] bf16 array
constexpr size_t kOffHi0 = 0;
constexpr size_t kOffHi1 = kOffHi0 + kNaX;
constexpr size_t kOffLo = kOffHi1 + kNaX;
constexpr size_t kOffA = kOffLo + kNaX;
constexpr size_t kOffB = kOffA + kNaA;
constexpr size_t kOffS = kOffB + kNaA;
constexpr size_t kOffNormPart = kOffS + 256;
constexpr size_t kOffNormCount = kOffNormPart + align256(kNaMaxChunks * sizeof(double));
constexpr size_t kOffRms = kOffNormCount + 256;
constexpr int kNaMaxRms = kNaMaxChunks;  // one update partial per chunk
constexpr size_t kOffStatus = kOffRms + align256(kNaMaxRms * sizeof(float));
constexpr size_t kOffMat = kOffStatus + 256;
constexpr size_t kOffPtrs = kOffMat + align256(sizeof(MatInfo));
constexpr size_t kOffSym = kOffPtrs + align256(sizeof(MatPtrs));
constexpr size_t kOffFull = kOffSym + align256(kNaMaxTiles * sizeof(TcTile));
constexpr size_t kOffChunks = kOffFull + align256(kNaMaxTiles * sizeof(TcTile));
constexpr size_t kOffTmaps = kOffChunks + align256(kNaMaxChunks * sizeof(ChunkDesc));
constexpr size_t kScratchBytes = kOffTmaps + align256(kMapsPerMat * sizeof(CUtensorMap));

// ~10.7 MB, zero-initialised at module load.
__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

struct DeviceState {
  unsigned char* base = nullptr;  // device address of g_noalloc_scratch on this device
  int npairs = 0;
  bool sm100 = false;             // compute capability 10.0
  std::atomic<bool> ready{false};
};
DeviceState g_state[64];
std::mutex g_setup_mutex;  // first calls from several host threads set a device up once

// Once per device, with that device current: resolve the scratch array's
// device address (in host code the symbol's name is only a host-side stand-in)
// and read the device's compute capability and persistent grid size.
muon_status_t setup_device(int dev) {
  DeviceState& st = g_state[dev];
  if (st.ready.load(std::memory_order_acquire)) return MUON_OK;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (st.ready.load(std::memory_order_relaxed)) return MUON_OK;
  int major = 0, minor = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return MUON_ERR_CUDA;
  }
  st.sm100 = (major == 10 && minor == 0);
  if (st.sm100) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return MUON_ERR_CUDA;
    }
    st.base = static_cast<unsigned char*>(p);
    st.npairs = gemm_tc_max_pairs();
    if (st.npairs < 1) st.npairs = std::max(1, sms / 2);
  }
  st.ready.store(true, std::memory_order_release);
  return MUON_OK;
}

}  // namespace

extern "C" muon_status_t muon_orthogonalize_noalloc(const void* X_in, float* O_out, int64_t rows, int64_t cols,
                                                    int32_t in_dtype, int32_t ns_steps, const float abc[3],
                                                    void* stream) {
  if (X_in == nullptr || O_out == nullptr || abc == nullptr) return MUON_ERR_INVALID_ARG;
  if (rows < 1 || cols < 1) return MUON_ERR_INVALID_ARG;
  if (in_dtype != MUON_DT_BF16 && in_dtype != MUON_DT_FP32) return MUON_ERR_INVALID_ARG;
  if (ns_steps < 0 || ns_steps > 32) return MUON_ERR_INVALID_ARG;
  if (!std::isfinite(abc[0]) || !std::isfinite(abc[1]) || !std::isfinite(abc[2])) return MUON_ERR_INVALID_ARG;
  if (rows > kNaMaxDim || cols > kNaMaxDim || rows * cols > kNaMaxElems || std::min(rows, cols) > kNaMaxM)
    return MUON_ERR_UNSUPPORTED;  // beyond the fixed scratch
  const size_t in_bytes = static_cast<size_t>(rows * cols) * (in_dtype == MUON_DT_BF16 ? 2 : 4);
  const uintptr_t x = reinterpret_cast<uintptr_t>(X_in), o = reinterpret_cast<uintptr_t>(O_out);
  if (x < o + static_cast<size_t>(rows * cols) * 4 && o < x + in_bytes) return MUON_ERR_ALIAS;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MUON_ERR_CUDA;
  muon_status_t su = setup_device(dev);
  if (su != MUON_OK) return su;
  if (!g_state[dev].sm100) return MUON_ERR_UNSUPPORTED;
  unsigned char* base = g_state[dev].base;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The descriptors below are copied from this call's stack frame; a stream
  // capture would record copies that read that frame again at replay, long
  // after it is gone.  Refuse a capturing stream before enqueuing anything.
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) {
    cudaGetLastError();
    return MUON_ERR_CUDA;
  }
  if (cap != cudaStreamCaptureStatusNone) return MUON_ERR_UNSUPPORTED;

  // ---- one matrix: descriptors built on the host stack
  const int R = static_cast<int>(rows), C = static_cast<int>(cols);
  MatInfo mi{};
  mi.rows = R;
  mi.cols = C;
  mi.m = std::min(R, C);
  mi.n = std::max(R, C);
  mi.tall = R > C ? 1 : 0;
  mi.ld = (C + 7) / 8 * 8;
  mi.lda = (mi.m + 7) / 8 * 8;
  mi.off_x = 0;
  mi.off_a = 0;
  ChunkDesc chunks[kNaMaxChunks];
  const int rows_per_chunk = std::max(1, kChunkElems / C);
  int nch = 0;
  for (int r = 0; r < R; r += rows_per_chunk) {
    if (nch == kNaMaxChunks) return MUON_ERR_UNSUPPORTED;
    chunks[nch] = make_int4(0, r, std::min(rows_per_chunk, R - r), nch);
    ++nch;
  }
  mi.chunk_base = 0;
  mi.nchunks = nch;
  TcTile sym[kNaMaxTiles], full[kNaMaxTiles];
  int nsym = 0, nfull = 0;
  bool fits = true;
  // as in a plan: a list with at most half as many tiles as CTA pairs is
  // split along N while each pair still gets at most one tile
  int cs = 0, cf = 0;
  for_each_sym_tile(mi.m, [&](const TcTile&) { ++cs; });
  for_each_full_tile(R, C, [&](const TcTile&) { ++cf; });
  auto levels = [&](int count) {
    int lv = 0;
    while (lv < 2 && count * 2 <= g_state[dev].npairs) {
      ++lv;
      count *= 2;
    }
    return lv;
  };
  const int ls = levels(cs), lf = levels(cf);
  for_each_sym_tile(mi.m, [&](const TcTile& whole) {
    split_n(whole, ls, mi.m, [&](const TcTile& t) {
      if (nsym == kNaMaxTiles) fits = false;
      else sym[nsym++] = t;
    });
  });
  for_each_full_tile(R, C, [&](const TcTile& whole) {
    split_n(whole, lf, C, [&](const TcTile& t) {
      if (nfull == kNaMaxTiles) fits = false;
      else full[nfull++] = t;
    });
  });
  if (!fits) return MUON_ERR_UNSUPPORTED;
  MatPtrs mp{};
  mp.W = O_out;
  mp.G = X_in;
  mp.M = nullptr;
  mp.g_dtype = in_dtype;
  mp.vec_ok = ((x | o) % 16 == 0 && C % 8 == 0) ? 1 : 0;

  Workspace ws{};
  ws.hi[0] = reinterpret_cast<__nv_bfloat16*>(base + kOffHi0);
  ws.hi[1] = reinterpret_cast<__nv_bfloat16*>(base + kOffHi1);
  ws.lo = reinterpret_cast<__nv_bfloat16*>(base + kOffLo);
  ws.A = reinterpret_cast<__nv_bfloat16*>(base + kOffA);
  ws.B = reinterpret_cast<__nv_bfloat16*>(base + kOffB);
  ws.s = reinterpret_cast<float*>(base + kOffS);
  ws.norm_part = reinterpret_cast<double*>(base + kOffNormPart);
  ws.norm_count = reinterpret_cast<unsigned*>(base + kOffNormCount);
  ws.rms_part = reinterpret_cast<float*>(base + kOffRms);
  ws.status = reinterpret_cast<unsigned*>(base + kOffStatus);
  CUtensorMap tm[kMapsPerMat];
  const bool ok = encode_matrix_maps(tm, mi, ws.hi[0], ws.hi[1], ws.lo, ws.A, ws.B);
  if (!ok) return MUON_ERR_CUDA;

  // ---- stage descriptors (pageable host -> device copies are staged by the
  // driver before the call returns) and clear what must start at zero
  MatInfo* mats_d = reinterpret_cast<MatInfo*>(base + kOffMat);
  MatPtrs* ptrs_d = reinterpret_cast<MatPtrs*>(base + kOffPtrs);
  TcTile* sym_d = reinterpret_cast<TcTile*>(base + kOffSym);
  TcTile* full_d = reinterpret_cast<TcTile*>(base + kOffFull);
  ChunkDesc* chunks_d = reinterpret_cast<ChunkDesc*>(base + kOffChunks);
  void* tmaps_d = base + kOffTmaps;
  cudaError_t e = cudaSuccess;
  e = e == cudaSuccess ? cudaMemcpyAsync(mats_d, &mi, sizeof(mi), cudaMemcpyHostToDevice, st) : e;
  e = e == cudaSuccess ? cudaMemcpyAsync(ptrs_d, &mp, sizeof(mp), cudaMemcpyHostToDevice, st) : e;
  e = e == cudaSuccess ? cudaMemcpyAsync(sym_d, sym, nsym * sizeof(TcTile), cudaMemcpyHostToDevice, st) : e;
  e = e == cudaSuccess ? cudaMemcpyAsync(full_d, full, nfull * sizeof(TcTile), cudaMemcpyHostToDevice, st) : e;
  e = e == cudaSuccess ? cudaMemcpyAsync(chunks_d, chunks, nch * sizeof(ChunkDesc), cudaMemcpyHostToDevice, st) : e;
  e = e == cudaSuccess ? cudaMemcpyAsync(tmaps_d, tm, sizeof(tm), cudaMemcpyHostToDevice, st) : e;
  e = e == cudaSuccess ? cudaMemsetAsync(ws.norm_count, 0, sizeof(unsigned), st) : e;
  e = e == cudaSuccess ? cudaMemsetAsync(ws.status, 0, sizeof(unsigned), st) : e;
  if (e != cudaSuccess) return MUON_ERR_CUDA;

  // ---- the same launch sequence as muon_orthogonalize on the bf16 path
  StepScalars sc{0.0f, 0.0f, 0.0f, abc[0], abc[1], abc[2], 0.0f, 0, kScaleMaxDim, 0.0f};
  if (launch_k1(chunks_d, nch, mats_d, ptrs_d, ws, sc, kK1Copy, 0, st) != cudaSuccess) return MUON_ERR_CUDA;
  int cur = 0;
  for (int it = 0; it < ns_steps; ++it) {
    for (int ph = kPhaseGram; ph <= kPhaseUpdate; ++ph) {
      GemmArgs a{};
      a.tiles = (ph == kPhaseUpdate) ? full_d : sym_d;
      a.ntiles = (ph == kPhaseUpdate) ? nfull : nsym;
      a.phase = ph;
      a.iter = it;
      a.cur = cur;
      a.mats = mats_d;
      a.ptrs = ptrs_d;
      a.tmaps = tmaps_d;
      a.ws = ws;
      a.sc = sc;
      if (launch_gemm_tc(a, g_state[dev].npairs, st) != cudaSuccess) return MUON_ERR_CUDA;
    }
    cur ^= 1;  // the X update wrote the other buffer
  }
  // O = X from hi[cur] + lo, or s Y when there are no iterations
  if (launch_apply_update(chunks_d, nch, mats_d, ptrs_d, ws, sc, kFinalOut, 0, cur, ns_steps == 0 ? 1 : 0, st) !=
      cudaSuccess)
    return MUON_ERR_CUDA;
  return MUON_OK;
}
