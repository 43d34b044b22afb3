// AdamW companion step for the parameters that are not matrices.
//
// "Muon is Scalable for LLM Training" keeps AdamW for the RMSNorm gains, the
// embedding and the LM head, with the learning rate and weight decay shared
// with Muon (Sec. 2.2, "Matching update RMS of AdamW"; decay on the gains,
// Appendix D).  The update is AdamW as the pages cite it (Loshchilov and
// Hutter 2019): bias-corrected moments and decoupled weight decay.
//
// One launch covers every tensor of the plan: the tensors are cut into chunks
// of kAdamChunk elements, one CTA per chunk, 8 elements per thread per pass
// with 16-byte accesses when the pointers allow.  The step is a pure stream
// (P, m, v read and written, G read), so it is HBM bound: 26 bytes per element
// with a bf16 gradient, 28 with fp32.
#include "muon.h"
#include "muon_internal.cuh"

#include <algorithm>
#include <cmath>
#include <cstring>
#include <new>
#include <vector>

namespace muon {
namespace {

constexpr int kAdamChunk = 65536;  // elements per CTA (a multiple of 8)
constexpr int kAdamThreads = 256;

struct AdamPtrs {
  float* P;
  const void* G;
  float* m;
  float* v;
  int32_t g_dtype;
  int32_t decay;
  int32_t vec_ok;  // P, G, m, v all 16-byte aligned
  int32_t pad_;
};

// .x tensor, .y first element, .z element count
using AdamChunk = int4;

struct AdamScalars {
  float lr, b1, b2, eps, wd, inv_bc1, inv_bc2;
};

__device__ __forceinline__ void adam_elem(float& p, float g, float& m, float& v, const AdamScalars& s, float wd) {
  m = fmaf(s.b1, m, (1.0f - s.b1) * g);
  v = fmaf(s.b2, v, (1.0f - s.b2) * (g * g));
  const float u = (m * s.inv_bc1) / (sqrtf(v * s.inv_bc2) + s.eps);
  p = p - s.lr * fmaf(wd, p, u);
}

__device__ __forceinline__ void load_g8(const void* G, int64_t e, int dtype, float* g) {
  if (dtype == MUON_DT_BF16) {
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(G) + e));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      g[2 * i] = f.x;
      g[2 * i + 1] = f.y;
    }
  } else {
    const float4* q = reinterpret_cast<const float4*>(static_cast<const float*>(G) + e);
    const float4 a = __ldg(q), b = __ldg(q + 1);
    g[0] = a.x; g[1] = a.y; g[2] = a.z; g[3] = a.w;
    g[4] = b.x; g[5] = b.y; g[6] = b.z; g[7] = b.w;
  }
}

__device__ __forceinline__ float load_g1(const void* G, int64_t e, int dtype) {
  return dtype == MUON_DT_BF16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(G)[e])
                               : static_cast<const float*>(G)[e];
}

__global__ void __launch_bounds__(kAdamThreads) adamw_kernel(const AdamChunk* __restrict__ chunks,
                                                            const AdamPtrs* __restrict__ ptrs, AdamScalars s) {
  const AdamChunk ch = chunks[blockIdx.x];
  const AdamPtrs pt = ptrs[ch.x];
  const float wd = pt.decay ? s.wd : 0.0f;
  const int64_t e0 = ch.y;
  const int n = ch.z;
  int done = 0;
  if (pt.vec_ok) {
    done = n & ~7;
    for (int i = threadIdx.x * 8; i < done; i += blockDim.x * 8) {
      const int64_t e = e0 + i;
      float g[8];
      load_g8(pt.G, e, pt.g_dtype, g);
      float4* P4 = reinterpret_cast<float4*>(pt.P + e);
      float4* m4 = reinterpret_cast<float4*>(pt.m + e);
      float4* v4 = reinterpret_cast<float4*>(pt.v + e);
      float4 pa = P4[0], pb = P4[1], ma = m4[0], mb = m4[1], va = v4[0], vb = v4[1];
      adam_elem(pa.x, g[0], ma.x, va.x, s, wd);
      adam_elem(pa.y, g[1], ma.y, va.y, s, wd);
      adam_elem(pa.z, g[2], ma.z, va.z, s, wd);
      adam_elem(pa.w, g[3], ma.w, va.w, s, wd);
      adam_elem(pb.x, g[4], mb.x, vb.x, s, wd);
      adam_elem(pb.y, g[5], mb.y, vb.y, s, wd);
      adam_elem(pb.z, g[6], mb.z, vb.z, s, wd);
      adam_elem(pb.w, g[7], mb.w, vb.w, s, wd);
      P4[0] = pa;
      P4[1] = pb;
      m4[0] = ma;
      m4[1] = mb;
      v4[0] = va;
      v4[1] = vb;
    }
  }
  for (int i = done + threadIdx.x; i < n; i += blockDim.x) {
    const int64_t e = e0 + i;
    float p = pt.P[e], m = pt.m[e], v = pt.v[e];
    adam_elem(p, load_g1(pt.G, e, pt.g_dtype), m, v, s, wd);
    pt.P[e] = p;
    pt.m[e] = m;
    pt.v[e] = v;
  }
}

bool is_finite(float x) { return std::isfinite(x); }

}  // namespace
}  // namespace muon

using namespace muon;

struct muon_adamw_plan_s {
  int device = 0;
  int n = 0;
  std::vector<int64_t> numel;
  std::vector<int32_t> dtype;
  int nchunks = 0;
  uint8_t* dmem = nullptr;
  AdamChunk* chunks_d = nullptr;
  AdamPtrs* ptrs_d = nullptr;
  AdamPtrs* pinned = nullptr;  // staging of the per-call pointer table
  cudaEvent_t ev = nullptr;    // the last upload from `pinned` has been read
  bool ev_pending = false;
  std::vector<AdamPtrs> cache;
  bool cache_valid = false;
  cudaStream_t last_stream = nullptr;
};

namespace {

void free_adamw(muon_adamw_plan_s* pl) {
  if (pl == nullptr) return;
  if (pl->dmem) cudaFree(pl->dmem);
  if (pl->pinned) cudaFreeHost(pl->pinned);
  if (pl->ev) cudaEventDestroy(pl->ev);
  delete pl;
}

bool valid_param(const muon_adamw_param_t& p) {
  return p.numel >= 1 && p.numel <= INT32_MAX && (p.g_dtype == MUON_DT_BF16 || p.g_dtype == MUON_DT_FP32) &&
         (p.decay == 0 || p.decay == 1);
}

}  // namespace

extern "C" muon_status_t muon_adamw_hparams_default(muon_adamw_hparams_t* hp) {
  if (hp == nullptr) return MUON_ERR_INVALID_ARG;
  hp->lr = 4.2e-4f;
  hp->beta1 = 0.9f;
  hp->beta2 = 0.95f;
  hp->eps = 1e-8f;
  hp->weight_decay = 0.1f;
  hp->step = 1;
  return MUON_OK;
}

extern "C" muon_status_t muon_adamw_init(muon_adamw_plan_t* out, const muon_adamw_param_t* params, int32_t n,
                                         uint32_t flags, void* stream) {
  if (out == nullptr || params == nullptr || n < 1) return MUON_ERR_INVALID_ARG;
  *out = nullptr;
  if ((flags & ~MUON_INIT_ZERO_MOMENTUM) != 0) return MUON_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    if (!valid_param(params[i])) return MUON_ERR_INVALID_ARG;
    if ((flags & MUON_INIT_ZERO_MOMENTUM) && (params[i].m == nullptr || params[i].v == nullptr))
      return MUON_ERR_INVALID_ARG;
  }
  int dev = 0;
  cudaDeviceProp prop;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
    cudaGetLastError();
    return MUON_ERR_CUDA;
  }
  if (prop.major != 10 || prop.minor != 0) return MUON_ERR_UNSUPPORTED;
  muon_adamw_plan_s* pl = new (std::nothrow) muon_adamw_plan_s();
  if (pl == nullptr) return MUON_ERR_NO_MEMORY;
  pl->device = dev;
  pl->n = n;
  std::vector<AdamChunk> chunks;
  for (int i = 0; i < n; ++i) {
    pl->numel.push_back(params[i].numel);
    pl->dtype.push_back(params[i].g_dtype);
    for (int64_t e = 0; e < params[i].numel; e += kAdamChunk)
      chunks.push_back(make_int4(i, static_cast<int>(e), static_cast<int>(std::min<int64_t>(kAdamChunk,
                                                                                          params[i].numel - e)), 0));
  }
  pl->nchunks = static_cast<int>(chunks.size());
  const size_t chunk_bytes = (chunks.size() * sizeof(AdamChunk) + 255) / 256 * 256;
  if (cudaMalloc(&pl->dmem, chunk_bytes + n * sizeof(AdamPtrs)) != cudaSuccess) {
    cudaGetLastError();
    free_adamw(pl);
    return MUON_ERR_NO_MEMORY;
  }
  pl->chunks_d = reinterpret_cast<AdamChunk*>(pl->dmem);
  pl->ptrs_d = reinterpret_cast<AdamPtrs*>(pl->dmem + chunk_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  bool ok = cudaMemcpy(pl->chunks_d, chunks.data(), chunks.size() * sizeof(AdamChunk), cudaMemcpyHostToDevice) ==
            cudaSuccess;
  ok = ok && cudaHostAlloc(reinterpret_cast<void**>(&pl->pinned), n * sizeof(AdamPtrs), cudaHostAllocDefault) ==
                 cudaSuccess;
  ok = ok && cudaEventCreateWithFlags(&pl->ev, cudaEventDisableTiming) == cudaSuccess;
  if (ok && (flags & MUON_INIT_ZERO_MOMENTUM)) {
    for (int i = 0; i < n && ok; ++i) {
      ok = cudaMemsetAsync(params[i].m, 0, params[i].numel * sizeof(float), st) == cudaSuccess &&
           cudaMemsetAsync(params[i].v, 0, params[i].numel * sizeof(float), st) == cudaSuccess;
    }
  }
  if (!ok) {
    cudaGetLastError();
    free_adamw(pl);
    return MUON_ERR_CUDA;
  }
  pl->last_stream = st;
  *out = pl;
  return MUON_OK;
}

extern "C" muon_status_t muon_adamw_step(muon_adamw_plan_t pl, const muon_adamw_param_t* params, int32_t n,
                                         const muon_adamw_hparams_t* hp, void* stream) {
  if (pl == nullptr || params == nullptr || hp == nullptr) return MUON_ERR_INVALID_ARG;
  if (n != pl->n) return MUON_ERR_SHAPE_MISMATCH;
  if (!is_finite(hp->lr) || !is_finite(hp->weight_decay) || !is_finite(hp->eps) || !(hp->eps > 0.0f) ||
      !(hp->beta1 >= 0.0f && hp->beta1 < 1.0f) || !(hp->beta2 >= 0.0f && hp->beta2 < 1.0f) || hp->step < 1)
    return MUON_ERR_INVALID_ARG;
  std::vector<AdamPtrs> t(n);
  std::vector<ByteRange> spans;
  spans.reserve(4 * static_cast<size_t>(n));
  for (int i = 0; i < n; ++i) {
    const muon_adamw_param_t& p = params[i];
    if (p.numel != pl->numel[i] || p.g_dtype != pl->dtype[i]) return MUON_ERR_SHAPE_MISMATCH;
    if (p.P == nullptr || p.G == nullptr || p.m == nullptr || p.v == nullptr || (p.decay != 0 && p.decay != 1))
      return MUON_ERR_INVALID_ARG;
    const size_t e = static_cast<size_t>(p.numel);
    const uintptr_t P = reinterpret_cast<uintptr_t>(p.P), G = reinterpret_cast<uintptr_t>(p.G),
                    m = reinterpret_cast<uintptr_t>(p.m), v = reinterpret_cast<uintptr_t>(p.v);
    spans.push_back({P, P + e * 4});
    spans.push_back({G, G + e * (p.g_dtype == MUON_DT_BF16 ? 2 : 4)});
    spans.push_back({m, m + e * 4});
    spans.push_back({v, v + e * 4});
    t[i] = AdamPtrs{p.P, p.G, p.m, p.v, p.g_dtype, p.decay, ((P | G | m | v) % 16 == 0) ? 1 : 0, 0};
  }
  if (any_overlap(spans)) return MUON_ERR_ALIAS;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != pl->device) return MUON_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // upload the pointer table only when it changed; the pinned staging is
  // reused once the previous upload has been read
  if (!(pl->cache_valid && std::memcmp(t.data(), pl->cache.data(), t.size() * sizeof(AdamPtrs)) == 0)) {
    if (pl->ev_pending) {
      if (cudaEventSynchronize(pl->ev) != cudaSuccess) return MUON_ERR_CUDA;
      pl->ev_pending = false;
    }
    std::memcpy(pl->pinned, t.data(), t.size() * sizeof(AdamPtrs));
    if (cudaMemcpyAsync(pl->ptrs_d, pl->pinned, t.size() * sizeof(AdamPtrs), cudaMemcpyHostToDevice, st) !=
            cudaSuccess ||
        cudaEventRecord(pl->ev, st) != cudaSuccess) {
      cudaGetLastError();
      return MUON_ERR_CUDA;
    }
    pl->ev_pending = true;
    pl->cache = t;
    pl->cache_valid = true;
  }
  const double bc1 = 1.0 - std::pow(static_cast<double>(hp->beta1), hp->step);
  const double bc2 = 1.0 - std::pow(static_cast<double>(hp->beta2), hp->step);
  if (!(bc1 > 0.0) || !(bc2 > 0.0)) return MUON_ERR_INVALID_ARG;
  AdamScalars s{hp->lr, hp->beta1, hp->beta2, hp->eps, hp->weight_decay, static_cast<float>(1.0 / bc1),
                static_cast<float>(1.0 / bc2)};
  adamw_kernel<<<pl->nchunks, kAdamThreads, 0, st>>>(pl->chunks_d, pl->ptrs_d, s);
  if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;
  pl->last_stream = st;
  return MUON_OK;
}

extern "C" void muon_adamw_destroy(muon_adamw_plan_t pl) {
  if (pl == nullptr) return;
  cudaStreamSynchronize(pl->last_stream);
  cudaGetLastError();
  free_adamw(pl);
}
