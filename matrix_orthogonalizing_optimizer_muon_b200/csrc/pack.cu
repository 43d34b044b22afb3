// Multi-segment copy with dtype conversion: the packing step of data-parallel
// Muon ("Muon is Scalable for LLM Training", Sec. 2.3, Algorithm 1), which
// moves every matrix's gradient into the flat buffer that the gradient
// reduce-scatter reads, and the updated weights into and out of the flat
// buffers of the weight all-gather.  One launch covers every segment of a
// plan, so a step issues a constant number of copies whatever its matrix
// count.
//
// Each segment is cut into chunks of kPackChunk elements, one CTA per chunk;
// a chunk whose source and destination allow it moves 16-byte vectors, the
// rest element by element.  Pure HBM traffic: (source + destination) bytes
// per element.
#include "muon.h"
#include "muon_internal.cuh"

#include <algorithm>
#include <iterator>
#include <new>
#include <vector>

namespace {

constexpr int kPackThreads = 256;
constexpr int64_t kPackChunk = 65536;

struct SegDev {
  const void* src;
  void* dst;
  int64_t numel;
  int32_t src_dtype;  // muon_dtype_t
  int32_t dst_dtype;
};

struct ChunkRef {
  int32_t seg;
  int32_t pad;
  int64_t first;  // first element of the chunk within its segment
};

__device__ __forceinline__ float load_elem(const void* p, int64_t i, int dt) {
  return dt == MUON_DT_BF16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i])
                            : static_cast<const float*>(p)[i];
}

__device__ __forceinline__ void store_elem(void* p, int64_t i, int dt, float v) {
  if (dt == MUON_DT_BF16) static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  else static_cast<float*>(p)[i] = v;
}

// Eight consecutive elements at element index i (16-byte aligned for fp32 pairs,
// 16-byte aligned for bf16 octets).
__device__ __forceinline__ void load8(const void* p, int64_t i, int dt, float* v) {
  if (dt == MUON_DT_BF16) {
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p) + i));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(h[k]);
      v[2 * k] = f.x;
      v[2 * k + 1] = f.y;
    }
  } else {
    const float4* q = reinterpret_cast<const float4*>(static_cast<const float*>(p) + i);
    const float4 a = __ldg(q), b = __ldg(q + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

__device__ __forceinline__ void store8(void* p, int64_t i, int dt, const float* v) {
  if (dt == MUON_DT_BF16) {
    __align__(16) __nv_bfloat16 h[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) h[k] = __float2bfloat16_rn(v[k]);
    *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p) + i) = *reinterpret_cast<const uint4*>(h);
  } else {
    float4* q = reinterpret_cast<float4*>(static_cast<float*>(p) + i);
    q[0] = make_float4(v[0], v[1], v[2], v[3]);
    q[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
}

__global__ void __launch_bounds__(kPackThreads) pack_kernel(const SegDev* __restrict__ segs,
                                                            const ChunkRef* __restrict__ chunks) {
  const ChunkRef c = chunks[blockIdx.x];
  const SegDev s = segs[c.seg];
  const int64_t left = s.numel - c.first;
  const int64_t n = left < kPackChunk ? left : kPackChunk;
  const int ss = s.src_dtype == MUON_DT_BF16 ? 2 : 4, ds = s.dst_dtype == MUON_DT_BF16 ? 2 : 4;
  const uintptr_t sa = reinterpret_cast<uintptr_t>(s.src) + static_cast<uintptr_t>(c.first) * ss;
  const uintptr_t da = reinterpret_cast<uintptr_t>(s.dst) + static_cast<uintptr_t>(c.first) * ds;
  const bool vec = (sa % 16 == 0) && (da % 16 == 0);
  int64_t done = 0;
  if (vec) {
    const int64_t n8 = n & ~int64_t(7);
    for (int64_t e = static_cast<int64_t>(threadIdx.x) * 8; e < n8; e += kPackThreads * 8) {
      float v[8];
      load8(s.src, c.first + e, s.src_dtype, v);
      store8(s.dst, c.first + e, s.dst_dtype, v);
    }
    done = n8;
  }
  for (int64_t e = done + threadIdx.x; e < n; e += kPackThreads)
    store_elem(s.dst, c.first + e, s.dst_dtype, load_elem(s.src, c.first + e, s.src_dtype));
}

}  // namespace

struct muon_pack_plan_s {
  int device = 0;
  int nseg = 0;
  int nchunks = 0;
  uint8_t* dmem = nullptr;
  SegDev* segs_d = nullptr;
  ChunkRef* chunks_d = nullptr;
  cudaStream_t last_stream = nullptr;
};

extern "C" {

muon_status_t muon_pack_init(muon_pack_plan_t* out, const muon_segment_t* segs, int32_t n, void* stream) {
  if (out == nullptr) return MUON_ERR_INVALID_ARG;
  *out = nullptr;
  if (segs == nullptr || n < 1 || n > (1 << 24)) return MUON_ERR_INVALID_ARG;
  std::vector<muon::ByteRange> dst_ranges, src_ranges;
  std::vector<SegDev> host(n);
  std::vector<ChunkRef> chunks;
  for (int i = 0; i < n; ++i) {
    const muon_segment_t& g = segs[i];
    if (g.src == nullptr || g.dst == nullptr || g.numel < 1 || g.numel > (int64_t(1) << 40)) return MUON_ERR_INVALID_ARG;
    if ((g.src_dtype != MUON_DT_BF16 && g.src_dtype != MUON_DT_FP32) ||
        (g.dst_dtype != MUON_DT_BF16 && g.dst_dtype != MUON_DT_FP32))
      return MUON_ERR_INVALID_ARG;
    const uintptr_t s = reinterpret_cast<uintptr_t>(g.src), d = reinterpret_cast<uintptr_t>(g.dst);
    src_ranges.push_back({s, s + static_cast<size_t>(g.numel) * (g.src_dtype == MUON_DT_BF16 ? 2 : 4)});
    dst_ranges.push_back({d, d + static_cast<size_t>(g.numel) * (g.dst_dtype == MUON_DT_BF16 ? 2 : 4)});
    host[i] = SegDev{g.src, g.dst, g.numel, g.src_dtype, g.dst_dtype};
    for (int64_t f = 0; f < g.numel; f += kPackChunk) chunks.push_back(ChunkRef{i, 0, f});
  }
  // destinations are pairwise disjoint (every element has one writer), and no
  // source overlaps any destination, so the chunks of a launch may run in any
  // order; sources may overlap each other (they are only read)
  if (muon::any_overlap(dst_ranges)) return MUON_ERR_ALIAS;  // sorts dst_ranges
  for (const muon::ByteRange& r : src_ranges) {
    auto it = std::upper_bound(dst_ranges.begin(), dst_ranges.end(), r.lo,
                               [](uintptr_t v, const muon::ByteRange& x) { return v < x.lo; });
    if (it != dst_ranges.end() && it->lo < r.hi) return MUON_ERR_ALIAS;
    if (it != dst_ranges.begin() && std::prev(it)->hi > r.lo) return MUON_ERR_ALIAS;
  }
  if (chunks.size() > static_cast<size_t>(0x7fffffff)) return MUON_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MUON_ERR_CUDA;
  muon_pack_plan_s* pl = new (std::nothrow) muon_pack_plan_s();
  if (pl == nullptr) return MUON_ERR_NO_MEMORY;
  pl->device = dev;
  pl->nseg = n;
  pl->nchunks = static_cast<int>(chunks.size());
  const size_t seg_bytes = (static_cast<size_t>(n) * sizeof(SegDev) + 255) / 256 * 256;
  const size_t bytes = seg_bytes + chunks.size() * sizeof(ChunkRef);
  if (cudaMalloc(&pl->dmem, bytes) != cudaSuccess) {
    cudaGetLastError();
    delete pl;
    return MUON_ERR_NO_MEMORY;
  }
  pl->segs_d = reinterpret_cast<SegDev*>(pl->dmem);
  pl->chunks_d = reinterpret_cast<ChunkRef*>(pl->dmem + seg_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  bool ok = cudaMemcpy(pl->segs_d, host.data(), n * sizeof(SegDev), cudaMemcpyHostToDevice) == cudaSuccess;
  ok = ok && cudaMemcpy(pl->chunks_d, chunks.data(), chunks.size() * sizeof(ChunkRef), cudaMemcpyHostToDevice) ==
                 cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    cudaFree(pl->dmem);
    delete pl;
    return MUON_ERR_CUDA;
  }
  pl->last_stream = st;
  *out = pl;
  return MUON_OK;
}

muon_status_t muon_pack_run(muon_pack_plan_t pl, void* stream) {
  if (pl == nullptr) return MUON_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != pl->device) return MUON_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  pack_kernel<<<pl->nchunks, kPackThreads, 0, st>>>(pl->segs_d, pl->chunks_d);
  pl->last_stream = st;
  return cudaGetLastError() == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}

void muon_pack_destroy(muon_pack_plan_t pl) {
  if (pl == nullptr) return;
  cudaStreamSynchronize(pl->last_stream);
  cudaGetLastError();
  cudaFree(pl->dmem);
  delete pl;
}

}  // extern "C"
