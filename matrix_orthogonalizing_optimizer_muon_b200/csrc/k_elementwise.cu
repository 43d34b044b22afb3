// Elementwise kernels of the Muon step.  All of them are HBM-bound: they are
// written as chunked streams with 16-byte vector accesses where the caller's
// pointers allow it, and every reduction is done in a fixed order so that a
// step is bitwise reproducible.
//
// k1: momentum + Nesterov input + Frobenius norm + bf16 hi/lo split
//     ("Muon is Scalable for LLM Training", Sec. 2.1, Eq. 1, the Nesterov
//     paragraph, and X_0 = M / ||M||_F).  One CTA per chunk of rows.  The norm
//     is accumulated in fp64 per chunk; the last CTA of each matrix (arrival
//     counter) reduces the chunk partials in chunk order and writes
//     s = 1 / ||Y||_F (0 for an all-zero Y, NaN plus a status bit if the sum
//     is not finite).
// apply_update: W <- W - lr (scale O + wd W) (Sec. 2.2, Eq. 4; Sec. 3.1,
//     Eq. 5/6 for the other scales), or O itself, from the iterate the last
//     X update left in workspace, with O = s X when there are no
//     Newton-Schulz iterations (N = 0).  A separate, fully coalesced pass: a
//     fused row-per-thread fp32 read-modify-write in the last GEMM epilogue
//     measured about twice as slow as this pass plus the extra iterate write.
// update_norm: RMS(O) per matrix and the Eq. 6 factor rms_scale / RMS(O)
//     (Sec. 3.1, "Update Norm"), chunk partials in fp64 reduced in chunk
//     order by the last CTA of each matrix.
// rms_finalize: sqrt(mean(O^2)) per matrix from the update pass's per-chunk partial sums
//     (Sec. 2.3, Algorithm 1, returned value).
#include "muon_internal.cuh"

namespace muon {
namespace {

__device__ __forceinline__ void load8(const void* base, size_t idx, int dtype, float* v) {
  if (dtype == 0) {
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + idx));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx);
    const float4 a = __ldg(p), b = __ldg(p + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

__device__ __forceinline__ float load1(const void* base, size_t idx, int dtype) {
  if (dtype == 0) return __bfloat162float(static_cast<const __nv_bfloat16*>(base)[idx]);
  return static_cast<const float*>(base)[idx];
}

// Split y into hi = bf16(y), lo = bf16(y - hi).
__device__ __forceinline__ void split_store8(__nv_bfloat16* hi, __nv_bfloat16* lo, const float* y) {
  __align__(16) __nv_bfloat16 h[8];
  __align__(16) __nv_bfloat16 l[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    h[i] = __float2bfloat16_rn(y[i]);
    l[i] = __float2bfloat16_rn(y[i] - __bfloat162float(h[i]));
  }
  *reinterpret_cast<uint4*>(hi) = *reinterpret_cast<const uint4*>(h);
  *reinterpret_cast<uint4*>(lo) = *reinterpret_cast<const uint4*>(l);
}

// Deterministic block sum (fixed shuffle tree, then warps in order).
template <typename T>
__device__ T block_sum(T v, T* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  T t = T(0);
  if (threadIdx.x == 0) {
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += red[i];
  }
  return t;  // valid in thread 0
}

__global__ void __launch_bounds__(kEwThreads) k1_kernel(const ChunkDesc* __restrict__ chunks,
                                                        const MatInfo* __restrict__ mats,
                                                        const MatPtrs* __restrict__ ptrs, Workspace ws,
                                                        StepScalars sc, int mode, int fp32_path) {
  __shared__ double red[kEwThreads / 32];
  __shared__ int am_last;
  pdl_wait();
  pdl_trigger();
  const ChunkDesc ch = chunks[blockIdx.x];
  const int p = ch.x;
  const MatInfo mi = mats[p];
  const MatPtrs pt = ptrs[p];
  const int C = mi.cols, r0 = ch.y, nr = ch.z;
  const float mu = sc.mu;
  double acc = 0.0;

  if (pt.vec_ok) {
    const int cv = C >> 3;
    const int units = nr * cv;
    for (int u = threadIdx.x; u < units; u += blockDim.x) {
      const int rr = u / cv;
      const int c8 = (u - rr * cv) << 3;
      const int r = r0 + rr;
      const size_t gi = (size_t)r * C + c8;
      const size_t wi = (size_t)mi.off_x + (size_t)r * mi.ld + c8;
      float y[8];
      load8(pt.G, gi, pt.g_dtype, y);
      if (mode == kK1Momentum) {
        float4* mp = reinterpret_cast<float4*>(pt.M + gi);
        float4 m0 = mp[0], m1 = mp[1];
        float m[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float g = y[i];
          m[i] = fmaf(mu, m[i], g);                      // M_t = mu M_{t-1} + G_t
          y[i] = sc.nesterov ? fmaf(mu, m[i], g) : m[i];  // Y = mu M_t + G_t
        }
        mp[0] = make_float4(m[0], m[1], m[2], m[3]);
        mp[1] = make_float4(m[4], m[5], m[6], m[7]);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) acc = fma((double)y[i], (double)y[i], acc);
      if (fp32_path) {
        float4* xp = reinterpret_cast<float4*>(ws.x32[0] + wi);
        xp[0] = make_float4(y[0], y[1], y[2], y[3]);
        xp[1] = make_float4(y[4], y[5], y[6], y[7]);
      } else {
        split_store8(ws.hi[0] + wi, ws.lo + wi, y);
      }
    }
  } else {
    const int64_t total = (int64_t)nr * C;
    for (int64_t e = threadIdx.x; e < total; e += blockDim.x) {
      const int rr = (int)(e / C);
      const int c = (int)(e - (int64_t)rr * C);
      const int r = r0 + rr;
      const size_t gi = (size_t)r * C + c;
      const size_t wi = (size_t)mi.off_x + (size_t)r * mi.ld + c;
      const float g = load1(pt.G, gi, pt.g_dtype);
      float y = g;
      if (mode == kK1Momentum) {
        const float m = fmaf(mu, pt.M[gi], g);
        pt.M[gi] = m;
        y = sc.nesterov ? fmaf(mu, m, g) : m;
      }
      acc = fma((double)y, (double)y, acc);
      if (fp32_path) {
        ws.x32[0][wi] = y;
      } else {
        const __nv_bfloat16 h = __float2bfloat16_rn(y);
        ws.hi[0][wi] = h;
        ws.lo[wi] = __float2bfloat16_rn(y - __bfloat162float(h));
      }
    }
  }

  const double part = block_sum(acc, red);
  if (threadIdx.x == 0) {
    ws.norm_part[ch.w] = part;
    __threadfence();
    const unsigned prev = atomicAdd(ws.norm_count + p, 1u);
    am_last = (prev == (unsigned)(mi.nchunks - 1));
  }
  __syncthreads();
  if (!am_last) return;
  __threadfence();
  double t = 0.0;
  for (int i = threadIdx.x; i < mi.nchunks; i += blockDim.x) t += __ldcg(ws.norm_part + mi.chunk_base + i);
  const double f2 = block_sum(t, red);
  if (threadIdx.x == 0) {
    float s;
    if (!isfinite(f2)) {
      s = __int_as_float(0x7fc00000);
      atomicOr(ws.status, kStatusNonFinite);
    } else {
      s = f2 > 0.0 ? (float)(1.0 / sqrt(f2)) : 0.0f;
    }
    ws.s[p] = s;
    ws.norm_count[p] = 0u;
  }
}

// The iterate X in workspace: fp32 x32 on the fp32 path, else the bf16 pair hi + lo.
struct XView {
  const float* x32;
  const __nv_bfloat16* hi;
  const __nv_bfloat16* lo;
};

__device__ __forceinline__ XView x_view(const Workspace& ws, int fp32_path, int xbuf) {
  // selects, not an indexed load: a runtime index into a kernel-parameter
  // array would copy the whole struct to local memory
  return fp32_path ? XView{xbuf ? ws.x32[1] : ws.x32[0], nullptr, nullptr}
                   : XView{nullptr, xbuf ? ws.hi[1] : ws.hi[0], ws.lo};
}

// Eight consecutive values of X at workspace index wi (16-byte aligned).
__device__ __forceinline__ void load_x8(XView xv, size_t wi, float* x) {
  if (xv.x32 != nullptr) {
    const float4* q = reinterpret_cast<const float4*>(xv.x32 + wi);
    const float4 u = q[0], v = q[1];
    x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w;
    x[4] = v.x; x[5] = v.y; x[6] = v.z; x[7] = v.w;
  } else {
    const uint4 h = *reinterpret_cast<const uint4*>(xv.hi + wi);
    const uint4 l = *reinterpret_cast<const uint4*>(xv.lo + wi);
    const __nv_bfloat162* hh = reinterpret_cast<const __nv_bfloat162*>(&h);
    const __nv_bfloat162* ll = reinterpret_cast<const __nv_bfloat162*>(&l);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 fh = __bfloat1622float2(hh[i]), fl = __bfloat1622float2(ll[i]);
      x[2 * i] = fh.x + fl.x;
      x[2 * i + 1] = fh.y + fl.y;
    }
  }
}

__device__ __forceinline__ float load_x1(XView xv, size_t wi) {
  return xv.x32 != nullptr ? xv.x32[wi] : __bfloat162float(xv.hi[wi]) + __bfloat162float(xv.lo[wi]);
}

__global__ void __launch_bounds__(kEwThreads) apply_update_kernel(const ChunkDesc* __restrict__ chunks,
                                                                  const MatInfo* __restrict__ mats,
                                                                  const MatPtrs* __restrict__ ptrs, Workspace ws,
                                                                  StepScalars sc, int final_mode, int fp32_path,
                                                                  int xbuf, int mul_s) {
  __shared__ float red[kEwThreads / 32];
  pdl_wait();
  pdl_trigger();
  const ChunkDesc ch = chunks[blockIdx.x];
  const int p = ch.x;
  const MatInfo mi = mats[p];
  const MatPtrs pt = ptrs[p];
  const int C = mi.cols, r0 = ch.y, nr = ch.z;
  // s == 0 marks Y == 0: O = 0, and the Newton-Schulz launches skipped this
  // matrix, so its iterate buffer holds nothing of this step
  const float sp = ws.s[p];
  const bool zero = (sp == 0.0f);
  const float s = zero ? 0.0f : (mul_s ? sp : 1.0f);
  const float scale = zero ? 0.0f : (sc.scale_mode == kScaleUpdateNorm ? ws.unorm[p] : update_scale_of(sc, mi.n));
  const bool weight = (final_mode == kFinalWeight);
  const XView xv = x_view(ws, fp32_path, xbuf);
  float acc = 0.0f;
  const int64_t total = (int64_t)nr * C;
  if (pt.vec_ok) {
    for (int64_t e = (int64_t)threadIdx.x * 8; e < total; e += (int64_t)blockDim.x * 8) {
      const int rr = (int)(e / C);
      const int c = (int)(e - (int64_t)rr * C);
      const int r = r0 + rr;
      const size_t gi = (size_t)r * C + c;
      const size_t wi = (size_t)mi.off_x + (size_t)r * mi.ld + c;
      float o[8] = {};
      if (!zero) load_x8(xv, wi, o);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        o[i] *= s;
        acc = fmaf(o[i], o[i], acc);
      }
      float4* w4 = reinterpret_cast<float4*>(pt.W + gi);
      float4 wa = w4[0], wb = w4[1];
      if (weight) {
        wa.x = wa.x - sc.lr * fmaf(scale, o[0], sc.wd * wa.x);
        wa.y = wa.y - sc.lr * fmaf(scale, o[1], sc.wd * wa.y);
        wa.z = wa.z - sc.lr * fmaf(scale, o[2], sc.wd * wa.z);
        wa.w = wa.w - sc.lr * fmaf(scale, o[3], sc.wd * wa.w);
        wb.x = wb.x - sc.lr * fmaf(scale, o[4], sc.wd * wb.x);
        wb.y = wb.y - sc.lr * fmaf(scale, o[5], sc.wd * wb.y);
        wb.z = wb.z - sc.lr * fmaf(scale, o[6], sc.wd * wb.z);
        wb.w = wb.w - sc.lr * fmaf(scale, o[7], sc.wd * wb.w);
      } else {
        wa = make_float4(o[0], o[1], o[2], o[3]);
        wb = make_float4(o[4], o[5], o[6], o[7]);
      }
      w4[0] = wa;
      w4[1] = wb;
    }
  } else {
    for (int64_t e = threadIdx.x; e < total; e += blockDim.x) {
      const int rr = (int)(e / C);
      const int c = (int)(e - (int64_t)rr * C);
      const int r = r0 + rr;
      const size_t gi = (size_t)r * C + c;
      const size_t wi = (size_t)mi.off_x + (size_t)r * mi.ld + c;
      const float o = zero ? 0.0f : s * load_x1(xv, wi);
      acc = fmaf(o, o, acc);
      if (weight) {
        const float w = pt.W[gi];
        pt.W[gi] = w - sc.lr * fmaf(scale, o, sc.wd * w);
      } else {
        pt.W[gi] = o;
      }
    }
  }
  const float part = block_sum(acc, red);
  if (threadIdx.x == 0) ws.rms_part[ch.w] = part;
}

__global__ void __launch_bounds__(kEwThreads) update_norm_kernel(const ChunkDesc* __restrict__ chunks,
                                                                 const MatInfo* __restrict__ mats, Workspace ws,
                                                                 StepScalars sc, int fp32_path, int xbuf, int mul_s,
                                                                 float* __restrict__ update_rms) {
  __shared__ double red[kEwThreads / 32];
  __shared__ bool am_last;
  pdl_wait();
  pdl_trigger();
  const ChunkDesc ch = chunks[blockIdx.x];
  const int p = ch.x;
  const MatInfo mi = mats[p];
  const int C = mi.cols, r0 = ch.y, nr = ch.z;
  const float sp = ws.s[p];
  const float s = mul_s ? sp : 1.0f;
  const XView xv = x_view(ws, fp32_path, xbuf);
  double acc = 0.0;
  const int64_t total = (int64_t)nr * C;
  if (sp == 0.0f) {
    // Y == 0: O = 0 (the iterate buffer was not written this step)
  } else if (C % 8 == 0) {
    for (int64_t e = (int64_t)threadIdx.x * 8; e < total; e += (int64_t)blockDim.x * 8) {
      const int rr = (int)(e / C);
      const int c = (int)(e - (int64_t)rr * C);
      float o[8];
      load_x8(xv, (size_t)mi.off_x + (size_t)(r0 + rr) * mi.ld + c, o);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float v = s * o[i];
        acc = fma((double)v, (double)v, acc);
      }
    }
  } else {
    for (int64_t e = threadIdx.x; e < total; e += blockDim.x) {
      const int rr = (int)(e / C);
      const int c = (int)(e - (int64_t)rr * C);
      const float v = s * load_x1(xv, (size_t)mi.off_x + (size_t)(r0 + rr) * mi.ld + c);
      acc = fma((double)v, (double)v, acc);
    }
  }
  const double part = block_sum(acc, red);
  if (threadIdx.x == 0) {
    ws.norm_part[ch.w] = part;
    __threadfence();
    const unsigned prev = atomicAdd(ws.norm_count + p, 1u);
    am_last = (prev == (unsigned)(mi.nchunks - 1));
  }
  __syncthreads();
  if (!am_last) return;
  __threadfence();
  double t = 0.0;
  for (int i = threadIdx.x; i < mi.nchunks; i += blockDim.x) t += __ldcg(ws.norm_part + mi.chunk_base + i);
  const double sum = block_sum(t, red);
  if (threadIdx.x == 0) {
    const double rms = sqrt(sum / ((double)mi.rows * (double)mi.cols));
    float f;
    if (!isfinite(rms)) {
      f = __int_as_float(0x7fc00000);
      atomicOr(ws.status, kStatusNonFinite);
    } else {
      f = rms > 0.0 ? (float)((double)sc.rms_scale / rms) : 0.0f;
    }
    ws.unorm[p] = f;
    if (update_rms != nullptr) update_rms[p] = (float)rms;
    ws.norm_count[p] = 0u;
  }
}

__global__ void __launch_bounds__(kEwThreads) rms_finalize_kernel(const MatInfo* __restrict__ mats,
                                                                  const float* __restrict__ part,
                                                                  float* __restrict__ out) {
  __shared__ double red[kEwThreads / 32];
  pdl_wait();
  pdl_trigger();
  const MatInfo mi = mats[blockIdx.x];
  double t = 0.0;
  for (int i = threadIdx.x; i < mi.nchunks; i += blockDim.x) t += (double)part[mi.chunk_base + i];
  const double sum = block_sum(t, red);
  if (threadIdx.x == 0) out[blockIdx.x] = (float)sqrt(sum / ((double)mi.rows * (double)mi.cols));
}

// Split-K reduction of a symmetric product: one CTA of 32 x 8 threads per
// 32 x 32 block on or below the diagonal.  Each element's parts are summed in
// part order (so the result does not depend on which CTA pair computed which
// part), the phase's epilogue arithmetic is applied, the bf16 value is
// written and, through a shared-memory transpose, its mirror.
__global__ void __launch_bounds__(256) split_reduce_kernel(const int4* __restrict__ blocks,
                                                           const MatInfo* __restrict__ mats, Workspace ws,
                                                           StepScalars sc, int phase, int iter, int split) {
  __shared__ __nv_bfloat16 tile[32][34];
  pdl_wait();
  pdl_trigger();
  const int4 bk = blocks[blockIdx.x];
  const MatInfo mi = mats[bk.x];
  const int i0 = bk.y, j0 = bk.z, m = mi.m;
  const float s = ws.s[bk.x];
  if (s == 0.0f) return;  // Y == 0: the matrix is skipped, as in the tensor-core launches
  __nv_bfloat16* out = (phase == kPhaseGram ? ws.A : ws.B) + mi.off_a;
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int j = j0 + tx;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = ty + 8 * k;
    const int i = i0 + r;
    __nv_bfloat16 h = __float2bfloat16_rn(0.0f);
    if (i < m && j < m && j <= i) {
      const size_t e = static_cast<size_t>(i) * mi.lda + j;
      float acc = 0.0f;
      for (int p = 0; p < split; ++p) acc += ws.part[p * ws.part_stride + mi.off_a + e];
      float v;
      if (phase == kPhaseGram) {
        v = (iter == 0) ? (acc * s) * s : acc;
      } else {
        v = fmaf(sc.c, acc, sc.b * __bfloat162float(ws.A[mi.off_a + e])) + (i == j ? sc.a : 0.0f);
      }
      h = __float2bfloat16_rn(v);
      out[e] = h;
    }
    tile[r][tx] = h;
  }
  __syncthreads();
  // mirror: element (j0 + r, i0 + tx) = tile[tx][r], for (i0 + tx) > (j0 + r)
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = ty + 8 * k;
    const int jr = j0 + r, ic = i0 + tx;
    if (jr < m && ic < m && ic > jr) out[static_cast<size_t>(jr) * mi.lda + ic] = tile[tx][r];
  }
}

}  // namespace

cudaError_t launch_split_reduce(const int4* blocks, int nblocks, const MatInfo* mats, Workspace ws, StepScalars sc,
                                int phase, int iter, int split, cudaStream_t st) {
  if (nblocks == 0) return cudaSuccess;
  return launch_pdl(kPdlElementwise, split_reduce_kernel, dim3(nblocks), dim3(32, 8), 0, st, blocks, mats, ws, sc,
                    phase, iter, split);
}

cudaError_t launch_k1(const ChunkDesc* chunks, int nchunks, const MatInfo* mats, const MatPtrs* ptrs,
                      Workspace ws, StepScalars sc, int mode, int fp32_path, cudaStream_t st) {
  return launch_pdl(kPdlElementwise, k1_kernel, dim3(nchunks), dim3(kEwThreads), 0, st, chunks, mats, ptrs, ws, sc,
                    mode, fp32_path);
}

cudaError_t launch_apply_update(const ChunkDesc* chunks, int nchunks, const MatInfo* mats, const MatPtrs* ptrs,
                                Workspace ws, StepScalars sc, int final_mode, int fp32_path, int xbuf, int mul_s,
                                cudaStream_t st) {
  return launch_pdl(kPdlElementwise, apply_update_kernel, dim3(nchunks), dim3(kEwThreads), 0, st, chunks, mats,
                    ptrs, ws, sc, final_mode, fp32_path, xbuf, mul_s);
}

cudaError_t launch_update_norm(const ChunkDesc* chunks, int nchunks, const MatInfo* mats, Workspace ws,
                               StepScalars sc, int fp32_path, int xbuf, int mul_s, float* update_rms,
                               cudaStream_t st) {
  return launch_pdl(kPdlElementwise, update_norm_kernel, dim3(nchunks), dim3(kEwThreads), 0, st, chunks, mats, ws,
                    sc, fp32_path, xbuf, mul_s, update_rms);
}

cudaError_t launch_rms_finalize(const MatInfo* mats, int nmat, const float* part, float* out, cudaStream_t st) {
  return launch_pdl(kPdlElementwise, rms_finalize_kernel, dim3(nmat), dim3(kEwThreads), 0, st, mats, part, out);
}

}  // namespace muon
