// fp32 Newton-Schulz path on the CUDA cores (validation precision).
//
// Same three phases as the tensor-core kernel ("Muon is Scalable for LLM
// Training", Sec. 2.1, Eq. 2 as A = X X^T, B = b A + c A^2, X' = a X + B X),
// but every operand, product and accumulator is fp32 and the symmetric
// matrices are computed in full.  One CTA per 64x64 output tile, 256 threads
// with a 4x4 register micro-tile, operands staged through shared memory in
// K slices of 16.  Operand (i, k) is read K-major (row i contiguous) or
// MN-major (column i contiguous) exactly as on the tensor-core path.
#include "muon_internal.cuh"

namespace muon {
namespace {

constexpr int kKS = 16;

struct Src {
  const float* p;
  int ld;    // pitch of the stored array
  int mn;    // 1: element (i, k) at p[k * ld + i]; 0: at p[i * ld + k]
  int rows;  // extent in i
};

__device__ __forceinline__ float fetch(const Src& s, int i, int k, int K) {
  if (i >= s.rows || k >= K) return 0.0f;
  return s.mn ? s.p[static_cast<size_t>(k) * s.ld + i] : s.p[static_cast<size_t>(i) * s.ld + k];
}

__global__ void __launch_bounds__(256) ns_gemm_f32_kernel(const __grid_constant__ Gemm32Args g) {
  __shared__ float As[kKS][kT32 + 4];
  __shared__ float Bs[kKS][kT32 + 4];
  const TileDesc td = g.tiles[blockIdx.x];
  const int p = td.x, row0 = td.y, col0 = td.z;
  const MatInfo mi = g.mats[p];
  const float s = g.ws.s[p];
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;

  const float* xcur = g.ws.x32[g.cur] + mi.off_x;
  const float* a32 = g.ws.a32 + mi.off_a;
  const float* b32 = g.ws.b32 + mi.off_a;
  Src sa, sb;
  int K, out_rows, out_cols;
  if (g.phase == kPhaseGram) {
    K = mi.n;
    sa = {xcur, mi.ld, mi.tall, mi.m};
    sb = sa;
    out_rows = out_cols = mi.m;
  } else if (g.phase == kPhasePoly) {
    K = mi.m;
    sa = {a32, mi.lda, 0, mi.m};
    sb = sa;
    out_rows = out_cols = mi.m;
  } else {
    K = mi.m;
    if (mi.tall) {
      sa = {xcur, mi.ld, 0, mi.rows};
      sb = {b32, mi.lda, 0, mi.m};
    } else {
      sa = {b32, mi.lda, 0, mi.m};
      sb = {xcur, mi.ld, 1, mi.cols};
    }
    out_rows = mi.rows;
    out_cols = mi.cols;
  }

  float acc[4][4] = {};
  if (s != 0.0f) {
    for (int k0 = 0; k0 < K; k0 += kKS) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int idx = tid + 256 * q;
        // K-major: consecutive threads walk k; MN-major: consecutive threads walk i
        const int ka = sa.mn ? idx / kT32 : idx % kKS, ia = sa.mn ? idx % kT32 : idx / kKS;
        As[ka][ia] = fetch(sa, row0 + ia, k0 + ka, K);
        const int kb = sb.mn ? idx / kT32 : idx % kKS, ib = sb.mn ? idx % kT32 : idx / kKS;
        Bs[kb][ib] = fetch(sb, col0 + ib, k0 + kb, K);
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < kKS; ++kk) {
        float a[4], b[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          a[u] = As[kk][ty * 4 + u];
          b[u] = Bs[kk][tx * 4 + u];
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
      }
      __syncthreads();
    }
  } else {
    return;  // Y == 0: nothing downstream reads this matrix (the update pass treats it as O = 0)
  }

#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = row0 + ty * 4 + u;
    if (i >= out_rows) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int j = col0 + tx * 4 + v;
      if (j >= out_cols) continue;
      const float r = acc[u][v];
      if (g.phase == kPhaseGram) {
        g.ws.a32[mi.off_a + static_cast<size_t>(i) * mi.lda + j] = g.iter == 0 ? (r * s) * s : r;
      } else if (g.phase == kPhasePoly) {
        const size_t o = mi.off_a + static_cast<size_t>(i) * mi.lda + j;
        g.ws.b32[o] = fmaf(g.sc.c, r, g.sc.b * g.ws.a32[o]);
      } else {
        const size_t o = static_cast<size_t>(i) * mi.ld + j;
        const float alpha = g.iter == 0 ? s : 1.0f;
        g.ws.x32[g.cur ^ 1][mi.off_x + o] = alpha * fmaf(g.sc.a, xcur[o], r);
      }
    }
  }
}

}  // namespace

cudaError_t launch_gemm_f32(const Gemm32Args& args, cudaStream_t st) {
  if (args.ntiles == 0) return cudaSuccess;
  ns_gemm_f32_kernel<<<args.ntiles, 256, 0, st>>>(args);
  return cudaGetLastError();
}

}  // namespace muon
