// SVD-entropy diagnostic of weight matrices.
//
// "Muon is Scalable for LLM Training", Sec. 3.4 ("Dynamics of singular
// spectrum", the SVD-entropy equation and Fig. 4) compares optimisers by the
// SVD entropy of each weight matrix:
//   H(sigma) = -(1 / log n) sum_i p_i log p_i,  p_i = sigma_i^2 / sum_j sigma_j^2
// over its n = min(rows, cols) singular values.
//
// sigma_i^2 are the eigenvalues of the Gram matrix G = X X^T of the wide
// orientation X (m x n, m <= n) of W.  Only the eigenvalues are needed, no
// vectors, so G is reduced to a symmetric tridiagonal matrix T with the same
// eigenvalues and those are found by bisection.  The path, all matrices of a
// plan per launch:
//   1. gram_kernel: G in fp64 on the CUDA cores (128 x 128 tiles of the
//      lower triangle, each also written mirrored), zero-padded to m_pad, a
//      multiple of 64.  Products of fp32 entries are exact in fp64.
//   2. tridiag_kernel, one CTA per matrix: Householder reduction
//      Q^T G Q = T (Golub and Van Loan, "Matrix Computations", Sec. 8.3.1) in
//      panels of kTdNb columns, the blocked form of Dongarra, Sorensen and
//      Hammarling ("Block reduction of matrices to condensed forms for
//      eigenvalue computations", 1989).  Within a panel the matrix is
//      G0 - V W^T - W V^T, G0 the matrix at the panel's start and V, W one
//      column per reflector so far.  Column j is brought up to date from
//      row j of G0 (G0 is symmetric) and V, W; its reflector
//      H = I - tau v v^T (v_{j+1} = 1) zeroes rows j+2 .. m-1; then
//      y = tau (G0 v - V (W^T v) - W (V^T v)) and w = y - (tau/2)(v^T y) v,
//      because H B H = B - v w^T - w v^T for a symmetric B.  G0 v is the one
//      pass over the trailing matrix per column.  At the panel's end the
//      trailing matrix becomes G0 - V W^T - W V^T, computed on 64 x 64 tiles
//      of the lower triangle and written with their mirror, so the stored
//      matrix stays exactly symmetric.
//   3. bisect_kernel: every eigenvalue of T by bisection on the Sturm count
//      of T - x I (Golub and Van Loan, Sec. 8.4.1), one thread per
//      eigenvalue.  The count is the number of negative pivots of the
//      LDL^T factorisation, q_i = (d_i - x) - e_{i-1}^2 / q_{i-1}, the form
//      whose floating-point count is exact for a matrix within a few ulps of
//      T (Kahan); a pivot of magnitude below pivmin is replaced by -pivmin.
//      Bisection runs from the Gershgorin interval to a width of
//      2 eps ||T||, about 52 halvings.
//   4. entropy_kernel: H from the eigenvalues with fp64 sums in a fixed
//      order, and the singular values, descending (a bitonic sort makes the
//      order exact).
// Everything is deterministic: reductions run in a fixed order and the only
// atomic is the sticky status flag.
//
// The arithmetic is fp64 throughout.  H weighs every eigenvalue by
// -p log p, whose slope is unbounded near p = 0: with an fp32 Gram matrix the
// rounding floor (about 1e-7 of the largest eigenvalue) alone moved H of a
// rank-10 200 x 300 matrix by about 6e-5.  The reduction is backward stable:
// T has the eigenvalues of a matrix within a small multiple of
// m eps ||G|| of G, and bisection adds 2 eps ||T||.
#include "muon.h"
#include "muon_internal.cuh"

#include <algorithm>
#include <cfloat>
#include <cmath>
#include <cstring>
#include <new>
#include <vector>

namespace muon {
namespace {

constexpr int kGramTile = 128;
constexpr int kGramK = 16;
constexpr int kGramLd = kGramTile + 2;  // shared-memory pitch of a staged operand row (doubles)
constexpr int kGramThreads = 256;
constexpr int kPad = 64;                // G's row pitch is m rounded up to a multiple of kPad
constexpr size_t kGramSmem = static_cast<size_t>(kGramTile) * (kGramTile + 1) * sizeof(double);
constexpr int kMaxDim = 8192;        // min(rows, cols) limit (the sort stages 8192 values)
constexpr int kSortThreads = 1024;

// tridiagonal reduction: one CTA per matrix, two CTAs per SM (so a batch of
// up to 2 x 148 matrices is resident at once and no matrix waits for an SM)
constexpr int kTdThreads = 256;
constexpr int kTdWarps = kTdThreads / 32;
constexpr int kTdNb = 32;            // columns per panel
constexpr int kTdTile = 64;          // trailing-update tile
constexpr int kSymvRows = 3;         // rows per warp and pass of G0 v (2, 3, 4, 8 measured: 3 best)
// shared memory of tridiag_kernel, in doubles: the column x, the reflector
// v and the product y (m_pad each) plus small arrays; the trailing update
// reuses the space for its operand tiles and the output tile
constexpr int kTdSmall = 6 * kTdNb + 2 * kTdWarps + 16;
constexpr int kTdTrail = 4 * kTdNb * kTdTile + kTdTile * (kTdTile + 1);

constexpr int kBisThreads = 256;     // bisection: one thread per eigenvalue
constexpr int kBisMaxIter = 64;

// conv[] values
constexpr int kConvDone = 1;
constexpr int kConvNonFinite = 2;

struct EntMat {
  int rows, cols;
  int m, n;         // min and max of rows, cols
  int tall;         // rows > cols: X = W^T
  int mp;           // m rounded up to a multiple of 64: G's row pitch
  int64_t off_g;    // doubles into the G workspace (mp x mp, row-major)
  int64_t off_vw;   // doubles into the panel store (V then W, kTdNb x mp each)
  int64_t sv_off;   // first eigenvalue / singular value of this matrix
};

struct EntCtl {
  int* conv;        // [n] kConv*
  int* computed;    // [n] 1 once the eigenvalues are computed, 0 for a non-finite matrix
  unsigned* status; // [1] sticky: kStatusNonFinite
};

size_t tridiag_smem_bytes(int mp) {
  return static_cast<size_t>(std::max(3 * mp + kTdSmall, kTdTrail)) * sizeof(double);
}
// With clusters, each CTA asks for more than half of an SM's shared memory,
// so the cluster's CTAs land on different SMs.
constexpr size_t kTdSpreadSmem = 116 * 1024;

// ---------------------------------------------------------------- 1. Gram
__device__ __forceinline__ float x_at(const float* W, const EntMat& mi, int i, int k) {
  if (i >= mi.m || k >= mi.n) return 0.0f;
  return mi.tall ? __ldg(W + static_cast<size_t>(k) * mi.cols + i) : __ldg(W + static_cast<size_t>(i) * mi.cols + k);
}

// G = X X^T over 128 x 128 tiles of the lower triangle (written with their
// mirror, so G is stored whole and exactly symmetric; a diagonal tile's two
// halves are the same products in the same order, hence equal).  K runs in
// chunks of kGramK: each chunk of both operands is converted to fp64 once,
// into shared memory [k][row], double-buffered through registers; a thread
// accumulates an 8 x 8 block (rows 8 ty + i, columns tx + 16 j) in k order,
// so every element is the sequential fp64 sum of the exact fp32 products.
__global__ void __launch_bounds__(kGramThreads, 1) gram_kernel(const int4* __restrict__ tiles,
                                                               const EntMat* __restrict__ mats,
                                                               const float* const* __restrict__ wptr,
                                                               double* __restrict__ G) {
  extern __shared__ double gsm[];
  double* As = gsm;                              // [2][kGramK][kGramLd]
  double* Bs = As + 2 * kGramK * kGramLd;        // [2][kGramK][kGramLd]
  double* Cs = gsm;                              // [kGramTile][kGramTile + 1], after the K loop
  const int4 td = tiles[blockIdx.x];
  const EntMat mi = mats[td.x];
  const float* W = wptr[td.x];
  const int i0 = td.y * kGramTile, j0 = td.z * kGramTile;
  const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
  // staging: wide (X = W): thread t takes row t mod 128 and 8 consecutive k;
  // tall (X = W^T): k = t mod 16 and 8 consecutive rows (W's contiguous dimension)
  const int sr = mi.tall ? (t >> 4) * 8 : (t & 127);
  const int sk = mi.tall ? (t & 15) : (t >> 7) * 8;
  float ra[8], rb[8];
  auto fetch = [&](int k0) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int r = mi.tall ? sr + q : sr, k = mi.tall ? sk : sk + q;
      ra[q] = x_at(W, mi, i0 + r, k0 + k);
      rb[q] = x_at(W, mi, j0 + r, k0 + k);
    }
  };
  auto stash = [&](int buf) {
    double* A_ = As + buf * kGramK * kGramLd;
    double* B_ = Bs + buf * kGramK * kGramLd;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int r = mi.tall ? sr + q : sr, k = mi.tall ? sk : sk + q;
      A_[k * kGramLd + r] = static_cast<double>(ra[q]);
      B_[k * kGramLd + r] = static_cast<double>(rb[q]);
    }
  };
  double acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0;
  const int nchunks = (mi.n + kGramK - 1) / kGramK;
  fetch(0);
  stash(0);
  __syncthreads();
  for (int c = 0; c < nchunks; ++c) {
    const int buf = c & 1;
    if (c + 1 < nchunks) fetch((c + 1) * kGramK);
    const double* A_ = As + buf * kGramK * kGramLd;
    const double* B_ = Bs + buf * kGramK * kGramLd;
#pragma unroll 4
    for (int k = 0; k < kGramK; ++k) {
      double av[8], bv[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const double2 a2 = *reinterpret_cast<const double2*>(A_ + k * kGramLd + ty * 8 + 2 * q);
        av[2 * q] = a2.x;
        av[2 * q + 1] = a2.y;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) bv[j] = B_[k * kGramLd + tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fma(av[i], bv[j], acc[i][j]);
    }
    if (c + 1 < nchunks) stash(buf ^ 1);  // that buffer's readers passed the previous barrier
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) Cs[(ty * 8 + i) * (kGramTile + 1) + tx + 16 * j] = acc[i][j];
  __syncthreads();
  double* g = G + mi.off_g;
  const size_t ld = static_cast<size_t>(mi.mp);
  for (int e = t; e < kGramTile * kGramTile; e += kGramThreads) {
    const int r = e >> 7, c = e & 127;
    if (i0 + r < mi.mp && j0 + c < mi.mp) g[(i0 + r) * ld + j0 + c] = Cs[r * (kGramTile + 1) + c];
    if (td.y != td.z && j0 + r < mi.mp && i0 + c < mi.mp) g[(j0 + r) * ld + i0 + c] = Cs[c * (kGramTile + 1) + r];
  }
}

// ---------------------------------------------------------------- 2. tridiagonal reduction
// Sum over a warp; lane 0 holds the result (a fixed butterfly order).
__device__ __forceinline__ double warp_sum(double s) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}

// Sum over the CTA, the same value in every thread: warp sums, then the
// warps' partials in warp order.  red holds kTdWarps doubles.
__device__ __forceinline__ double td_block_sum(double s, double* red) {
  s = warp_sum(s);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = s;
  __syncthreads();
  double tot = 0.0;
#pragma unroll
  for (int w = 0; w < kTdWarps; ++w) tot += red[w];
  __syncthreads();
  return tot;
}

// A[r][c] -= sum_k (V_k[r] W_k[c] + W_k[r] V_k[c]) over the lower 64 x 64
// tiles of the trailing block [t0, m)^2, each written with its mirror.  The
// k-sum of one element and of its mirror would round differently, so the
// mirror is copied, not recomputed.
__device__ void td_trailing_update(double* A, int ld, int m, int t0, int nbk, const double* Vg, const double* Wg,
                                   double* sm, int rank, int C) {
  double* Vr = sm;                         // [kTdNb][64]: V_k[r0 + rr]
  double* Wr = Vr + kTdNb * kTdTile;
  double* Vc = Wr + kTdNb * kTdTile;       // [kTdNb][64]: V_k[c0 + cc]
  double* Wc = Vc + kTdNb * kTdTile;
  double* Cs = Wc + kTdNb * kTdTile;       // [64][65] updated tile
  const int t = threadIdx.x, tx = t & 15, ty = t >> 4;  // rows ty + 16 u; columns tx + 16 q
  const int nt = (m - t0 + kTdTile - 1) / kTdTile;
  int tix = 0;  // tile index; tile tix belongs to CTA tix mod C of the cluster
  for (int a = 0; a < nt; ++a) {
    for (int b = 0; b <= a; ++b, ++tix) {
      if (tix % C != rank) continue;
      const int r0 = t0 + a * kTdTile, c0 = t0 + b * kTdTile;
      for (int e = t; e < kTdNb * kTdTile; e += kTdThreads) {
        const int k = e >> 6, q = e & 63;
        const bool kin = k < nbk;
        Vr[e] = (kin && r0 + q < m) ? __ldcg(Vg + static_cast<size_t>(k) * ld + r0 + q) : 0.0;
        Wr[e] = (kin && r0 + q < m) ? __ldcg(Wg + static_cast<size_t>(k) * ld + r0 + q) : 0.0;
        Vc[e] = (kin && c0 + q < m) ? __ldcg(Vg + static_cast<size_t>(k) * ld + c0 + q) : 0.0;
        Wc[e] = (kin && c0 + q < m) ? __ldcg(Wg + static_cast<size_t>(k) * ld + c0 + q) : 0.0;
      }
      __syncthreads();
      // each thread: kRows rows (ty + kTdThreads / 16 apart) x 4 columns (16 apart)
      constexpr int kRows = kTdTile * kTdTile / (4 * kTdThreads);
      static_assert(kRows * (kTdThreads / 16) == kTdTile, "trailing tile rows");
      double acc[kRows][4];
#pragma unroll
      for (int u = 0; u < kRows; ++u)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[u][q] = 0.0;
      for (int k = 0; k < nbk; ++k) {
        double vr[kRows], wr[kRows], vc[4], wc[4];
#pragma unroll
        for (int u = 0; u < kRows; ++u) {
          vr[u] = Vr[k * kTdTile + ty + (kTdThreads / 16) * u];
          wr[u] = Wr[k * kTdTile + ty + (kTdThreads / 16) * u];
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          vc[q] = Vc[k * kTdTile + tx + 16 * q];
          wc[q] = Wc[k * kTdTile + tx + 16 * q];
        }
#pragma unroll
        for (int u = 0; u < kRows; ++u)
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[u][q] = fma(vr[u], wc[q], fma(wr[u], vc[q], acc[u][q]));
      }
#pragma unroll
      for (int u = 0; u < kRows; ++u) {
        const int r = r0 + ty + (kTdThreads / 16) * u;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int c = c0 + tx + 16 * q;
          double val = 0.0;
          if (r < m && c < m) val = __ldcg(A + static_cast<size_t>(r) * ld + c) - acc[u][q];
          Cs[(ty + (kTdThreads / 16) * u) * (kTdTile + 1) + tx + 16 * q] = val;
        }
      }
      __syncthreads();
      // write the tile's lower part (all of it off the diagonal) and the mirror
      for (int e = t; e < kTdTile * kTdTile; e += kTdThreads) {
        const int rr = e >> 6, cc = e & 63;
        const int r = r0 + rr, c = c0 + cc;
        if (r < m && c < m && (a != b || rr >= cc)) A[static_cast<size_t>(r) * ld + c] = Cs[rr * (kTdTile + 1) + cc];
        // mirror: element (c0 + rr, r0 + cc) = tile element (cc, rr)
        const int mr = c0 + rr, mc = r0 + cc;
        if (mr < m && mc < m && (a != b || cc > rr)) A[static_cast<size_t>(mr) * ld + mc] = Cs[cc * (kTdTile + 1) + rr];
      }
      __syncthreads();
    }
  }
}

// Thread-block cluster helpers: the kernel runs one cluster of C CTAs per
// matrix (C = 1 for large batches).
__device__ __forceinline__ uint32_t cl_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cl_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cl_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
// every thread of every CTA of the cluster; release/acquire at cluster scope
// orders the CTAs' global and shared writes before the other CTAs' reads
__device__ __forceinline__ void cl_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// a double in CTA `rank`'s shared memory at the address of `p` in this CTA
__device__ __forceinline__ double cl_load(const double* p, uint32_t rank) {
  const uint32_t local = static_cast<uint32_t>(__cvta_generic_to_shared(p));
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(rank));
  double v;
  asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(v) : "r"(remote) : "memory");
  return v;
}

__global__ void __launch_bounds__(kTdThreads, 2)
    tridiag_kernel(const EntMat* __restrict__ mats, double* __restrict__ G, double* __restrict__ VW,
                   double* __restrict__ d_out, double* __restrict__ e_out, const EntCtl ctl) {
  extern __shared__ double td_smem[];
  // one cluster of C CTAs per matrix.  Every CTA forms column j, the
  // reflector and v in full (the same arithmetic on the same data, so the
  // same values); the rows j+1 .. m-1 of G0 v, of the dot products and of w
  // are split into C contiguous chunks, and the chunks' partial dot
  // products are summed over the ranks in rank order.
  const int C = static_cast<int>(cl_nctarank());
  const uint32_t rank = cl_ctarank();
  const int p = static_cast<int>(cl_id_x());
  const EntMat mi = mats[p];
  const int m = mi.m, ld = mi.mp;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  double* A = G + mi.off_g;
  double* Vg = VW + mi.off_vw;  // V_k[r] = Vg[k ld + r]
  double* Wg = Vg + static_cast<size_t>(kTdNb) * ld;
  double* d = d_out + mi.sv_off;
  double* e = e_out + mi.sv_off;
  double* x = td_smem;          // column j, rows j .. m-1
  double* v = x + ld;           // reflector, zero outside j+1 .. m-1 (and over the padding)
  double* y = v + ld;           // G0 v, then w (this CTA's rows)
  double* vj = y + ld;          // V_k[j], W_k[j] for the panel's earlier reflectors
  double* wj = vj + kTdNb;
  double* pq = wj + kTdNb;      // [2 kTdNb]: V_k^T v, W_k^T v interleaved
  double* red = pq + 2 * kTdNb; // [kTdWarps]
  double* pq_part = red + kTdWarps;      // [2 kTdNb]: this CTA's chunk of the dots
  double* sv_part = pq_part + 2 * kTdNb; // [1]
  auto csync = [&]() {
    if (C > 1) cl_sync();
    else __syncthreads();
  };

  for (int k = 0; k < m - 1; k += kTdNb) {
    const int nbk = min(kTdNb, m - 1 - k);
    for (int i = 0; i < nbk; ++i) {
      const int j = k + i;
      // this CTA's rows of j+1 .. m-1
      const int chunk = (m - 1 - j + C - 1) / C;
      const int lo = min(m, j + 1 + static_cast<int>(rank) * chunk);
      const int hi = min(m, lo + chunk);
      if (t < i) {
        vj[t] = __ldcg(Vg + static_cast<size_t>(t) * ld + j);
        wj[t] = __ldcg(Wg + static_cast<size_t>(t) * ld + j);
      }
      __syncthreads();
      // column j of the current matrix: row j of G0 minus the panel's terms
      double s2 = 0.0;
      for (int r = j + t; r < m; r += kTdThreads) {
        double a = __ldcg(A + static_cast<size_t>(j) * ld + r);
        for (int c = 0; c < i; ++c)
          a -= fma(__ldcg(Vg + static_cast<size_t>(c) * ld + r), wj[c],
                   __ldcg(Wg + static_cast<size_t>(c) * ld + r) * vj[c]);
        x[r] = a;
        if (r >= j + 2) s2 = fma(a, a, s2);
      }
      s2 = td_block_sum(s2, red);  // also orders the x writes before the reads below
      const double alpha = x[j + 1];
      double tau = 0.0, sc = 0.0, ej = alpha;
      if (s2 != 0.0) {
        const double beta = -copysign(sqrt(fma(alpha, alpha, s2)), alpha);
        tau = (beta - alpha) / beta;
        sc = 1.0 / (alpha - beta);
        ej = beta;
      }
      if (t == 0 && rank == 0) {
        d[j] = x[j];
        e[j] = ej;
      }
      // v over the whole padded range (zero outside j+1 .. m-1); V_i = v on this CTA's rows
      for (int r = t; r < ld; r += kTdThreads) {
        double val = 0.0;
        if (tau != 0.0) {
          if (r == j + 1) val = 1.0;
          else if (r > j + 1 && r < m) val = x[r] * sc;
        }
        v[r] = val;
        if (r >= lo && r < hi) Vg[static_cast<size_t>(i) * ld + r] = val;
      }
      __syncthreads();
      if (tau == 0.0) {  // the reflector is the identity (tau is the same in every thread of the cluster)
        for (int r = lo + t; r < hi; r += kTdThreads) Wg[static_cast<size_t>(i) * ld + r] = 0.0;
        csync();
        continue;
      }
      // y = G0 v over this CTA's rows: each warp takes kSymvRows rows at a
      // time (kTdWarps apart), 16-byte loads from the 64-aligned column at or
      // below j+1 to the padded end (v and the padding are zero there), so
      // that kSymvRows x the unroll depth loads are in flight per lane
      {
        const int cs = (j + 1) & ~63;
        const int nq = (ld - cs) >> 6;
        const double2* vv = reinterpret_cast<const double2*>(v + cs) + lane;
        for (int r = lo + warp; r < hi; r += kSymvRows * kTdWarps) {
          const double2* ap[kSymvRows];
          double sr[kSymvRows];
#pragma unroll
          for (int k = 0; k < kSymvRows; ++k) {
            const int rk = r + k * kTdWarps;
            ap[k] = reinterpret_cast<const double2*>(A + static_cast<size_t>(rk < hi ? rk : r) * ld + cs) + lane;
            sr[k] = 0.0;
          }
#pragma unroll 4
          for (int q = 0; q < nq; ++q) {
            const double2 b = vv[32 * q];
#pragma unroll
            for (int k = 0; k < kSymvRows; ++k) {
              const double2 u = __ldcg(ap[k] + 32 * q);
              sr[k] = fma(u.y, b.y, fma(u.x, b.x, sr[k]));
            }
          }
#pragma unroll
          for (int k = 0; k < kSymvRows; ++k) {
            const double tot = warp_sum(sr[k]);
            if (lane == 0 && r + k * kTdWarps < hi) y[r + k * kTdWarps] = tot;
          }
        }
        // this CTA's chunk of V_k^T v and W_k^T v, one warp per dot
        for (int dd = warp; dd < 2 * i; dd += kTdWarps) {
          const double* src = ((dd & 1) ? Wg : Vg) + static_cast<size_t>(dd >> 1) * ld;
          double s = 0.0;
          for (int r = lo + lane; r < hi; r += 32) s = fma(__ldcg(src + r), v[r], s);
          s = warp_sum(s);
          if (lane == 0) pq_part[dd] = s;
        }
      }
      csync();
      if (t < 2 * i) {
        double s = 0.0;
        for (int q = 0; q < C; ++q) s += (C > 1) ? cl_load(pq_part + t, static_cast<uint32_t>(q)) : pq_part[t];
        pq[t] = s;
      }
      __syncthreads();
      // y <- tau (y - V (W^T v) - W (V^T v)); then w = y - (tau/2)(v^T y) v
      double sv = 0.0;
      for (int r = lo + t; r < hi; r += kTdThreads) {
        double yy = y[r];
        for (int c = 0; c < i; ++c)
          yy -= fma(__ldcg(Vg + static_cast<size_t>(c) * ld + r), pq[2 * c + 1],
                    __ldcg(Wg + static_cast<size_t>(c) * ld + r) * pq[2 * c]);
        yy *= tau;
        y[r] = yy;
        sv = fma(yy, v[r], sv);
      }
      sv = td_block_sum(sv, red);
      if (C > 1) {
        if (t == 0) sv_part[0] = sv;
        csync();
        sv = 0.0;
        for (int q = 0; q < C; ++q) sv += cl_load(sv_part, static_cast<uint32_t>(q));
      }
      const double a2 = -0.5 * tau * sv;
      for (int r = lo + t; r < hi; r += kTdThreads) Wg[static_cast<size_t>(i) * ld + r] = fma(a2, v[r], y[r]);
      csync();  // W_i (and V_i) complete in every CTA of the cluster
    }
    td_trailing_update(A, ld, m, k + nbk, nbk, Vg, Wg, td_smem, static_cast<int>(rank), C);
    csync();
  }
  // the last diagonal element, then the finiteness check of T (rank 0)
  if (rank == 0) {
    if (t == 0) d[m - 1] = __ldcg(A + static_cast<size_t>(m - 1) * ld + m - 1);
    __syncthreads();
    int bad = 0;
    for (int r = t; r < m; r += kTdThreads) {
      if (!isfinite(d[r])) bad = 1;
      if (r < m - 1 && !isfinite(e[r])) bad = 1;
    }
    bad = __syncthreads_or(bad);
    if (t == 0) {
      if (bad) {
        ctl.conv[p] = kConvNonFinite;
        ctl.computed[p] = 0;
        atomicOr(ctl.status, kStatusNonFinite);
      } else {
        ctl.conv[p] = kConvDone;
        ctl.computed[p] = 1;
      }
    }
  }
}

// ---------------------------------------------------------------- 3. bisection
// blocks: (matrix, first eigenvalue index) for every kBisThreads indices.
// Eigenvalue k in ascending order (0-based) is the x where the count of
// eigenvalues below x passes k; it is written at position m-1-k, so each
// matrix's eigenvalues come out descending.
__global__ void __launch_bounds__(kBisThreads) bisect_kernel(const int2* __restrict__ blocks,
                                                             const EntMat* __restrict__ mats,
                                                             const double* __restrict__ d_in,
                                                             const double* __restrict__ e_in,
                                                             double* __restrict__ lam, const EntCtl ctl) {
  extern __shared__ double bis_smem[];
  __shared__ double rlo[kBisThreads / 32], rhi[kBisThreads / 32], rem[kBisThreads / 32];
  const int2 bk = blocks[blockIdx.x];
  const EntMat mi = mats[bk.x];
  if (ctl.conv[bk.x] == kConvNonFinite) return;  // the entropy pass writes NaN for it
  const int m = mi.m, t = threadIdx.x;
  double* dd = bis_smem;     // [m]
  double* e2 = dd + m;       // [m - 1]: e_i^2
  const double* d = d_in + mi.sv_off;
  const double* e = e_in + mi.sv_off;
  // Gershgorin interval of T and the largest e_i^2 (min / max are exact, so
  // the reduction order does not matter)
  double lo = INFINITY, hi = -INFINITY, emax = 0.0;
  for (int i = t; i < m; i += kBisThreads) {
    const double di = d[i];
    const double el = i > 0 ? fabs(e[i - 1]) : 0.0;
    const double er = i < m - 1 ? fabs(e[i]) : 0.0;
    dd[i] = di;
    if (i < m - 1) e2[i] = er * er;
    lo = fmin(lo, di - el - er);
    hi = fmax(hi, di + el + er);
    emax = fmax(emax, er * er);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fmin(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmax(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    emax = fmax(emax, __shfl_xor_sync(0xffffffffu, emax, o));
  }
  if ((t & 31) == 0) {
    rlo[t >> 5] = lo;
    rhi[t >> 5] = hi;
    rem[t >> 5] = emax;
  }
  __syncthreads();
  lo = rlo[0];
  hi = rhi[0];
  emax = rem[0];
  for (int w = 1; w < kBisThreads / 32; ++w) {
    lo = fmin(lo, rlo[w]);
    hi = fmax(hi, rhi[w]);
    emax = fmax(emax, rem[w]);
  }
  const int k = bk.y + t;
  if (k >= m) return;  // no barrier follows
  const double tnorm = fmax(fabs(lo), fabs(hi));
  const double pivmin = DBL_MIN * fmax(1.0, emax);
  // widen the interval by the rounding of the counts themselves
  const double slack = 2.1 * tnorm * DBL_EPSILON * m + 4.2 * pivmin;
  lo -= slack;
  hi += slack;
  const double tol = 2.0 * DBL_EPSILON * tnorm;
  for (int it = 0; it < kBisMaxIter && hi - lo > tol; ++it) {
    const double x = 0.5 * (lo + hi);
    int cnt = 0;
    double q = dd[0] - x;
    if (fabs(q) < pivmin) q = -pivmin;
    cnt += q < 0.0 ? 1 : 0;
    for (int i = 1; i < m; ++i) {
      q = (dd[i] - x) - e2[i - 1] / q;
      if (fabs(q) < pivmin) q = -pivmin;
      cnt += q < 0.0 ? 1 : 0;
    }
    if (cnt > k) hi = x;
    else lo = x;
  }
  lam[mi.sv_off + (m - 1 - k)] = 0.5 * (lo + hi);
}

// ---------------------------------------------------------------- 4. entropy
__global__ void __launch_bounds__(kSortThreads) entropy_kernel(const EntMat* __restrict__ mats, const double* __restrict__ lam_in,
                                                               float* __restrict__ H_out, float* __restrict__ sigma_out,
                                                               const EntCtl ctl) {
  __shared__ float sv[kMaxDim];
  __shared__ double red[kSortThreads];
  const int p = blockIdx.x, t = threadIdx.x;
  const EntMat mi = mats[p];
  const double* lam_p = lam_in + mi.sv_off;
  const bool finite = ctl.conv[p] != kConvNonFinite;
  // sigma_i^2, clamped at 0 (G is positive semi-definite)
  auto lam = [&](int i) {
    const double v = lam_p[i];
    return v > 0.0 ? v : 0.0;
  };
  double s_local = 0.0;
  if (finite)
    for (int i = t; i < mi.m; i += kSortThreads) s_local += lam(i);
  red[t] = s_local;
  __syncthreads();
  for (int s = kSortThreads / 2; s > 0; s >>= 1) {
    if (t < s) red[t] += red[t + s];
    __syncthreads();
  }
  const double total = red[0];
  __syncthreads();
  double h_local = 0.0;
  if (finite && total > 0.0) {
    for (int i = t; i < mi.m; i += kSortThreads) {
      const double q = lam(i) / total;
      if (q > 0.0) h_local += q * log(q);
    }
  }
  red[t] = h_local;
  __syncthreads();
  for (int s = kSortThreads / 2; s > 0; s >>= 1) {
    if (t < s) red[t] += red[t + s];
    __syncthreads();
  }
  if (t == 0) {
    const bool defined = finite && mi.m > 1 && total > 0.0 && isfinite(total);
    H_out[p] = defined ? static_cast<float>(-red[0] / log(static_cast<double>(mi.m))) : __int_as_float(0x7fc00000);
  }
  if (sigma_out == nullptr) return;
  // bitonic sort of the singular values, descending, over the next power of
  // two (pads of -1 sort last)
  int np2 = 1;
  while (np2 < mi.m) np2 <<= 1;
  for (int i = t; i < np2; i += kSortThreads)
    sv[i] = i < mi.m ? (finite ? static_cast<float>(sqrt(lam(i))) : __int_as_float(0x7fc00000)) : -1.0f;
  __syncthreads();
  for (int k = 2; k <= np2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = t; i < np2; i += kSortThreads) {
        const int l = i ^ j;
        if (l > i) {
          const float a = sv[i], b = sv[l];
          const bool desc = (i & k) == 0;
          if (desc ? (a < b) : (a > b)) {
            sv[i] = b;
            sv[l] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  float* out = sigma_out + mi.sv_off;
  for (int i = t; i < mi.m; i += kSortThreads) out[i] = sv[i];
}

}  // namespace
}  // namespace muon

using namespace muon;

struct muon_entropy_plan_s {
  int device = 0;
  int n = 0;
  int ntiles = 0, nbis = 0;
  int mp_max = 64, m_max = 1;
  int td_cluster = 1;     // CTAs per matrix in the tridiagonal reduction
  size_t td_smem = 0;     // its dynamic shared memory per CTA
  int64_t total_sv = 0;
  std::vector<EntMat> mats;
  char* dmem = nullptr;
  double* G = nullptr;
  double* VW = nullptr;
  double* dvec = nullptr;
  double* evec = nullptr;
  double* lam = nullptr;
  EntMat* mats_d = nullptr;
  int4* tiles_d = nullptr;
  int2* bis_d = nullptr;
  const float** wptr_d = nullptr;
  EntCtl ctl{};
  const float** pinned = nullptr;
  std::vector<const float*> cache;
  bool cache_valid = false;
  bool ev_pending = false;
  cudaEvent_t ev = nullptr;
  cudaEvent_t prof[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};
  bool profiling = false;
  bool prof_recorded = false;
  cudaStream_t last_stream = nullptr;
};

namespace {

void free_entropy(muon_entropy_plan_s* pl) {
  if (pl->dmem) cudaFree(pl->dmem);
  if (pl->pinned) cudaFreeHost(pl->pinned);
  if (pl->ev) cudaEventDestroy(pl->ev);
  for (cudaEvent_t e : pl->prof)
    if (e) cudaEventDestroy(e);
  delete pl;
}

size_t align256(size_t b) { return (b + 255) / 256 * 256; }

}  // namespace

extern "C" muon_status_t muon_entropy_init(muon_entropy_plan_t* out, const int64_t* shapes, int32_t n, void* stream) {
  if (out == nullptr || shapes == nullptr || n < 1) return MUON_ERR_INVALID_ARG;
  *out = nullptr;
  for (int i = 0; i < n; ++i) {
    const int64_t r = shapes[2 * i], c = shapes[2 * i + 1];
    if (r < 1 || c < 1 || r > INT32_MAX || c > INT32_MAX || r * c > INT32_MAX) return MUON_ERR_INVALID_ARG;
    if (std::min(r, c) > kMaxDim) return MUON_ERR_UNSUPPORTED;
  }
  int dev = 0;
  cudaDeviceProp prop;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
    cudaGetLastError();
    return MUON_ERR_CUDA;
  }
  if (prop.major != 10 || prop.minor != 0) return MUON_ERR_UNSUPPORTED;
  muon_entropy_plan_s* pl = new (std::nothrow) muon_entropy_plan_s();
  if (pl == nullptr) return MUON_ERR_NO_MEMORY;
  pl->device = dev;
  pl->n = n;
  pl->mats.resize(n);
  std::vector<int4> tiles;
  std::vector<int2> bis;
  int64_t off_g = 0, off_vw = 0, sv = 0;
  for (int i = 0; i < n; ++i) {
    EntMat& mi = pl->mats[i];
    mi.rows = static_cast<int>(shapes[2 * i]);
    mi.cols = static_cast<int>(shapes[2 * i + 1]);
    mi.m = std::min(mi.rows, mi.cols);
    mi.n = std::max(mi.rows, mi.cols);
    mi.tall = mi.rows > mi.cols ? 1 : 0;
    mi.mp = (mi.m + kPad - 1) / kPad * kPad;
    mi.off_g = off_g;
    mi.off_vw = off_vw;
    mi.sv_off = sv;
    off_g += static_cast<int64_t>(align256(static_cast<size_t>(mi.mp) * mi.mp * sizeof(double)) / sizeof(double));
    off_vw += static_cast<int64_t>(2) * kTdNb * mi.mp;
    sv += mi.m;
    pl->mp_max = std::max(pl->mp_max, mi.mp);
    pl->m_max = std::max(pl->m_max, mi.m);
    const int nt = (mi.mp + kGramTile - 1) / kGramTile;
    for (int a = 0; a < nt; ++a)
      for (int b = 0; b <= a; ++b) tiles.push_back(make_int4(i, a, b, 0));
    for (int k = 0; k < mi.m; k += kBisThreads) bis.push_back(make_int2(i, k));
  }
  pl->ntiles = static_cast<int>(tiles.size());
  pl->nbis = static_cast<int>(bis.size());
  pl->total_sv = sv;

  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  const size_t o_g = take(static_cast<size_t>(off_g) * sizeof(double));
  const size_t o_vw = take(static_cast<size_t>(off_vw) * sizeof(double));
  const size_t o_d = take(static_cast<size_t>(sv) * sizeof(double));
  const size_t o_e = take(static_cast<size_t>(sv) * sizeof(double));
  const size_t o_l = take(static_cast<size_t>(sv) * sizeof(double));
  const size_t o_m = take(n * sizeof(EntMat));
  const size_t o_t = take(tiles.size() * sizeof(int4));
  const size_t o_b = take(bis.size() * sizeof(int2));
  const size_t o_w = take(n * sizeof(float*));
  const size_t o_conv = take(n * sizeof(int));
  const size_t o_sw = take(n * sizeof(int));
  const size_t o_st = take(sizeof(unsigned));
  if (cudaMalloc(&pl->dmem, off) != cudaSuccess) {
    cudaGetLastError();
    free_entropy(pl);
    return MUON_ERR_NO_MEMORY;
  }
  char* b = pl->dmem;
  pl->G = reinterpret_cast<double*>(b + o_g);
  pl->VW = reinterpret_cast<double*>(b + o_vw);
  pl->dvec = reinterpret_cast<double*>(b + o_d);
  pl->evec = reinterpret_cast<double*>(b + o_e);
  pl->lam = reinterpret_cast<double*>(b + o_l);
  pl->mats_d = reinterpret_cast<EntMat*>(b + o_m);
  pl->tiles_d = reinterpret_cast<int4*>(b + o_t);
  pl->bis_d = reinterpret_cast<int2*>(b + o_b);
  pl->wptr_d = reinterpret_cast<const float**>(b + o_w);
  pl->ctl.conv = reinterpret_cast<int*>(b + o_conv);
  pl->ctl.computed = reinterpret_cast<int*>(b + o_sw);
  pl->ctl.status = reinterpret_cast<unsigned*>(b + o_st);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  bool ok = cudaMemcpy(pl->mats_d, pl->mats.data(), n * sizeof(EntMat), cudaMemcpyHostToDevice) == cudaSuccess &&
            cudaMemcpy(pl->tiles_d, tiles.data(), tiles.size() * sizeof(int4), cudaMemcpyHostToDevice) == cudaSuccess &&
            cudaMemcpy(pl->bis_d, bis.data(), bis.size() * sizeof(int2), cudaMemcpyHostToDevice) == cudaSuccess &&
            cudaMemset(pl->ctl.status, 0, sizeof(unsigned)) == cudaSuccess &&
            cudaMemset(pl->ctl.computed, 0, n * sizeof(int)) == cudaSuccess;
  ok = ok && cudaHostAlloc(reinterpret_cast<void**>(&pl->pinned), n * sizeof(float*), cudaHostAllocDefault) ==
                 cudaSuccess;
  ok = ok && cudaEventCreateWithFlags(&pl->ev, cudaEventDisableTiming) == cudaSuccess;
  for (int k = 0; k < 5 && ok; ++k) ok = cudaEventCreate(&pl->prof[k]) == cudaSuccess;
  // Cluster size of the reduction: the largest C in {16, 8, 4, 2} for which
  // all n clusters are resident at once with one CTA per SM (a plan of a
  // few large matrices then spreads each matrix over C SMs); otherwise one
  // CTA per matrix, two per SM.
  const size_t smem1 = tridiag_smem_bytes(pl->mp_max);
  const size_t smem_c = std::max(smem1, kTdSpreadSmem);
  ok = ok && cudaFuncSetAttribute(tridiag_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(smem_c)) == cudaSuccess;
  if (ok) {
    const bool nonportable =
        cudaFuncSetAttribute(tridiag_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
    cudaGetLastError();
    pl->td_cluster = 1;
    pl->td_smem = smem1;
    for (int c : {16, 8, 4, 2}) {
      if (c > 8 && !nonportable) continue;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(c, 1, 1);
      cfg.blockDim = dim3(kTdThreads, 1, 1);
      cfg.dynamicSmemBytes = smem_c;
      cudaLaunchAttribute at;
      at.id = cudaLaunchAttributeClusterDimension;
      at.val.clusterDim.x = c;
      at.val.clusterDim.y = 1;
      at.val.clusterDim.z = 1;
      cfg.attrs = &at;
      cfg.numAttrs = 1;
      int nc = 0;
      if (cudaOccupancyMaxActiveClusters(&nc, tridiag_kernel, &cfg) == cudaSuccess && nc >= n) {
        pl->td_cluster = c;
        pl->td_smem = smem_c;
        break;
      }
      cudaGetLastError();
    }
  }
  ok = ok && cudaFuncSetAttribute(gram_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(kGramSmem)) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(bisect_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(2 * pl->m_max * sizeof(double))) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    free_entropy(pl);
    return MUON_ERR_CUDA;
  }
  pl->last_stream = st;
  *out = pl;
  return MUON_OK;
}

extern "C" muon_status_t muon_entropy_compute(muon_entropy_plan_t pl, const float* const* W, int32_t n, float* H_out,
                                              float* sigma_out, void* stream) {
  if (pl == nullptr || W == nullptr || H_out == nullptr) return MUON_ERR_INVALID_ARG;
  if (n != pl->n) return MUON_ERR_SHAPE_MISMATCH;
  std::vector<ByteRange> spans;
  spans.reserve(n + 2);
  std::vector<const float*> t(n);
  for (int i = 0; i < n; ++i) {
    if (W[i] == nullptr || reinterpret_cast<uintptr_t>(W[i]) % sizeof(float) != 0) return MUON_ERR_INVALID_ARG;
    const uintptr_t w = reinterpret_cast<uintptr_t>(W[i]);
    spans.push_back({w, w + static_cast<size_t>(pl->mats[i].rows) * pl->mats[i].cols * sizeof(float)});
    t[i] = W[i];
  }
  // the inputs may overlap one another (they are only read); the outputs may not touch them
  std::sort(spans.begin(), spans.end(), [](const ByteRange& a, const ByteRange& b) { return a.lo < b.lo; });
  auto hits_inputs = [&](uintptr_t lo, uintptr_t hi) {
    for (const ByteRange& s : spans)
      if (lo < s.hi && s.lo < hi) return true;
    return false;
  };
  const uintptr_t h = reinterpret_cast<uintptr_t>(H_out);
  if (h % sizeof(float) != 0) return MUON_ERR_INVALID_ARG;
  if (hits_inputs(h, h + n * sizeof(float))) return MUON_ERR_ALIAS;
  if (sigma_out != nullptr) {
    const uintptr_t s = reinterpret_cast<uintptr_t>(sigma_out);
    if (s % sizeof(float) != 0) return MUON_ERR_INVALID_ARG;
    if (hits_inputs(s, s + pl->total_sv * sizeof(float))) return MUON_ERR_ALIAS;
    std::vector<ByteRange> outs{{h, h + n * sizeof(float)}, {s, s + pl->total_sv * sizeof(float)}};
    if (any_overlap(outs)) return MUON_ERR_ALIAS;
  }
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != pl->device) return MUON_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!(pl->cache_valid && std::memcmp(t.data(), pl->cache.data(), n * sizeof(float*)) == 0)) {
    if (pl->ev_pending) {
      if (cudaEventSynchronize(pl->ev) != cudaSuccess) return MUON_ERR_CUDA;
      pl->ev_pending = false;
    }
    std::memcpy(pl->pinned, t.data(), n * sizeof(float*));
    if (cudaMemcpyAsync(pl->wptr_d, pl->pinned, n * sizeof(float*), cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaEventRecord(pl->ev, st) != cudaSuccess) {
      cudaGetLastError();
      return MUON_ERR_CUDA;
    }
    pl->ev_pending = true;
    pl->cache = t;
    pl->cache_valid = true;
  }
  const EntCtl ctl = pl->ctl;
  bool ok = cudaMemsetAsync(ctl.conv, 0, n * sizeof(int), st) == cudaSuccess &&
            cudaMemsetAsync(ctl.computed, 0, n * sizeof(int), st) == cudaSuccess;
  if (ok && pl->profiling) ok = cudaEventRecord(pl->prof[0], st) == cudaSuccess;
  if (ok) gram_kernel<<<pl->ntiles, kGramThreads, kGramSmem, st>>>(pl->tiles_d, pl->mats_d, pl->wptr_d, pl->G);
  if (ok && pl->profiling) ok = cudaEventRecord(pl->prof[1], st) == cudaSuccess;
  if (ok) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(n * pl->td_cluster), 1, 1);
    cfg.blockDim = dim3(kTdThreads, 1, 1);
    cfg.dynamicSmemBytes = pl->td_smem;
    cfg.stream = st;
    cudaLaunchAttribute at;
    at.id = cudaLaunchAttributeClusterDimension;
    at.val.clusterDim.x = static_cast<unsigned>(pl->td_cluster);
    at.val.clusterDim.y = 1;
    at.val.clusterDim.z = 1;
    cfg.attrs = &at;
    cfg.numAttrs = 1;
    ok = cudaLaunchKernelEx(&cfg, tridiag_kernel, static_cast<const EntMat*>(pl->mats_d), pl->G, pl->VW, pl->dvec,
                            pl->evec, ctl) == cudaSuccess;
  }
  if (ok && pl->profiling) ok = cudaEventRecord(pl->prof[2], st) == cudaSuccess;
  if (ok)
    bisect_kernel<<<pl->nbis, kBisThreads, 2 * pl->m_max * sizeof(double), st>>>(pl->bis_d, pl->mats_d, pl->dvec,
                                                                                 pl->evec, pl->lam, ctl);
  if (ok && pl->profiling) ok = cudaEventRecord(pl->prof[3], st) == cudaSuccess;
  if (ok) entropy_kernel<<<n, kSortThreads, 0, st>>>(pl->mats_d, pl->lam, H_out, sigma_out, ctl);
  if (ok && pl->profiling) ok = cudaEventRecord(pl->prof[4], st) == cudaSuccess;
  if (!ok || cudaGetLastError() != cudaSuccess) {
    cudaGetLastError();
    return MUON_ERR_CUDA;
  }
  pl->prof_recorded = pl->profiling;
  pl->last_stream = st;
  return MUON_OK;
}

extern "C" muon_status_t muon_entropy_get_status(muon_entropy_plan_t pl, int32_t* computed_out) {
  if (pl == nullptr) return MUON_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(pl->last_stream) != cudaSuccess) {
    cudaGetLastError();
    return MUON_ERR_CUDA;
  }
  unsigned s = 0;
  if (cudaMemcpy(&s, pl->ctl.status, sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemset(pl->ctl.status, 0, sizeof(unsigned)) != cudaSuccess ||
      (computed_out != nullptr &&
       cudaMemcpy(computed_out, pl->ctl.computed, pl->n * sizeof(int32_t), cudaMemcpyDeviceToHost) != cudaSuccess)) {
    cudaGetLastError();
    return MUON_ERR_CUDA;
  }
  if (s & kStatusNonFinite) return MUON_ERR_NONFINITE;
  return MUON_OK;
}

extern "C" muon_status_t muon_entropy_profile(muon_entropy_plan_t pl, int32_t enable, double* ms_out) {
  if (pl == nullptr) return MUON_ERR_INVALID_ARG;
  if (ms_out != nullptr) {
    if (!pl->prof_recorded) return MUON_ERR_INVALID_ARG;
    if (cudaEventSynchronize(pl->prof[4]) != cudaSuccess) {
      cudaGetLastError();
      return MUON_ERR_CUDA;
    }
    for (int k = 0; k < 4; ++k) {
      float ms = 0.0f;
      if (cudaEventElapsedTime(&ms, pl->prof[k], pl->prof[k + 1]) != cudaSuccess) {
        cudaGetLastError();
        return MUON_ERR_CUDA;
      }
      ms_out[k] = ms;
    }
  }
  pl->profiling = enable != 0;
  return MUON_OK;
}

extern "C" int64_t muon_entropy_num_singular_values(muon_entropy_plan_t pl) {
  return pl == nullptr ? -1 : pl->total_sv;
}

extern "C" int32_t muon_entropy_cluster_size(muon_entropy_plan_t pl) { return pl == nullptr ? -1 : pl->td_cluster; }

extern "C" void muon_entropy_destroy(muon_entropy_plan_t pl) {
  if (pl == nullptr) return;
  cudaStreamSynchronize(pl->last_stream);
  cudaGetLastError();
  free_entropy(pl);
}
