// SVD-entropy diagnostic of weight matrices.
//
// "Muon is Scalable for LLM Training", Sec. 3.4 ("Dynamics of singular
// spectrum", the SVD-entropy equation and Fig. 4) compares optimisers by the
// SVD entropy of each weight matrix:
//   H(sigma) = -(1 / log n) sum_i p_i log p_i,  p_i = sigma_i^2 / sum_j sigma_j^2
// over its n = min(rows, cols) singular values.
//
// sigma_i^2 are the eigenvalues of the Gram matrix G = X X^T of the wide
// orientation X (m x n, m <= n) of W.  The path, all matrices of a plan per
// launch:
//   1. gram_kernel: G in fp64 on the CUDA cores (64 x 64 tiles of the lower
//      triangle, each also written mirrored), zero-padded to m_pad, a
//      multiple of 64.  Products of fp32 entries are exact in fp64.
//   2. Two-sided block Jacobi on G.  The 32-row blocks are paired by a
//      round-robin tournament, nb - 1 rounds per sweep.  In a round, every
//      pair's 64 x 64 subproblem [G_PP G_PQ; G_QP G_QQ] gets one sweep of
//      cyclic Jacobi in shared memory (jacobi_solve_kernel), which keeps the
//      accumulated rotation V (re-orthonormalised by one polar Newton-Schulz
//      step at the end); then G <- J^T G J for the block-diagonal J of all
//      pairs, one 64 x 64 super-block per CTA iteration
//      (jacobi_update_kernel: two small GEMMs, V_u^T T V_v).
//   3. After each sweep, off_norm_kernel and converge_kernel compare the
//      off-diagonal Frobenius norm with ||G||_F (fp64, fixed order).  A
//      matrix below kOffTol is done; once all are done, every later launch
//      returns at once.
//   4. entropy_kernel: the diagonal now holds sigma_i^2.  fp64 sums in a
//      fixed order give H; a bitonic sort gives the singular values,
//      descending.
// The zero padding never mixes with the matrix: a padded index has a zero
// row and column, so every rotation that touches it is the identity.
// Everything is deterministic (no atomics, fixed reduction orders).
//
// The arithmetic is fp64 throughout.  H weighs every eigenvalue by
// -p log p, whose slope is unbounded near p = 0: with an fp32 Gram matrix the
// rounding floor (about 1e-7 of the largest eigenvalue) alone moved H of a
// rank-10 200 x 300 matrix by about 6e-5.
#include "muon.h"
#include "muon_internal.cuh"

#include <algorithm>
#include <cmath>
#include <cstring>
#include <new>
#include <vector>

namespace muon {
namespace {

constexpr int kEb = 32;              // rows of a Jacobi block
constexpr int kEs = 2 * kEb;         // order of a block-pair subproblem
constexpr int kEsLd = kEs + 1;       // shared-memory row pitch (conflict-free columns)
constexpr int kEsElems = kEs * kEs;  // 4096
constexpr int kEThreads = 256;
constexpr int kGramTile = 64;
constexpr int kGramK = 32;
constexpr int kMaxSweeps = 24;
// One cyclic sweep per subproblem and round: solving the 64 x 64 problems to
// convergence (up to 10 sweeps) saved at most one outer sweep in fp64
// simulations of 704 x 704 Gram matrices (Gaussian: 11 against 10; three
// decades of singular values: 17 against 17) for five times the inner work.
constexpr int kInnerSweeps = 1;
constexpr int kMaxDim = 8192;        // min(rows, cols) limit (the sort stages 8192 values)
constexpr int kSortThreads = 1024;
// A pair (a, b) of a subproblem is rotated when |S_ab| > kInnerTol max(|S_aa|, |S_bb|):
// a skipped entry moves an eigenvalue by at most S_ab^2 / |S_aa - S_bb|, or by
// |S_ab| itself for a near-degenerate pair.
constexpr double kInnerTol = 1e-13;
// A matrix is done when off(G) <= kOffTol ||G||_F (Frobenius norms).  The
// rest moves the eigenvalues by second-order amounts: in the same
// simulations at most 3e-9 of the largest eigenvalue, and H by 1e-10, far
// below the rounding of the fp32 outputs.
constexpr double kOffTol = 1e-6;
constexpr size_t kSolveSmem = 2 * kEs * kEsLd * sizeof(double);
constexpr size_t kUpdSmem = 3 * kEs * (kEs + 2) * sizeof(double);

// conv[] values
constexpr int kConvRunning = 0;
constexpr int kConvDone = 1;
constexpr int kConvNonFinite = 2;

struct EntMat {
  int rows, cols;
  int m, n;         // min and max of rows, cols
  int tall;         // rows > cols: X = W^T
  int nb;           // 32-row blocks, even; m_pad = 32 nb
  int rb_first;     // first row block of this matrix in the off-norm partials
  int pad_;
  int64_t off_g;    // doubles into the G workspace (m_pad x m_pad, row-major)
  int64_t off_v;    // doubles into the rotation store (nb / 2 blocks of 64 x 64)
  int64_t sv_off;   // first singular value of this matrix in sigma_out
};

struct EntCtl {
  int* conv;        // [n] kConv*
  int* sweeps;      // [n] sweeps until done (0: not done)
  int* all_done;    // [1] every matrix is done
  unsigned* status; // [1] sticky: kStatusNonFinite, kStatusNotConverged
};

constexpr unsigned kStatusNotConverged = 4u;

// round-robin tournament over nb players (nb even), round r in [0, nb - 1):
// player nb - 1 meets r, and for u >= 1 player (r + u) mod (nb - 1) meets
// (r - u) mod (nb - 1).  Every pair meets once per nb - 1 rounds.
__host__ __device__ __forceinline__ int2 tournament(int nb, int r, int u) {
  int a, b;
  if (u == 0) {
    a = nb - 1;
    b = r;
  } else {
    a = (r + u) % (nb - 1);
    b = (r - u + (nb - 1)) % (nb - 1);
  }
  return make_int2(a < b ? a : b, a < b ? b : a);
}

// row of G for index a in [0, 64) of the subproblem of block pair (P, Q)
__device__ __forceinline__ int sub_row(int2 pq, int a) { return a < kEb ? pq.x * kEb + a : pq.y * kEb + (a - kEb); }

// ---------------------------------------------------------------- 1. Gram
__device__ __forceinline__ float x_at(const float* W, const EntMat& mi, int i, int k) {
  if (i >= mi.m || k >= mi.n) return 0.0f;
  return mi.tall ? __ldg(W + static_cast<size_t>(k) * mi.cols + i) : __ldg(W + static_cast<size_t>(i) * mi.cols + k);
}

__global__ void __launch_bounds__(kEThreads) gram_kernel(const int4* __restrict__ tiles, const EntMat* __restrict__ mats,
                                                         const float* const* __restrict__ wptr, double* __restrict__ G) {
  // the K-loop staging (As, Bs) and the output tile (Cs) share one buffer
  __shared__ double buf[kGramTile * (kGramTile + 1)];
  float (*As)[kGramTile + 1] = reinterpret_cast<float (*)[kGramTile + 1]>(buf);
  float (*Bs)[kGramTile + 1] = As + kGramK;
  double (*Cs)[kGramTile + 1] = reinterpret_cast<double (*)[kGramTile + 1]>(buf);
  const int4 td = tiles[blockIdx.x];
  const EntMat mi = mats[td.x];
  const float* W = wptr[td.x];
  const int i0 = td.y * kGramTile, j0 = td.z * kGramTile;
  const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
  double acc[4][4];
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int w = 0; w < 4; ++w) acc[q][w] = 0.0;
  for (int k0 = 0; k0 < mi.n; k0 += kGramK) {
    // stage X[i0 + r][k0 + k] and X[j0 + r][k0 + k] as [k][r]; the global
    // reads run along W's contiguous dimension
    for (int e = t; e < kGramTile * kGramK; e += kEThreads) {
      int r, k;
      if (mi.tall) {
        k = e >> 6;
        r = e & 63;
      } else {
        r = e >> 5;
        k = e & 31;
      }
      As[k][r] = x_at(W, mi, i0 + r, k0 + k);
      Bs[k][r] = x_at(W, mi, j0 + r, k0 + k);
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < kGramK; ++k) {
      double a[4], b[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        a[q] = As[k][ty * 4 + q];
        b[q] = Bs[k][tx + 16 * q];
      }
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[q][w] = fma(a[q], b[w], acc[q][w]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int w = 0; w < 4; ++w) Cs[ty * 4 + q][tx + 16 * w] = acc[q][w];
  __syncthreads();
  double* g = G + mi.off_g;
  const size_t ld = static_cast<size_t>(kEb) * mi.nb;
  for (int e = t; e < kGramTile * kGramTile; e += kEThreads) {
    const int r = e >> 6, c = e & 63;
    g[(i0 + r) * ld + j0 + c] = Cs[r][c];
    if (td.y != td.z) g[(j0 + r) * ld + i0 + c] = Cs[c][r];
  }
}

// ---------------------------------------------------------------- 2a. subproblem solve
// 64 x 64 product C = A^T B or A B (row pitch kEsLd) into acc: thread
// (tx, ty) owns rows 4 ty + q and columns tx + 16 w, so a warp reads 16
// consecutive doubles of a row of B (no bank conflicts) and broadcasts A
template <bool kTransA>
__device__ __forceinline__ void small_gemm(const double* A, const double* B, double (&acc)[4][4], int tx, int ty) {
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int w = 0; w < 4; ++w) acc[q][w] = 0.0;
#pragma unroll 4
  for (int k = 0; k < kEs; ++k) {
    double a[4], b[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      a[q] = kTransA ? A[k * kEsLd + ty * 4 + q] : A[(ty * 4 + q) * kEsLd + k];
      b[q] = B[k * kEsLd + tx + 16 * q];
    }
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int w = 0; w < 4; ++w) acc[q][w] = fma(a[q], b[w], acc[q][w]);
  }
}

// Cyclic Jacobi on S (64 x 64, symmetric) with the same tournament over its
// 64 indices: 63 rounds of 32 disjoint rotations per sweep.  For a pair with
// alpha = S_aa, beta = S_bb, gamma = S_ab the rotation J = [c s; -s c] zeroes
// S_ab in J^T S J when t = s / c is the smaller root of t^2 + 2 tau t - 1 = 0,
// tau = (beta - alpha) / (2 gamma) (the symmetric 2 x 2 Schur decomposition);
// with d = beta - alpha that root is t = 2 gamma sgn(d) / (|d| + sqrt(d^2 + 4 gamma^2)).
// A round applies its rotations to the rows of S, then to the columns of S
// and V; each warp works on one pair and 32 consecutive rows or columns.
__global__ void __launch_bounds__(kEThreads) jacobi_solve_kernel(const int2* __restrict__ pairs, int npairs,
                                                                 const EntMat* __restrict__ mats, const double* __restrict__ G,
                                                                 double* __restrict__ Vst, const EntCtl ctl, int round) {
  extern __shared__ double smem_d[];
  double* S = smem_d;
  double* V = S + kEs * kEsLd;
  __shared__ double rc[kEb], rs[kEb];
  __shared__ int ra[kEb], rb[kEb];
  if (*ctl.all_done) return;
  const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
  for (int item = blockIdx.x; item < npairs; item += gridDim.x) {
    const int2 pm = pairs[item];
    const EntMat mi = mats[pm.x];
    if (ctl.conv[pm.x] != kConvRunning || round >= mi.nb - 1) continue;
    const int2 pq = tournament(mi.nb, round, pm.y);
    const double* g = G + mi.off_g;
    const size_t ld = static_cast<size_t>(kEb) * mi.nb;
    __syncthreads();  // the previous item's V has been written out
    for (int e = t; e < kEsElems; e += kEThreads) {
      const int a = e >> 6, b = e & 63;
      S[a * kEsLd + b] = g[sub_row(pq, a) * ld + sub_row(pq, b)];
      V[a * kEsLd + b] = (a == b) ? 1.0 : 0.0;
    }
    __syncthreads();
    for (int sweep = 0; sweep < kInnerSweeps; ++sweep) {
      int rotated = 0;
      for (int rr = 0; rr < kEs - 1; ++rr) {
        int rot = 0;
        if (t < kEb) {
          const int2 ab = tournament(kEs, rr, t);
          const double alpha = S[ab.x * kEsLd + ab.x], beta = S[ab.y * kEsLd + ab.y], gamma = S[ab.x * kEsLd + ab.y];
          double c = 1.0, s = 0.0;
          if (fabs(gamma) > kInnerTol * fmax(fabs(alpha), fabs(beta))) {
            const double d = beta - alpha;
            const double tt = (d >= 0.0 ? 2.0 * gamma : -2.0 * gamma) / (fabs(d) + sqrt(fma(d, d, 4.0 * gamma * gamma)));
            c = rsqrt(fma(tt, tt, 1.0));
            s = tt * c;
            rot = 1;
          }
          ra[t] = ab.x;
          rb[t] = ab.y;
          rc[t] = c;
          rs[t] = s;
        }
        if (!__syncthreads_or(rot)) continue;  // nothing to rotate in this round
        rotated = 1;
        // rows: S <- J^T S (pair k, column j; a warp takes one pair, 32 columns)
        for (int e = t; e < kEb * kEs; e += kEThreads) {
          const int k = e >> 6, j = e & 63;
          const double c = rc[k], s = rs[k];
          if (s == 0.0) continue;
          const int a = ra[k], b = rb[k];
          const double sa = S[a * kEsLd + j], sb = S[b * kEsLd + j];
          S[a * kEsLd + j] = c * sa - s * sb;
          S[b * kEsLd + j] = s * sa + c * sb;
        }
        __syncthreads();
        // columns: S <- S J and V <- V J (pair k, row i; a warp takes one pair, 32 rows)
        for (int e = t; e < kEb * kEs; e += kEThreads) {
          const int k = e >> 6, i = e & 63;
          const double c = rc[k], s = rs[k];
          if (s == 0.0) continue;
          const int a = ra[k], b = rb[k];
          const double sa = S[i * kEsLd + a], sb = S[i * kEsLd + b];
          S[i * kEsLd + a] = c * sa - s * sb;
          S[i * kEsLd + b] = s * sa + c * sb;
          const double va = V[i * kEsLd + a], vb = V[i * kEsLd + b];
          V[i * kEsLd + a] = c * va - s * vb;
          V[i * kEsLd + b] = s * va + c * vb;
        }
        __syncthreads();
      }
      if (!__syncthreads_or(rotated)) break;
    }
    // Hundreds of rotations leave V a few hundred ulps from orthogonal, and
    // the update would scale G's eigenvalues by that much every round.  One
    // Newton-Schulz step towards the polar factor, V <- V - V (V^T V - I) / 2,
    // squares the error (down to rounding).  E = V^T V - I goes into S.
    double acc[4][4];
    small_gemm<true>(V, V, acc, tx, ty);
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int w = 0; w < 4; ++w)
        S[(ty * 4 + q) * kEsLd + tx + 16 * w] = acc[q][w] - ((ty * 4 + q == tx + 16 * w) ? 1.0 : 0.0);
    __syncthreads();
    small_gemm<false>(V, S, acc, tx, ty);
    double* vout = Vst + mi.off_v + static_cast<size_t>(pm.y) * kEsElems;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = ty * 4 + q;
#pragma unroll
      for (int w = 0; w < 4; ++w) vout[i * kEs + tx + 16 * w] = fma(-0.5, acc[q][w], V[i * kEsLd + tx + 16 * w]);
    }
  }
}

// ---------------------------------------------------------------- 2b. G <- J^T G J
// Super-block (u, v), u <= v: T = G[rows of pair u][rows of pair v] (64 x 64)
// becomes V_u^T T V_v, and its transpose is written to (v, u).
// Shared memory holds T transposed (Tt), R = T V_v and one rotation block
// (V_v, then V_u), each 64 rows of kUpdLd doubles (16-byte aligned rows).
// Thread (tx, ty) owns rows 4 ty + q and columns 2 tx + {0, 1} + 32 {0, 1} of
// each product, so every operand fetch is a double2: the A side is a
// broadcast within a half-warp, the B side 256 contiguous bytes.
constexpr int kUpdLd = kEs + 2;

// acc[q][w] = sum_k A[k][4 ty + q] B[k][col(w)], A and B row-major with pitch kUpdLd
__device__ __forceinline__ void gemm_tn(const double* A, const double* B, double (&acc)[4][4], int tx, int ty) {
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int w = 0; w < 4; ++w) acc[q][w] = 0.0;
#pragma unroll 4
  for (int k = 0; k < kEs; ++k) {
    const double2 a01 = *reinterpret_cast<const double2*>(A + k * kUpdLd + ty * 4);
    const double2 a23 = *reinterpret_cast<const double2*>(A + k * kUpdLd + ty * 4 + 2);
    const double2 b01 = *reinterpret_cast<const double2*>(B + k * kUpdLd + tx * 2);
    const double2 b23 = *reinterpret_cast<const double2*>(B + k * kUpdLd + tx * 2 + 32);
    const double a[4] = {a01.x, a01.y, a23.x, a23.y};
    const double b[4] = {b01.x, b01.y, b23.x, b23.y};
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int w = 0; w < 4; ++w) acc[q][w] = fma(a[q], b[w], acc[q][w]);
  }
}

__device__ __forceinline__ int upd_col(int tx, int w) { return tx * 2 + (w & 1) + 32 * (w >> 1); }

__global__ void __launch_bounds__(kEThreads) jacobi_update_kernel(const int4* __restrict__ sblk, int nsblk,
                                                                  const EntMat* __restrict__ mats, double* __restrict__ G,
                                                                  const double* __restrict__ Vst, const EntCtl ctl, int round) {
  extern __shared__ __align__(16) double smem_d[];
  double* Tt = smem_d;             // T transposed, then T' (row-major)
  double* R = Tt + kEs * kUpdLd;   // T V_v
  double* Vb = R + kEs * kUpdLd;   // V_v, then V_u
  if (*ctl.all_done) return;
  const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
  for (int item = blockIdx.x; item < nsblk; item += gridDim.x) {
    const int4 sb = sblk[item];
    const EntMat mi = mats[sb.x];
    if (ctl.conv[sb.x] != kConvRunning || round >= mi.nb - 1) continue;
    const int2 pu = tournament(mi.nb, round, sb.y), pv = tournament(mi.nb, round, sb.z);
    double* g = G + mi.off_g;
    const size_t ld = static_cast<size_t>(kEb) * mi.nb;
    const double* vu = Vst + mi.off_v + static_cast<size_t>(sb.y) * kEsElems;
    const double* vv = Vst + mi.off_v + static_cast<size_t>(sb.z) * kEsElems;
    __syncthreads();  // the previous item's T' has been written out
    for (int e = t; e < kEsElems; e += kEThreads) {
      const int a = e >> 6, b = e & 63;
      Tt[b * kUpdLd + a] = g[sub_row(pu, a) * ld + sub_row(pv, b)];
      Vb[a * kUpdLd + b] = vv[e];
    }
    __syncthreads();
    double acc[4][4];
    gemm_tn(Tt, Vb, acc, tx, ty);  // R = T V_v
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int w = 0; w < 4; ++w) R[(ty * 4 + q) * kUpdLd + upd_col(tx, w)] = acc[q][w];
    __syncthreads();
    for (int e = t; e < kEsElems; e += kEThreads) Vb[(e >> 6) * kUpdLd + (e & 63)] = vu[e];
    __syncthreads();
    gemm_tn(Vb, R, acc, tx, ty);   // T' = V_u^T R
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int w = 0; w < 4; ++w) Tt[(ty * 4 + q) * kUpdLd + upd_col(tx, w)] = acc[q][w];
    __syncthreads();
    const bool diag = (sb.y == sb.z);
    for (int e = t; e < kEsElems; e += kEThreads) {
      const int a = e >> 6, b = e & 63;
      if (diag) {
        // keep G exactly symmetric: the lower half, mirrored
        g[sub_row(pu, a) * ld + sub_row(pu, b)] = (a >= b) ? Tt[a * kUpdLd + b] : Tt[b * kUpdLd + a];
      } else {
        g[sub_row(pu, a) * ld + sub_row(pv, b)] = Tt[a * kUpdLd + b];
        g[sub_row(pv, a) * ld + sub_row(pu, b)] = Tt[b * kUpdLd + a];
      }
    }
  }
}

// ---------------------------------------------------------------- 3. convergence
// Per 32-row block: fp64 sums of the squared off-diagonal and diagonal entries.
__global__ void __launch_bounds__(kEThreads) off_norm_kernel(const int2* __restrict__ rblk, const EntMat* __restrict__ mats,
                                                             const double* __restrict__ G, double* __restrict__ part,
                                                             const EntCtl ctl) {
  __shared__ double red[2][kEThreads];
  if (*ctl.all_done) return;
  const int2 rm = rblk[blockIdx.x];
  const EntMat mi = mats[rm.x];
  if (ctl.conv[rm.x] != kConvRunning) return;
  const int mp = kEb * mi.nb;
  const double* g = G + mi.off_g + static_cast<size_t>(rm.y) * kEb * mp;
  double off = 0.0, dia = 0.0;
  for (int e = threadIdx.x; e < kEb * mp; e += kEThreads) {
    const int r = e / mp, c = e - r * mp;
    const double v = g[e];
    if (c == rm.y * kEb + r) dia += v * v;
    else off += v * v;
  }
  red[0][threadIdx.x] = off;
  red[1][threadIdx.x] = dia;
  __syncthreads();
  for (int s = kEThreads / 2; s > 0; s >>= 1) {
    if (threadIdx.x < s) {
      red[0][threadIdx.x] += red[0][threadIdx.x + s];
      red[1][threadIdx.x] += red[1][threadIdx.x + s];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    part[2 * blockIdx.x] = red[0][0];
    part[2 * blockIdx.x + 1] = red[1][0];
  }
}

__global__ void converge_kernel(const EntMat* __restrict__ mats, int n, const double* __restrict__ part,
                                const EntCtl ctl, int sweep, int last) {
  if (*ctl.all_done) return;
  __shared__ int running;
  if (threadIdx.x == 0) running = 0;
  __syncthreads();
  for (int p = threadIdx.x; p < n; p += blockDim.x) {
    if (ctl.conv[p] == kConvRunning) {
      const EntMat& mi = mats[p];
      double off = 0.0, dia = 0.0;
      for (int k = 0; k < mi.nb; ++k) {
        off += part[2 * (mi.rb_first + k)];
        dia += part[2 * (mi.rb_first + k) + 1];
      }
      if (!isfinite(off) || !isfinite(dia)) {
        ctl.conv[p] = kConvNonFinite;
        atomicOr(ctl.status, kStatusNonFinite);
      } else if (off <= kOffTol * kOffTol * (off + dia)) {
        ctl.conv[p] = kConvDone;
        ctl.sweeps[p] = sweep + 1;
      } else if (last) {
        atomicOr(ctl.status, kStatusNotConverged);
      } else {
        running = 1;
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && (!running || last)) *ctl.all_done = 1;
}

// ---------------------------------------------------------------- 4. entropy
__global__ void __launch_bounds__(kSortThreads) entropy_kernel(const EntMat* __restrict__ mats, const double* __restrict__ G,
                                                               float* __restrict__ H_out, float* __restrict__ sigma_out,
                                                               const EntCtl ctl) {
  __shared__ float sv[kMaxDim];
  __shared__ double red[kSortThreads];
  const int p = blockIdx.x, t = threadIdx.x;
  const EntMat mi = mats[p];
  const double* g = G + mi.off_g;
  const size_t ld = static_cast<size_t>(kEb) * mi.nb;
  const bool finite = ctl.conv[p] != kConvNonFinite;
  // sigma_i^2 = G_ii, clamped at 0 (G is positive semi-definite)
  auto lam = [&](int i) {
    const double v = g[i * ld + i];
    return v > 0.0 ? v : 0.0;
  };
  double s_local = 0.0;
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
  if (total > 0.0) {
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
  int nb_max = 2;
  int ntiles = 0, npairs = 0, nsblk = 0, nrb = 0;
  int grid_solve = 1, grid_update = 1;
  int64_t total_sv = 0;
  std::vector<EntMat> mats;
  char* dmem = nullptr;
  double* G = nullptr;
  double* V = nullptr;
  EntMat* mats_d = nullptr;
  int4* tiles_d = nullptr;
  int2* pairs_d = nullptr;
  int4* sblk_d = nullptr;
  int2* rb_d = nullptr;
  double* part_d = nullptr;
  const float** wptr_d = nullptr;
  EntCtl ctl{};
  const float** pinned = nullptr;
  std::vector<const float*> cache;
  bool cache_valid = false;
  bool ev_pending = false;
  cudaEvent_t ev = nullptr;
  cudaEvent_t prof[4] = {nullptr, nullptr, nullptr, nullptr};
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
  std::vector<int4> tiles, sblk;
  std::vector<int2> pairs, rbs;
  int64_t off_g = 0, off_v = 0, sv = 0;
  for (int i = 0; i < n; ++i) {
    EntMat& mi = pl->mats[i];
    mi.rows = static_cast<int>(shapes[2 * i]);
    mi.cols = static_cast<int>(shapes[2 * i + 1]);
    mi.m = std::min(mi.rows, mi.cols);
    mi.n = std::max(mi.rows, mi.cols);
    mi.tall = mi.rows > mi.cols ? 1 : 0;
    int nb = (mi.m + kEb - 1) / kEb;
    nb += nb & 1;
    mi.nb = nb;
    mi.rb_first = static_cast<int>(rbs.size());
    mi.pad_ = 0;
    mi.off_g = off_g;
    mi.off_v = off_v;
    mi.sv_off = sv;
    const int mp = kEb * nb;
    off_g += static_cast<int64_t>(align256(static_cast<size_t>(mp) * mp * sizeof(double)) / sizeof(double));
    off_v += static_cast<int64_t>(nb / 2) * kEsElems;
    sv += mi.m;
    pl->nb_max = std::max(pl->nb_max, nb);
    const int nt = mp / kGramTile;
    for (int a = 0; a < nt; ++a)
      for (int b = 0; b <= a; ++b) tiles.push_back(make_int4(i, a, b, 0));
    for (int u = 0; u < nb / 2; ++u) pairs.push_back(make_int2(i, u));
    for (int u = 0; u < nb / 2; ++u)
      for (int v = u; v < nb / 2; ++v) sblk.push_back(make_int4(i, u, v, 0));
    for (int k = 0; k < nb; ++k) rbs.push_back(make_int2(i, k));
  }
  pl->ntiles = static_cast<int>(tiles.size());
  pl->npairs = static_cast<int>(pairs.size());
  pl->nsblk = static_cast<int>(sblk.size());
  pl->nrb = static_cast<int>(rbs.size());
  pl->total_sv = sv;
  const int sms = prop.multiProcessorCount;
  pl->grid_solve = std::max(1, std::min(pl->npairs, sms * 3));
  pl->grid_update = std::max(1, std::min(pl->nsblk, sms * 2));

  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  const size_t o_g = take(static_cast<size_t>(off_g) * sizeof(double));
  const size_t o_v = take(static_cast<size_t>(off_v) * sizeof(double));
  const size_t o_m = take(n * sizeof(EntMat));
  const size_t o_t = take(tiles.size() * sizeof(int4));
  const size_t o_p = take(pairs.size() * sizeof(int2));
  const size_t o_s = take(sblk.size() * sizeof(int4));
  const size_t o_r = take(rbs.size() * sizeof(int2));
  const size_t o_part = take(rbs.size() * 2 * sizeof(double));
  const size_t o_w = take(n * sizeof(float*));
  const size_t o_conv = take(n * sizeof(int));
  const size_t o_sw = take(n * sizeof(int));
  const size_t o_ad = take(sizeof(int));
  const size_t o_st = take(sizeof(unsigned));
  if (cudaMalloc(&pl->dmem, off) != cudaSuccess) {
    cudaGetLastError();
    free_entropy(pl);
    return MUON_ERR_NO_MEMORY;
  }
  char* b = pl->dmem;
  pl->G = reinterpret_cast<double*>(b + o_g);
  pl->V = reinterpret_cast<double*>(b + o_v);
  pl->mats_d = reinterpret_cast<EntMat*>(b + o_m);
  pl->tiles_d = reinterpret_cast<int4*>(b + o_t);
  pl->pairs_d = reinterpret_cast<int2*>(b + o_p);
  pl->sblk_d = reinterpret_cast<int4*>(b + o_s);
  pl->rb_d = reinterpret_cast<int2*>(b + o_r);
  pl->part_d = reinterpret_cast<double*>(b + o_part);
  pl->wptr_d = reinterpret_cast<const float**>(b + o_w);
  pl->ctl.conv = reinterpret_cast<int*>(b + o_conv);
  pl->ctl.sweeps = reinterpret_cast<int*>(b + o_sw);
  pl->ctl.all_done = reinterpret_cast<int*>(b + o_ad);
  pl->ctl.status = reinterpret_cast<unsigned*>(b + o_st);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  bool ok = cudaMemcpy(pl->mats_d, pl->mats.data(), n * sizeof(EntMat), cudaMemcpyHostToDevice) == cudaSuccess &&
            cudaMemcpy(pl->tiles_d, tiles.data(), tiles.size() * sizeof(int4), cudaMemcpyHostToDevice) == cudaSuccess &&
            cudaMemcpy(pl->pairs_d, pairs.data(), pairs.size() * sizeof(int2), cudaMemcpyHostToDevice) == cudaSuccess &&
            cudaMemcpy(pl->sblk_d, sblk.data(), sblk.size() * sizeof(int4), cudaMemcpyHostToDevice) == cudaSuccess &&
            cudaMemcpy(pl->rb_d, rbs.data(), rbs.size() * sizeof(int2), cudaMemcpyHostToDevice) == cudaSuccess &&
            cudaMemset(pl->ctl.status, 0, sizeof(unsigned)) == cudaSuccess &&
            cudaMemset(pl->ctl.sweeps, 0, n * sizeof(int)) == cudaSuccess;
  ok = ok && cudaHostAlloc(reinterpret_cast<void**>(&pl->pinned), n * sizeof(float*), cudaHostAllocDefault) ==
                 cudaSuccess;
  ok = ok && cudaEventCreateWithFlags(&pl->ev, cudaEventDisableTiming) == cudaSuccess;
  for (int k = 0; k < 4 && ok; ++k) ok = cudaEventCreate(&pl->prof[k]) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(jacobi_solve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(kSolveSmem)) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(jacobi_update_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(kUpdSmem)) == cudaSuccess;
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
            cudaMemsetAsync(ctl.sweeps, 0, n * sizeof(int), st) == cudaSuccess &&
            cudaMemsetAsync(ctl.all_done, 0, sizeof(int), st) == cudaSuccess;
  if (ok && pl->profiling) ok = cudaEventRecord(pl->prof[0], st) == cudaSuccess;
  if (ok) gram_kernel<<<pl->ntiles, kEThreads, 0, st>>>(pl->tiles_d, pl->mats_d, pl->wptr_d, pl->G);
  if (ok && pl->profiling) ok = cudaEventRecord(pl->prof[1], st) == cudaSuccess;
  for (int sweep = 0; ok && sweep < kMaxSweeps; ++sweep) {
    for (int r = 0; r < pl->nb_max - 1; ++r) {
      jacobi_solve_kernel<<<pl->grid_solve, kEThreads, kSolveSmem, st>>>(pl->pairs_d, pl->npairs, pl->mats_d, pl->G,
                                                                         pl->V, ctl, r);
      jacobi_update_kernel<<<pl->grid_update, kEThreads, kUpdSmem, st>>>(pl->sblk_d, pl->nsblk, pl->mats_d, pl->G,
                                                                         pl->V, ctl, r);
    }
    off_norm_kernel<<<pl->nrb, kEThreads, 0, st>>>(pl->rb_d, pl->mats_d, pl->G, pl->part_d, ctl);
    converge_kernel<<<1, 1024, 0, st>>>(pl->mats_d, n, pl->part_d, ctl, sweep, sweep == kMaxSweeps - 1 ? 1 : 0);
  }
  if (ok && pl->profiling) ok = cudaEventRecord(pl->prof[2], st) == cudaSuccess;
  if (ok) entropy_kernel<<<n, kSortThreads, 0, st>>>(pl->mats_d, pl->G, H_out, sigma_out, ctl);
  if (ok && pl->profiling) ok = cudaEventRecord(pl->prof[3], st) == cudaSuccess;
  if (!ok || cudaGetLastError() != cudaSuccess) {
    cudaGetLastError();
    return MUON_ERR_CUDA;
  }
  pl->prof_recorded = pl->profiling;
  pl->last_stream = st;
  return MUON_OK;
}

extern "C" muon_status_t muon_entropy_get_status(muon_entropy_plan_t pl, int32_t* sweeps_out) {
  if (pl == nullptr) return MUON_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(pl->last_stream) != cudaSuccess) {
    cudaGetLastError();
    return MUON_ERR_CUDA;
  }
  unsigned s = 0;
  if (cudaMemcpy(&s, pl->ctl.status, sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemset(pl->ctl.status, 0, sizeof(unsigned)) != cudaSuccess ||
      (sweeps_out != nullptr &&
       cudaMemcpy(sweeps_out, pl->ctl.sweeps, pl->n * sizeof(int32_t), cudaMemcpyDeviceToHost) != cudaSuccess)) {
    cudaGetLastError();
    return MUON_ERR_CUDA;
  }
  if (s & kStatusNonFinite) return MUON_ERR_NONFINITE;
  if (s & kStatusNotConverged) return MUON_ERR_NOT_CONVERGED;
  return MUON_OK;
}

extern "C" muon_status_t muon_entropy_profile(muon_entropy_plan_t pl, int32_t enable, double* ms_out) {
  if (pl == nullptr) return MUON_ERR_INVALID_ARG;
  if (ms_out != nullptr) {
    if (!pl->prof_recorded) return MUON_ERR_INVALID_ARG;
    if (cudaEventSynchronize(pl->prof[3]) != cudaSuccess) {
      cudaGetLastError();
      return MUON_ERR_CUDA;
    }
    for (int k = 0; k < 3; ++k) {
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

extern "C" void muon_entropy_destroy(muon_entropy_plan_t pl) {
  if (pl == nullptr) return;
  cudaStreamSynchronize(pl->last_stream);
  cudaGetLastError();
  free_entropy(pl);
}
