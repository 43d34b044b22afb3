// Newton-Schulz products on the 5th-generation tensor cores (sm_100a).
//
// One launch computes one phase of one quintic iteration ("Muon is Scalable
// for LLM Training", Sec. 2.1, Eq. 2, factored as A = X X^T, B = b A + c A^2,
// X' = a X + B X) for every matrix of the plan:
//   kPhaseGram   A  = scale * X X^T         (wide)   or Y^T Y (tall)  [m, m]
//   kPhasePoly   B  = b A + c A A            (A symmetric, so A A = A A^T)
//   kPhaseUpdate X' = alpha (a X + B X)      (wide)   or Y' = alpha (a Y + Y B) (tall)
// with scale = s^2 and alpha = s on iteration 0 (s = 1/||Y||_F folds the
// normalisation X_0 = Y/||Y||_F into the first products), 1 afterwards.  The
// last X update instead applies the weight update of Eq. 4 (or stores O).
//
// Kernel structure: persistent, one CTA per SM, warp specialised.
//   warp 0      TMA producer: 64x64 bf16 boxes (128-byte swizzle) into a
//               kStages-deep ring of shared-memory stages, mbarrier tx-count.
//   warp 1      TMEM allocator and MMA issuer: tcgen05.mma kind::f16,
//               M=128, N<=256, K=16, bf16 operands, fp32 accumulators in TMEM;
//               two accumulators so the epilogue of one tile overlaps the
//               main loop of the next.  K-major or MN-major operands are a
//               descriptor choice, so tall matrices are never transposed.
//   warps 2..5  epilogue: tcgen05.ld of 32 columns at a time, fused
//               polynomial/update arithmetic, direct vector stores.
// Symmetric outputs (A, B) are computed only for tiles that touch the lower
// triangle; each entry is written exactly once, either directly (i >= j) or
// through its mirror (i > j), so the result is symmetric bit for bit.
// Every mbarrier wait is bounded by time; on timeout the CTA raises a status
// bit, stops issuing work, drains what it has in flight, frees TMEM and exits.
#include "muon_internal.cuh"

#include <cuda.h>

namespace muon {
namespace {

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0u;
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for the phase with the given parity to complete; false after
// kWaitLimitNs or as soon as another role of this CTA raised `abort`.
__device__ __noinline__ bool wait_bounded(uint32_t bar, uint32_t parity, const volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0u) {
      if (abort_flag != nullptr && *abort_flag) return false;
      if (global_ns() - t0 > kWaitLimitNs) return false;
    }
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(dst),
      "l"(tmap), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor for a 128-byte-swizzled canonical layout.
//   K-major : rows of 64 bf16 (128 B) at 128-byte pitch; SBO = 1024 B between
//             8-row groups; LBO unused (16 B).
//   MN-major: 64 contiguous MN elements per 128-byte row, one row per k;
//             SBO = 1024 B between 8-k groups, LBO = 8 KiB between 64-wide
//             MN blocks (one TMA box each).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1u) << 46;  // descriptor version of sm_100
  d |= static_cast<uint64_t>(2u) << 61;  // 128-byte swizzle
  return d;
}

// Instruction descriptor of kind::f16: bf16 x bf16 -> fp32, M = 128.
__device__ __forceinline__ uint32_t make_idesc(int n, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(a_mn) << 15) |
         (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(kBM >> 4) << 24);
}

// ---------------------------------------------------------------- shared memory plan
struct SmemLayout {
  static constexpr int kA = 0;
  static constexpr int kB = kA + kStages * kStageABytes;
  static constexpr int kBar = kB + kStages * kStageBBytes;
  // barriers: full[kStages], empty[kStages], tfull[2], tempty[2], drain
  static constexpr int kNumBars = 2 * kStages + 5;
  static constexpr int kMisc = kBar + kNumBars * 8;  // tmem base (u32), abort (int)
  static constexpr int kBytes = kMisc + 16;
};
constexpr int kSmemBytes = SmemLayout::kBytes + 1024;  // + alignment slack

// Operand selection of one tile.
struct Operand {
  const void* tmap;
  int mn;  // 1: MN-major (column-contiguous), 0: K-major
};

struct TileCfg {
  int p, row0, col0, n_need, n_mma, nb_b, nk, skip;
  Operand a, b;
};

__device__ __forceinline__ const void* tmap_of(const GemmArgs& g, int p, int which) {
  return static_cast<const uint8_t*>(g.tmaps) + (static_cast<size_t>(p) * 4 + which) * 128;
}

__device__ __forceinline__ TileCfg decode_tile(const GemmArgs& g, int t) {
  const TileDesc d = g.tiles[t];
  TileCfg c;
  c.p = d.x;
  c.row0 = d.y;
  c.col0 = d.z;
  c.n_need = d.w;
  c.n_mma = (c.n_need + 15) & ~15;
  c.nb_b = (c.n_mma + kBox - 1) / kBox;
  const MatInfo& mi = g.mats[c.p];
  const int hi = g.cur;  // tensor map 0/1 = hi buffers
  int K;
  if (g.phase == kPhaseGram) {
    K = mi.n;
    c.a = {tmap_of(g, c.p, hi), mi.tall};
    c.b = c.a;
  } else if (g.phase == kPhasePoly) {
    K = mi.m;
    c.a = {tmap_of(g, c.p, 2), 0};
    c.b = c.a;
  } else {
    K = mi.m;
    if (mi.tall) {
      c.a = {tmap_of(g, c.p, hi), 0};
      c.b = {tmap_of(g, c.p, 3), 0};
    } else {
      c.a = {tmap_of(g, c.p, 3), 0};
      c.b = {tmap_of(g, c.p, hi), 1};
    }
  }
  c.nk = (K + kBK - 1) / kBK;
  c.skip = (g.ws.s[c.p] == 0.0f) ? 1 : 0;
  return c;
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, unsigned* status) {
  *abort_flag = 1;
  atomicOr(status, kStatusTimeout);
}

// ---------------------------------------------------------------- epilogue helpers
__device__ __forceinline__ float u2f(uint32_t v) { return __uint_as_float(v); }

__device__ __forceinline__ void load_bf16x32(const __nv_bfloat16* p, float* out) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 v = q[i];
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(h[k]);
      out[8 * i + 2 * k] = f.x;
      out[8 * i + 2 * k + 1] = f.y;
    }
  }
}

__device__ __forceinline__ void store_bf16x8(__nv_bfloat16* p, const __nv_bfloat16* v) {
  *reinterpret_cast<uint4*>(p) = *reinterpret_cast<const uint4*>(v);
}

// Symmetric output chunk: row i, columns j0..j0+31 of an [m, m] matrix.
__device__ __forceinline__ void store_sym_chunk(__nv_bfloat16* out, int lda, int m, int i, int j0,
                                                const float* val) {
  __align__(16) __nv_bfloat16 h[32];
#pragma unroll
  for (int q = 0; q < 32; ++q) h[q] = __float2bfloat16_rn(val[q]);
  __nv_bfloat16* row = out + static_cast<size_t>(i) * lda;
  if (j0 + 31 <= i && j0 + 32 <= m) {
#pragma unroll
    for (int q = 0; q < 32; q += 8) store_bf16x8(row + j0 + q, h + q);
  } else {
#pragma unroll
    for (int q = 0; q < 32; ++q) {
      const int j = j0 + q;
      if (j <= i && j < m) row[j] = h[q];
    }
  }
  // mirror of the strictly lower part: out[j, i] for j < i
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    const int j = j0 + q;
    if (j < i && j < m) out[static_cast<size_t>(j) * lda + i] = h[q];
  }
}

// ---------------------------------------------------------------- the kernel
__global__ void __launch_bounds__(kGemmThreads, 1) ns_gemm_kernel(const __grid_constant__ GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + SmemLayout::kBar;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * kStages + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * kStages + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SmemLayout::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SmemLayout::kMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), kEpiWarps * 32);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  unsigned* status = g.ws.status;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long fills = 0;
      for (int t = blockIdx.x; t < g.ntiles && !*abort_flag; t += gridDim.x) {
        const TileCfg c = decode_tile(g, t);
        if (c.skip) continue;
        const uint32_t bytes = static_cast<uint32_t>((2 + c.nb_b) * kBoxBytes);
        for (int kb = 0; kb < c.nk; ++kb) {
          if (!wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag)) {
            raise_abort(abort_flag, status);
            break;
          }
          const uint32_t fb = full_bar(stage);
          mbar_arrive_expect_tx(fb, bytes);
          const uint32_t sa = sbase + SmemLayout::kA + stage * kStageABytes;
          const uint32_t sb = sbase + SmemLayout::kB + stage * kStageBBytes;
          const int k0 = kb * kBK;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (c.a.mn) tma_load_2d(sa + h * kBoxBytes, c.a.tmap, c.row0 + h * kBox, k0, fb);
            else        tma_load_2d(sa + h * kBoxBytes, c.a.tmap, k0, c.row0 + h * kBox, fb);
          }
          for (int h = 0; h < c.nb_b; ++h) {
            if (c.b.mn) tma_load_2d(sb + h * kBoxBytes, c.b.tmap, c.col0 + h * kBox, k0, fb);
            else        tma_load_2d(sb + h * kBoxBytes, c.b.tmap, k0, c.col0 + h * kBox, fb);
          }
          ++fills;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain: every stage's most recent fill must have landed before exit.
      for (int s = 0; s < kStages; ++s) {
        const long cnt = fills / kStages + ((s < fills % kStages) ? 1 : 0);
        if (cnt > 0 && !wait_bounded(full_bar(s), static_cast<uint32_t>((cnt - 1) & 1), nullptr))
          atomicOr(status, kStatusTimeout);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool issued = false;
      for (int t = blockIdx.x; t < g.ntiles && !*abort_flag; t += gridDim.x) {
        const TileCfg c = decode_tile(g, t);
        if (c.skip) continue;
        if (!wait_bounded(tempty_bar(acc), acc_phase ^ 1u, abort_flag)) {
          raise_abort(abort_flag, status);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
        const uint32_t idesc = make_idesc(c.n_mma, c.a.mn, c.b.mn);
        const uint32_t a_lbo = c.a.mn ? kBoxBytes : 16u, b_lbo = c.b.mn ? kBoxBytes : 16u;
        const uint32_t a_step = c.a.mn ? 2u * 1024u : 32u, b_step = c.b.mn ? 2u * 1024u : 32u;
        bool ok = true;
        for (int kb = 0; kb < c.nk; ++kb) {
          if (!wait_bounded(full_bar(stage), phase, abort_flag)) {
            raise_abort(abort_flag, status);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = sbase + SmemLayout::kA + stage * kStageABytes;
          const uint32_t sb = sbase + SmemLayout::kB + stage * kStageBBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
            const uint64_t ad = smem_desc(sa + kk * a_step, a_lbo, 1024u);
            const uint64_t bd = smem_desc(sb + kk * b_step, b_lbo, 1024u);
            tc_mma(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          issued = true;
          tc_commit(empty_bar(stage));  // frees the stage once these MMAs have read it
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(tfull_bar(acc));  // accumulator complete
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (issued) {
        tc_commit(drain_bar);
        if (!wait_bounded(drain_bar, 0u, nullptr)) atomicOr(status, kStatusTimeout);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;          // 0..kEpiWarps-1
    const int quad = warp & 3;        // TMEM lane quadrant this warp may access
    const int r_in_tile = quad * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    const float a_c = g.sc.a, b_c = g.sc.b, c_c = g.sc.c;
    for (int t = blockIdx.x; t < g.ntiles; t += gridDim.x) {
      if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;  // warp-uniform exit
      const TileCfg c = decode_tile(g, t);
      const MatInfo& mi = g.mats[c.p];
      const int final_tile = (g.phase == kPhaseUpdate && g.final_mode != kFinalNone);
      if (c.skip && !final_tile) continue;
      const int i = c.row0 + r_in_tile;
      const int nch = (c.n_need + 31) >> 5;
      float rms = 0.0f;
      if (c.skip) {
        // Y == 0: O = 0, so the step is pure weight decay (or a zero output).
        // Rows go to warps and columns to lanes so the stores coalesce.
        const MatPtrs pt = g.ptrs[c.p];
        for (int rr = ew; rr < kBM; rr += kEpiWarps) {
          const int r = c.row0 + rr;
          if (r >= mi.rows) break;
          float* wrow = pt.W + static_cast<size_t>(r) * mi.cols;
          for (int j = c.col0 + lane; j < c.col0 + c.n_need; j += 32) {
            if (g.final_mode == kFinalWeight) wrow[j] = wrow[j] - g.sc.lr * (g.sc.wd * wrow[j]);
            else wrow[j] = 0.0f;
          }
        }
      } else {
        // one lane waits and the warp follows its verdict, so the warp stays
        // converged for the .sync.aligned TMEM loads
        int ready = 0;
        if (lane == 0) ready = wait_bounded(tfull_bar(acc), acc_phase, abort_flag) ? 1 : 0;
        ready = __shfl_sync(0xffffffffu, ready, 0);
        if (!ready) {
          if (lane == 0) raise_abort(abort_flag, status);
          break;
        }
        tc_fence_after();
        const uint32_t t_row = tmem_base + static_cast<uint32_t>(acc * kBN) + (static_cast<uint32_t>(quad * 32) << 16);
        const float s = g.ws.s[c.p];
        for (int ch = 0; ch < nch; ++ch) {
          uint32_t v[32];
          __syncwarp();
          tmem_ld32(t_row + static_cast<uint32_t>(ch * 32), v);
          tmem_ld_wait();
          const int j0 = c.col0 + ch * 32;
          float val[32];
          if (g.phase == kPhaseGram) {
            if (i < mi.m) {
              const bool first = (g.iter == 0);
#pragma unroll
              for (int q = 0; q < 32; ++q) val[q] = first ? (u2f(v[q]) * s) * s : u2f(v[q]);
              store_sym_chunk(g.ws.A + mi.off_a, mi.lda, mi.m, i, j0, val);
            }
          } else if (g.phase == kPhasePoly) {
            if (i < mi.m) {
              const __nv_bfloat16* arow = g.ws.A + mi.off_a + static_cast<size_t>(i) * mi.lda;
              float av[32];
              if (j0 + 32 <= mi.m) {
                load_bf16x32(arow + j0, av);
              } else {
#pragma unroll
                for (int q = 0; q < 32; ++q) av[q] = (j0 + q < mi.m) ? __bfloat162float(arow[j0 + q]) : 0.0f;
              }
#pragma unroll
              for (int q = 0; q < 32; ++q) val[q] = fmaf(c_c, u2f(v[q]), b_c * av[q]);
              store_sym_chunk(g.ws.B + mi.off_a, mi.lda, mi.m, i, j0, val);
            }
          } else {
            if (i < mi.rows) {
              const float alpha = (g.iter == 0) ? s : 1.0f;
              const size_t wi = static_cast<size_t>(mi.off_x) + static_cast<size_t>(i) * mi.ld + j0;
              const __nv_bfloat16* hrow = g.ws.hi[g.cur] + wi;
              const __nv_bfloat16* lrow = g.ws.lo + wi;
              const bool full = (j0 + 32 <= mi.cols);
              float xh[32], xl[32];
              if (full) {
                load_bf16x32(hrow, xh);
                load_bf16x32(lrow, xl);
              } else {
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                  const bool in = (j0 + q < mi.cols);
                  xh[q] = in ? __bfloat162float(hrow[q]) : 0.0f;
                  xl[q] = in ? __bfloat162float(lrow[q]) : 0.0f;
                }
              }
#pragma unroll
              for (int q = 0; q < 32; ++q) val[q] = alpha * fmaf(a_c, xh[q] + xl[q], u2f(v[q]));
              if (g.final_mode == kFinalNone) {
                __align__(16) __nv_bfloat16 h[32];
                __align__(16) __nv_bfloat16 l[32];
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                  h[q] = __float2bfloat16_rn(val[q]);
                  l[q] = __float2bfloat16_rn(val[q] - __bfloat162float(h[q]));
                }
                __nv_bfloat16* hout = g.ws.hi[g.cur ^ 1] + wi;
                __nv_bfloat16* lout = g.ws.lo + wi;
                if (full) {
#pragma unroll
                  for (int q = 0; q < 32; q += 8) {
                    store_bf16x8(hout + q, h + q);
                    store_bf16x8(lout + q, l + q);
                  }
                } else {
#pragma unroll
                  for (int q = 0; q < 32; ++q)
                    if (j0 + q < mi.cols) {
                      hout[q] = h[q];
                      lout[q] = l[q];
                    }
                }
              } else {
                const MatPtrs pt = g.ptrs[c.p];
                float* wrow = pt.W + static_cast<size_t>(i) * mi.cols + j0;
                const float scale = g.sc.rms_scale * sqrtf(static_cast<float>(mi.n));
#pragma unroll
                for (int q = 0; q < 32; ++q)
                  if (j0 + q < mi.cols) rms = fmaf(val[q], val[q], rms);
                if (full && pt.vec_ok) {
                  float4* w4 = reinterpret_cast<float4*>(wrow);
#pragma unroll
                  for (int q = 0; q < 8; ++q) {
                    float4 w = w4[q];
                    if (g.final_mode == kFinalWeight) {
                      w.x = w.x - g.sc.lr * fmaf(scale, val[4 * q + 0], g.sc.wd * w.x);
                      w.y = w.y - g.sc.lr * fmaf(scale, val[4 * q + 1], g.sc.wd * w.y);
                      w.z = w.z - g.sc.lr * fmaf(scale, val[4 * q + 2], g.sc.wd * w.z);
                      w.w = w.w - g.sc.lr * fmaf(scale, val[4 * q + 3], g.sc.wd * w.w);
                    } else {
                      w = make_float4(val[4 * q], val[4 * q + 1], val[4 * q + 2], val[4 * q + 3]);
                    }
                    w4[q] = w;
                  }
                } else {
#pragma unroll
                  for (int q = 0; q < 32; ++q) {
                    if (j0 + q < mi.cols) {
                      if (g.final_mode == kFinalWeight) {
                        const float w = wrow[q];
                        wrow[q] = w - g.sc.lr * fmaf(scale, val[q], g.sc.wd * w);
                      } else {
                        wrow[q] = val[q];
                      }
                    }
                  }
                }
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(tempty_bar(acc));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (final_tile) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) rms += __shfl_xor_sync(0xffffffffu, rms, o);
        if (lane == 0) {
          const int tiles_c = (mi.cols + kBN - 1) / kBN;
          const int local = (c.row0 / kBM) * tiles_c + c.col0 / kBN;
          g.ws.rms_part[mi.rms_tile_base + local * kEpiWarps + ew] = rms;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
  }
}

}  // namespace

int gemm_tc_smem_bytes() { return kSmemBytes; }

cudaError_t launch_gemm_tc(const GemmArgs& args, int grid, cudaStream_t st) {
  static unsigned long long configured = 0;  // one bit per device ordinal
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(configured & (1ull << dev))) {
    e = cudaFuncSetAttribute(ns_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    if (dev < 64) configured |= (1ull << dev);
  }
  if (args.ntiles == 0) return cudaSuccess;
  ns_gemm_kernel<<<grid, kGemmThreads, kSmemBytes, st>>>(args);
  return cudaGetLastError();
}

}  // namespace muon
