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
// Structure: persistent 2-CTA clusters (one CTA per SM).  A pair owns a
// 256 x 256 output tile; tcgen05.mma.cta_group::2 (M = 256, N <= 256, K = 16,
// bf16 operands, fp32 accumulators in TMEM) reads 128 A rows and N/2 B rows
// from each CTA's shared memory, so each SM streams 64 KiB per 128-deep K
// stage for 16.8 MFLOP of the pair.  Per CTA:
//   warp 0      TMA producer: four lanes each issue one 64 x 128 bf16 box
//               (128-byte swizzle) per 128-deep K stage into a ring of 3
//               stages (2 for the X update, which gives its epilogue the
//               room); both CTAs' loads complete on the leader's "full" barrier.
//   warp 1      TMEM allocator (both CTAs) and MMA issuer (leader only); two
//               256-column accumulators so the epilogue of one tile overlaps
//               the main loop of the next.
//   warps 2..9  epilogue: two warps per TMEM lane quadrant, each owning whole
//               32 x 32 blocks (tcgen05.ld of 32 columns, one row per thread),
//               fused arithmetic, and coalesced 64-byte row-segment stores
//               through warp-private swizzled staging blocks.  The X update
//               feeds its hi/lo inputs through a per-warp cp.async ring.
#include "muon_internal.cuh"

#include <cuda.h>

namespace muon {
namespace {

#ifndef MUON_TC_STAGES
#define MUON_TC_STAGES 3
#endif
constexpr int kStages = MUON_TC_STAGES;   // stages of the Gram and polynomial phases
constexpr int kStagesUpd = 2;              // stages of the X-update phase
constexpr int kStageABytes = kHalfM * kBK * 2;   // 32 KiB: this CTA's 128 A rows x 128 K
constexpr int kStageBBytes = 128 * kBK * 2;      // 32 KiB: up to 128 B rows (half of N) x 128 K
// Epilogue: two groups of four warps (one warp per TMEM lane quadrant each);
// group g takes the 32-column chunks g, g+2, ... of every tile, so each warp
// owns whole 32 x 32 blocks.  Each warp has 4 KiB of shared memory: two
// 32 x 32 bf16 blocks through which its inputs and outputs are transposed
// between coalesced global accesses (64-byte row segments) and the
// row-per-thread layout of the TMEM accumulator.  The epilogue uses no TMA,
// so its traffic never queues behind the main loop's operand copies.
constexpr int kEpiGroups = 2;
constexpr int kEpiBlockBytes = 32 * 32 * 2;               // 2 KiB
constexpr int kEpiWarpBytes = 2 * kEpiBlockBytes;         // 4 KiB
constexpr int kEpiBytes = kEpiWarps * kEpiWarpBytes;      // 32 KiB
constexpr int kWarpProducer = 0, kWarpMma = 1, kWarpEpi0 = 2;
constexpr int kThreads = 32 * (kWarpEpi0 + kEpiWarps);

// X-update epilogue: per warp a ring of 3 buffers, each a 32 x 32 hi block and
// lo block (4 KiB), filled by cp.async.  With 2 main-loop stages the free
// shared memory is [64 KiB, 96 KiB) and [160 KiB, 224 KiB): 24 buffers.
constexpr int kUpdBufs = 3;
constexpr int kUpdBufBytes = 2 * kEpiBlockBytes;

struct SmemLayout {
  static constexpr int kA = 0;
  static constexpr int kB = kA + kStages * kStageABytes;
  static constexpr int kEpi = kB + kStages * kStageBBytes;
  static constexpr int kUpdLo = kA + kStagesUpd * kStageABytes;  // [64 KiB, 96 KiB)
  static constexpr int kUpdHi = kB + kStagesUpd * kStageBBytes;  // [160 KiB, 224 KiB)
  static constexpr int kBar = kEpi + kEpiBytes;
  // full[S], empty[S], tfull[2], tempty[2], drain
  static constexpr int kNumBars = 2 * kStages + 5;
  static constexpr int kMisc = kBar + kNumBars * 8;  // tmem base (u32), abort (int)
  static constexpr int kBytes = kMisc + 16;
};
constexpr int kSmemBytes = SmemLayout::kBytes + 1024;  // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget");

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t cta_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t num_clusters_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}

// shared::cta address -> shared::cluster address of the same object in CTA `rank`
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// arrive on a barrier given by its shared::cluster address (may be the peer's)
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
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

// TMA load into this CTA's shared memory, completing on a barrier that may
// live in the peer CTA (2-CTA form, no multicast).
__device__ __forceinline__ void tma_load_pair(uint32_t dst, const void* tmap, int x, int y, uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(dst),
      "l"(tmap), "r"(x), "r"(y), "r"(bar_cluster)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Arrive on a barrier (shared::cluster address) once all prior tcgen05 ops of
// this thread have completed.
__device__ __forceinline__ void tc_commit(uint32_t bar_cluster) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_cluster)
               : "memory");
}

__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
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
// A stage holds each operand as two 16 KiB TMA boxes (64 contiguous x 128).
//   K-major : box h holds K [64h, 64h+64) for 128 rows, one 128-byte row per
//             MN index; SBO = 1024 B between 8-row groups, LBO unused (16 B).
//   MN-major: box h holds MN [64h, 64h+64) for all 128 k, one 128-byte row per
//             k; SBO = 1024 B between 8-k groups, LBO = 16 KiB between boxes.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1u) << 46;  // descriptor version of sm_100
  d |= static_cast<uint64_t>(2u) << 61;  // 128-byte swizzle
  return d;
}

// Instruction descriptor of kind::f16: bf16 x bf16 -> fp32, M = 256 (pair).
__device__ __forceinline__ uint32_t make_idesc(int n, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(a_mn) << 15) |
         (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(kTileM >> 4) << 24);
}

// ---------------------------------------------------------------- tile decoding
struct Operand {
  const void* tmap;
  int mn;  // 1: MN-major (column-contiguous), 0: K-major
};

struct TileCfg {
  int p, row0, col0, n_need, n_mma, half, nb_b, nk, nch, skip;
  Operand a, b;
};

__device__ __forceinline__ const void* tmap_of(const GemmArgs& g, int p, int which) {
  return static_cast<const uint8_t*>(g.tmaps) + (static_cast<size_t>(p) * kMapsPerMat + which) * 128;
}

__device__ __forceinline__ TileCfg decode_tile(const GemmArgs& g, int t) {
  const TileDesc d = g.tiles[t];
  TileCfg c;
  c.p = d.x;
  c.row0 = d.y;
  c.col0 = d.z;
  c.n_need = d.w;
  c.n_mma = (c.n_need + 31) & ~31;
  c.half = c.n_mma >> 1;
  c.nch = (c.n_need + kEpiBoxCols - 1) / kEpiBoxCols;
  const MatInfo& mi = g.mats[c.p];
  const int hi = g.cur;  // tensor maps 0/1 = hi buffers
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
  c.nb_b = c.b.mn ? (c.half + kBoxInner - 1) / kBoxInner : 2;  // B boxes per CTA
  c.skip = (g.ws.s[c.p] == 0.0f) ? 1 : 0;
  return c;
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, unsigned* status) {
  *abort_flag = 1;
  atomicOr(status, kStatusTimeout);
}

// ---------------------------------------------------------------- epilogue helpers
__device__ __forceinline__ float u2f(uint32_t v) { return __uint_as_float(v); }

// Staging blocks hold 32 rows of 32 bf16 (64 bytes each), with the 16-byte
// chunk q of row r stored at chunk q ^ ((r >> 1) & 3): a thread reading or
// writing its own row, and a warp moving eight whole rows, both touch
// distinct bank groups.
__device__ __forceinline__ uint32_t swz64(int row, int col) {
  return static_cast<uint32_t>(row * 64 + ((((col >> 3) ^ ((row >> 1) & 3))) << 4) + (col & 7) * 2);
}

__device__ __forceinline__ uint32_t chunk_off(int row, int q) {
  return static_cast<uint32_t>(row * 64 + ((q ^ ((row >> 1) & 3)) << 4));
}

// this thread's row r of a staged block, packed
__device__ __forceinline__ void read_row32(const uint8_t* blk, int r, uint4 (&out)[4]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) out[q] = *reinterpret_cast<const uint4*>(blk + chunk_off(r, q));
}

__device__ __forceinline__ void write_row32(uint8_t* blk, int r, const __nv_bfloat16* h) {
#pragma unroll
  for (int q = 0; q < 4; ++q) *reinterpret_cast<uint4*>(blk + chunk_off(r, q)) = reinterpret_cast<const uint4*>(h)[q];
}

// Coalesced read of a 32 x 32 bf16 block src[(g_row0 + rr) * ld + g_col0 + cc]
// into registers: lane l holds rows 8k + l/4, 16-byte chunk l % 4.
__device__ __forceinline__ void load_block32(const __nv_bfloat16* src, int ld, int g_row0, int g_col0, int lane,
                                             uint4 (&out)[4]) {
  const int c16 = lane & 3;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int rr = 8 * k + (lane >> 2);
    out[k] = __ldcg(reinterpret_cast<const uint4*>(src + static_cast<size_t>(g_row0 + rr) * ld + g_col0 + c16 * 8));
  }
}

__device__ __forceinline__ void put_block32(uint8_t* blk, int lane, const uint4 (&in)[4]) {
  const int c16 = lane & 3;
#pragma unroll
  for (int k = 0; k < 4; ++k) *reinterpret_cast<uint4*>(blk + chunk_off(8 * k + (lane >> 2), c16)) = in[k];
}

// Copy a staged 32 x 32 block to out[(g_row0 + rr) * ld + g_col0 + cc]: every
// warp store writes eight full 64-byte row segments.
__device__ __forceinline__ void store_block32(const uint8_t* blk, __nv_bfloat16* out, int ld, int g_row0, int g_col0,
                                              int lane) {
  const int c16 = lane & 3;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int rr = 8 * k + (lane >> 2);
    const uint4 v = *reinterpret_cast<const uint4*>(blk + chunk_off(rr, c16));
    *reinterpret_cast<uint4*>(out + static_cast<size_t>(g_row0 + rr) * ld + g_col0 + c16 * 8) = v;
  }
}

// Asynchronous (cp.async, no registers) copy of a 32 x 32 bf16 block
// src[(g_row0 + rr) * ld + g_col0 + cc] into a staging block, 16 bytes per
// lane per row segment; completion is tracked by cp.async groups.
__device__ __forceinline__ void cp_block32(uint8_t* blk, const __nv_bfloat16* src, int ld, int g_row0, int g_col0,
                                           int lane) {
  const int c16 = lane & 3;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int rr = 8 * k + (lane >> 2);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(blk + chunk_off(rr, c16))),
                 "l"(src + static_cast<size_t>(g_row0 + rr) * ld + g_col0 + c16 * 8)
                 : "memory");
  }
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

// wait until at most `pending` of this thread's most recent groups are in flight
__device__ __forceinline__ void cp_async_wait(int pending) {
  if (pending <= 0) asm volatile("cp.async.wait_group 0;" ::: "memory");
  else if (pending == 1) asm volatile("cp.async.wait_group 1;" ::: "memory");
  else asm volatile("cp.async.wait_group 2;" ::: "memory");
}

// Row i, columns [j0, j0+32) of a [rows, cols] bf16 array, zero outside.
__device__ __forceinline__ void load_row32_masked(const __nv_bfloat16* src, int ld, int rows, int cols, int i, int j0,
                                                  uint4 (&out)[4]) {
  __align__(16) __nv_bfloat16 h[32];
#pragma unroll
  for (int q = 0; q < 32; ++q)
    h[q] = (i < rows && j0 + q < cols) ? src[static_cast<size_t>(i) * ld + j0 + q] : __float2bfloat16_rn(0.0f);
#pragma unroll
  for (int q = 0; q < 4; ++q) out[q] = reinterpret_cast<const uint4*>(h)[q];
}

// element q (0..31) of a packed 32-value bf16 row segment
__device__ __forceinline__ float bf_at(const uint4 (&p)[4], int q) {
  const uint32_t w = reinterpret_cast<const uint32_t*>(&p[q >> 3])[(q & 7) >> 1];
  return __uint_as_float((q & 1) ? (w & 0xFFFF0000u) : (w << 16));
}

// ---------------------------------------------------------------- the kernel
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    ns_gemm_kernel(const __grid_constant__ GemmArgs g) {
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
  const uint32_t rank = cta_rank();
  const bool leader = (rank == 0);
  const int pair = static_cast<int>(cluster_id_x());
  const int npairs = static_cast<int>(num_clusters_x());

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 2 * kEpiWarps);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kWarpMma) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // peer barriers initialised before any remote arrive / load
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  unsigned* status = g.ws.status;

  if (warp == kWarpProducer) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    // Lanes 0..3 each issue one 16 KiB box per stage (A k-half 0, A k-half 1,
    // B box 0, B box 1): TMA throughput per SM grows with the number of
    // threads issuing, so one thread per box keeps the copies in flight
    // concurrently.  Lane 0 owns the barriers.
    const int nst = (g.phase == kPhaseUpdate) ? kStagesUpd : kStages;
    int stage = 0;
    uint32_t phase = 0;
    long fills = 0;
    for (int t = pair; t < g.ntiles; t += npairs) {
      if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;
      const TileCfg c = decode_tile(g, t);
      if (c.skip) continue;
      const uint32_t bytes = static_cast<uint32_t>(2 * (2 + c.nb_b) * kBoxBytes);
      const int arow = c.row0 + static_cast<int>(rank) * kHalfM;
      const int brow = c.col0 + static_cast<int>(rank) * c.half;
      bool ok = true;
      for (int kb = 0; kb < c.nk; ++kb) {
        int ready = 0;
        if (lane == 0) {
          ready = wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag) ? 1 : 0;
          if (!ready) raise_abort(abort_flag, status);
          else if (leader) mbar_arrive_expect_tx(full_bar(stage), bytes);
        }
        ready = __shfl_sync(0xffffffffu, ready, 0);
        if (!ready) {
          ok = false;
          break;
        }
        const uint32_t fb = map_to_rank(full_bar(stage), 0);
        const uint32_t sa = sbase + SmemLayout::kA + stage * kStageABytes;
        const uint32_t sb = sbase + SmemLayout::kB + stage * kStageBBytes;
        const int k0 = kb * kBK;
        if (lane < 2) {
          const int h = lane;
          if (c.a.mn) tma_load_pair(sa + h * kBoxBytes, c.a.tmap, arow + h * kBoxInner, k0, fb);
          else        tma_load_pair(sa + h * kBoxBytes, c.a.tmap, k0 + h * kBoxInner, arow, fb);
        } else if (lane < 2 + c.nb_b) {
          const int h = lane - 2;
          if (c.b.mn) tma_load_pair(sb + h * kBoxBytes, c.b.tmap, brow + h * kBoxInner, k0, fb);
          else        tma_load_pair(sb + h * kBoxBytes, c.b.tmap, k0 + h * kBoxInner, brow, fb);
        }
        ++fills;
        if (++stage == nst) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
    }
    // Drain (leader): both CTAs' loads complete on the leader's barriers,
    // so every stage's most recent fill must have landed before exit.
    if (leader && lane == 0) {
      for (int s = 0; s < nst; ++s) {
        const long cnt = fills / nst + ((s < fills % nst) ? 1 : 0);
        if (cnt > 0 && !wait_bounded(full_bar(s), static_cast<uint32_t>((cnt - 1) & 1), nullptr))
          atomicOr(status, kStatusTimeout);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer (leader CTA)
    if (leader && lane == 0) {
      const int nst = (g.phase == kPhaseUpdate) ? kStagesUpd : kStages;
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool issued = false;
      for (int t = pair; t < g.ntiles && !*abort_flag; t += npairs) {
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
        // descriptor start-address fields advance by (byte offset >> 4); shared
        // addresses stay below 256 KiB, so the 14-bit field never carries
        const uint64_t a_desc0 = smem_desc(sbase + SmemLayout::kA, a_lbo, 1024u);
        const uint64_t b_desc0 = smem_desc(sbase + SmemLayout::kB, b_lbo, 1024u);
        // byte offset of MMA k-step kk (16 deep) inside a stage: MN-major moves
        // down 16 rows of 128 B; K-major moves 32 B inside a box, then to box 1
        auto koff = [](int mn, int kk) -> uint64_t {
          return mn ? static_cast<uint64_t>(kk * 2048) >> 4
                    : static_cast<uint64_t>((kk >> 2) * kBoxBytes + (kk & 3) * 32) >> 4;
        };
        bool ok = true;
        for (int kb = 0; kb < c.nk; ++kb) {
          if (!wait_bounded(full_bar(stage), phase, abort_flag)) {
            raise_abort(abort_flag, status);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = a_desc0 + static_cast<uint64_t>((stage * kStageABytes) >> 4);
          const uint64_t bd = b_desc0 + static_cast<uint64_t>((stage * kStageBBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk)
            tc_mma_pair(d_tmem, ad + koff(c.a.mn, kk), bd + koff(c.b.mn, kk), idesc, (kb | kk) != 0 ? 1u : 0u);
          issued = true;
          // free the stage in both CTAs once these MMAs have read it
          tc_commit(empty_bar(stage));
          tc_commit(map_to_rank(empty_bar(stage), 1));
          if (++stage == nst) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(tfull_bar(acc));  // accumulator complete, both halves
        tc_commit(map_to_rank(tfull_bar(acc), 1));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (issued) {
        tc_commit(drain_bar);
        if (!wait_bounded(drain_bar, 0u, nullptr)) atomicOr(status, kStatusTimeout);
      }
    }
  } else if (warp >= kWarpEpi0) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int ew = warp - kWarpEpi0;          // 0..kEpiWarps-1
    const int quad = warp & 3;                // TMEM lane quadrant this warp may access
    const int grp = ew >> 2;                  // chunk group: 32-column chunks grp, grp + 2, ...
    // warp-private staging: two 32 x 32 bf16 blocks (64-byte rows, swizzled)
    uint8_t* blk0 = smem + SmemLayout::kEpi + ew * kEpiWarpBytes;
    uint8_t* blk1 = blk0 + kEpiBlockBytes;
    int acc = 0;
    uint32_t acc_phase = 0;
    const float a_c = g.sc.a, b_c = g.sc.b, c_c = g.sc.c;
    const uint32_t tempty_leader0 = map_to_rank(tempty_bar(0), 0);
    const uint32_t tempty_leader1 = map_to_rank(tempty_bar(1), 0);
    for (int t = pair; t < g.ntiles; t += npairs) {
      if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;  // warp-uniform exit
      const TileCfg c = decode_tile(g, t);
      const MatInfo& mi = g.mats[c.p];
      const int final_tile = (g.phase == kPhaseUpdate && g.final_mode != kFinalNone);
      if (c.skip && !final_tile) continue;
      const int i_lo = c.row0 + static_cast<int>(rank) * kHalfM + quad * 32;  // first row of this warp
      const int i = i_lo + lane;
      float rms = 0.0f;
      if (c.skip) {
        // Y == 0: O = 0, so the step is pure weight decay (or a zero output).
        // Rows go to warps and columns to lanes so the stores coalesce.
        const MatPtrs pt = g.ptrs[c.p];
        const int rbase = c.row0 + static_cast<int>(rank) * kHalfM;
        for (int rr = ew; rr < kHalfM; rr += kEpiWarps) {
          const int r = rbase + rr;
          if (r >= mi.rows) break;
          float* wrow = pt.W + static_cast<size_t>(r) * mi.cols;
          for (int j = c.col0 + lane; j < c.col0 + c.n_need; j += 32) {
            if (g.final_mode == kFinalWeight) wrow[j] = wrow[j] - g.sc.lr * (g.sc.wd * wrow[j]);
            else wrow[j] = 0.0f;
          }
        }
      } else {
        const bool upd = (g.phase == kPhaseUpdate);
        const bool sym = !upd;
        // inputs the epilogue reads: A (polynomial) or the hi/lo iterate (X update)
        const __nv_bfloat16* in0 = upd ? g.ws.hi[g.cur] + mi.off_x : g.ws.A + mi.off_a;
        const __nv_bfloat16* in1 = g.ws.lo + mi.off_x;
        const int ld_in = upd ? mi.ld : mi.lda;
        const int rows_in = upd ? mi.rows : mi.m, cols_in = upd ? mi.cols : mi.m;
        const int nin = (g.phase == kPhaseGram) ? 0 : (upd ? 2 : 1);
        // a chunk needs work unless it is a block strictly above the diagonal
        // of a symmetric output (its mirror writes it)
        auto needed = [&](int ch) { return !(sym && (c.col0 + ch * kEpiBoxCols > i_lo + 31)); };
        auto block_inside = [&](int ch) {
          return i_lo + 31 < rows_in && c.col0 + ch * kEpiBoxCols + 32 <= cols_in;
        };
        // coalesced prefetch of one chunk's input blocks into registers
        uint4 pf0[4], pf1[4];
        auto prefetch = [&](int ch) {
          if (nin == 0 || !needed(ch) || !block_inside(ch)) return;
          const int j0 = c.col0 + ch * kEpiBoxCols;
          load_block32(in0, ld_in, i_lo, j0, lane, pf0);
          if (nin == 2) load_block32(in1, ld_in, i_lo, j0, lane, pf1);
        };
        // X update: a per-warp ring of kUpdBufs buffers (hi, lo) fed by cp.async,
        // up to three chunks ahead; the polynomial prefetches into registers
        auto upd_buf = [&](int b) -> uint8_t* {
          const int id = ew * kUpdBufs + b;
          return smem + (id < 8 ? SmemLayout::kUpdLo + id * kUpdBufBytes : SmemLayout::kUpdHi + (id - 8) * kUpdBufBytes);
        };
        int kc = 0;  // chunks of this warp in this tile
        for (int x = grp; x < c.nch; x += kEpiGroups) ++kc;
        int issued = 0;
        auto stage_chunk = [&](int k) {
          const int chh = grp + k * kEpiGroups;
          if (block_inside(chh)) {
            uint8_t* b = upd_buf(k % kUpdBufs);
            cp_block32(b, in0, ld_in, i_lo, c.col0 + chh * kEpiBoxCols, lane);
            cp_block32(b + kEpiBlockBytes, in1, ld_in, i_lo, c.col0 + chh * kEpiBoxCols, lane);
          }
          cp_async_commit();  // one group per chunk, empty for ragged chunks
        };
        int ch = grp;
        if (upd) {
          for (; issued < kc && issued < kUpdBufs; ++issued) stage_chunk(issued);
        } else {
          prefetch(ch);
        }
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
        for (int k = 0; ch < c.nch; ch += kEpiGroups, ++k) {
          const int j0 = c.col0 + ch * kEpiBoxCols;
          if (!needed(ch)) continue;
          const bool inside = block_inside(ch);
          uint32_t v[32];
          __syncwarp();
          tmem_ld32(t_row + static_cast<uint32_t>(ch * kEpiBoxCols), v);  // completes at tmem_ld_wait
          // land this chunk's prefetched inputs in the warp's staging blocks,
          // then start fetching the next chunk
          uint4 xa[4], xb[4];  // this thread's row, packed bf16
          uint8_t* ub = upd ? upd_buf(k % kUpdBufs) : nullptr;
          if (upd) {
            if (inside) {
              cp_async_wait(issued - k - 1);
              __syncwarp();
              read_row32(ub, lane, xa);
              read_row32(ub + kEpiBlockBytes, lane, xb);
            } else {
              load_row32_masked(in0, ld_in, rows_in, cols_in, i, j0, xa);
              load_row32_masked(in1, ld_in, rows_in, cols_in, i, j0, xb);
            }
          } else if (nin > 0) {
            if (inside) {
              put_block32(blk0, lane, pf0);
              if (nin == 2) put_block32(blk1, lane, pf1);
              __syncwarp();
              read_row32(blk0, lane, xa);
              if (nin == 2) read_row32(blk1, lane, xb);
              __syncwarp();
            } else {
              load_row32_masked(in0, ld_in, rows_in, cols_in, i, j0, xa);
              if (nin == 2) load_row32_masked(in1, ld_in, rows_in, cols_in, i, j0, xb);
            }
          }
          if (!upd && ch + kEpiGroups < c.nch) prefetch(ch + kEpiGroups);
          tmem_ld_wait();
          float val[32];
          if (g.phase == kPhaseGram) {
            const bool first = (g.iter == 0);
#pragma unroll
            for (int q = 0; q < 32; ++q) val[q] = first ? (u2f(v[q]) * s) * s : u2f(v[q]);
          } else if (g.phase == kPhasePoly) {
#pragma unroll
            for (int q = 0; q < 32; ++q) val[q] = fmaf(c_c, u2f(v[q]), b_c * bf_at(xa, q));
          } else {
            const float alpha = (g.iter == 0) ? s : 1.0f;
#pragma unroll
            for (int q = 0; q < 32; ++q) val[q] = alpha * fmaf(a_c, bf_at(xa, q) + bf_at(xb, q), u2f(v[q]));
          }
          if (sym) {
            __nv_bfloat16* out = (g.phase == kPhaseGram ? g.ws.A : g.ws.B) + mi.off_a;
            __align__(16) __nv_bfloat16 h[32];
#pragma unroll
            for (int q = 0; q < 32; ++q) h[q] = __float2bfloat16_rn(val[q]);
            if (inside && j0 + 31 < i_lo) {
              // strictly lower block: stage it and its transpose, store both
              // as 64-byte row segments
              write_row32(blk0, lane, h);
#pragma unroll
              for (int q = 0; q < 32; ++q) *reinterpret_cast<__nv_bfloat16*>(blk1 + swz64(q, lane)) = h[q];
              __syncwarp();
              store_block32(blk0, out, mi.lda, i_lo, j0, lane);
              store_block32(blk1, out, mi.lda, j0, i_lo, lane);
            } else {
              // diagonal or ragged block: element-wise with masks
              __nv_bfloat16* row = out + static_cast<size_t>(i) * mi.lda;
#pragma unroll
              for (int q = 0; q < 32; ++q) {
                const int j = j0 + q;
                if (i < mi.m && j < mi.m) {
                  if (j <= i) row[j] = h[q];
                  if (j < i) out[static_cast<size_t>(j) * mi.lda + i] = h[q];
                }
              }
            }
          } else if (g.final_mode == kFinalNone) {
            __align__(16) __nv_bfloat16 h[32];
            __align__(16) __nv_bfloat16 l[32];
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              h[q] = __float2bfloat16_rn(val[q]);
              l[q] = __float2bfloat16_rn(val[q] - __bfloat162float(h[q]));
            }
            __nv_bfloat16* hout = g.ws.hi[g.cur ^ 1] + mi.off_x;
            __nv_bfloat16* lout = g.ws.lo + mi.off_x;
            if (inside) {
              write_row32(ub, lane, h);
              write_row32(ub + kEpiBlockBytes, lane, l);
              __syncwarp();
              store_block32(ub, hout, mi.ld, i_lo, j0, lane);
              store_block32(ub + kEpiBlockBytes, lout, mi.ld, i_lo, j0, lane);
            } else if (i < mi.rows) {
              const size_t wi = static_cast<size_t>(i) * mi.ld + j0;
#pragma unroll
              for (int q = 0; q < 32; ++q)
                if (j0 + q < mi.cols) {
                  hout[wi + q] = h[q];
                  lout[wi + q] = l[q];
                }
            }
          } else if (i < mi.rows) {
            const MatPtrs pt = g.ptrs[c.p];
            float* wrow = pt.W + static_cast<size_t>(i) * mi.cols + j0;
            const float scale = g.sc.rms_scale * sqrtf(static_cast<float>(mi.n));
            const bool full = (j0 + 32 <= mi.cols);
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
          if (upd && issued < kc) {
            __syncwarp();  // every lane is done with this buffer before it is refilled
            stage_chunk(issued);
            ++issued;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc == 0 ? tempty_leader0 : tempty_leader1);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (final_tile) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) rms += __shfl_xor_sync(0xffffffffu, rms, o);
        if (lane == 0) {
          const int tiles_c = (mi.cols + kBN - 1) / kBN;
          const int local = (c.row0 / kTileM) * tiles_c + c.col0 / kBN;
          g.ws.rms_part[mi.rms_tile_base + local * kRmsSlotsPerTile + static_cast<int>(rank) * kEpiWarps + ew] = rms;
        }
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // nothing may land in freed shared memory
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA leaves while its peer may still touch its barriers or operands
  if (warp == kWarpMma) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
  }
}

bool configure_device() {
  static unsigned long long configured = 0;  // one bit per device ordinal
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (dev < 64 && (configured & (1ull << dev))) return true;
  if (cudaFuncSetAttribute(ns_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
    return false;
  if (dev < 64) configured |= (1ull << dev);
  return true;
}

}  // namespace

int gemm_tc_smem_bytes() { return kSmemBytes; }

// Number of 2-CTA clusters that can be resident at once (the persistent grid).
int gemm_tc_max_pairs() {
  if (!configure_device()) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, ns_gemm_kernel, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

cudaError_t launch_gemm_tc(const GemmArgs& args, int npairs, cudaStream_t st) {
  if (args.ntiles == 0) return cudaSuccess;
  if (!configure_device()) return cudaErrorInvalidDeviceFunction;
  npairs = npairs < args.ntiles ? npairs : args.ntiles;
  if (npairs < 1) npairs = 1;
  ns_gemm_kernel<<<2 * npairs, kThreads, kSmemBytes, st>>>(args);
  return cudaGetLastError();
}

}  // namespace muon
