// Newton-Schulz products on the 5th-generation tensor cores (sm_100a).
//
// One launch computes one phase of one quintic iteration ("Muon is Scalable
// for LLM Training", Sec. 2.1, Eq. 2, factored as A = X X^T, B = b A + c A^2,
// X' = a X + B X) for every matrix of the plan:
//   kPhaseGram   A  = scale * X X^T         (wide)   or Y^T Y (tall)  [m, m]
//   kPhasePoly   B' = b A + c A A + a I      (A symmetric, so A A = A A^T)
//   kPhaseUpdate X' = alpha (B' hi + a lo)   (wide)   or Y' = alpha (hi B' + a lo) (tall)
// with X = hi + lo the bf16 pair of the iterate, so that X' = alpha (a X + B hi):
// the a X term of Eq. 2 rides on the product, and the epilogue adds only the
// a lo part.  scale = s^2 and alpha = s on iteration 0 (s = 1/||Y||_F folds
// the normalisation X_0 = Y/||Y||_F into the first products), 1 afterwards.
// The weight update of Eq. 4 is a separate elementwise pass over the last
// iterate.
//
// Structure: persistent 2-CTA clusters (one CTA per SM).  A pair owns a
// 256 x 256 output tile; tcgen05.mma.cta_group::2 (M = 256, N <= 256, K = 16,
// bf16 operands, fp32 accumulators in TMEM) reads 128 A rows and N/2 B rows
// from each CTA's shared memory, so each SM streams 32 KiB per 64-deep K
// stage for 8.4 MFLOP of the pair.  The operand stream is latency bound (a
// stage takes about two stage-times of MMA to arrive), so the ring is as deep
// as shared memory allows: 6 stages for the Gram and polynomial phases, 5 for
// the X update, whose epilogue also stages its lo inputs.  Per CTA:
//   warps 0, 10 TMA producers taking alternate stage fills: up to four lanes
//               issue one box each per stage in a single instruction (a
//               64 x 128 K-major box, or 64 x 64 boxes for MN-major operands
//               and narrow K-major ones); both CTAs' loads complete on the
//               leader's "full" barrier.
//   warp 1      TMEM allocator (both CTAs) and MMA issuer (leader only); two
//               256-column accumulators so the epilogue of one tile overlaps
//               the main loop of the next.
//   warps 2..9  epilogue: two warps per TMEM lane quadrant, each owning whole
//               32 x 32 blocks (tcgen05.ld of 32 columns, one row per thread)
//               and the fused arithmetic.  Results go through a warp-private
//               swizzled staging block to TMA bulk stores, so the load/store
//               units and the L1 path stay free for the inputs (the X
//               update's lo blocks via a per-warp cp.async ring).
#include "muon_internal.cuh"

#include <cuda.h>

namespace muon {
namespace {

#ifndef MUON_TC_STAGES_SYM
#define MUON_TC_STAGES_SYM 6
#endif
#ifndef MUON_TC_STAGES_UPD
#define MUON_TC_STAGES_UPD 5
#endif
constexpr int kStagesSym = MUON_TC_STAGES_SYM;  // stages of the Gram and polynomial phases
constexpr int kStagesUpd = MUON_TC_STAGES_UPD;  // stages of the X-update phase
constexpr int kStagesMax = kStagesSym > kStagesUpd ? kStagesSym : kStagesUpd;
constexpr int kOpBytes = kHalfM * kBK * 2;      // 16 KiB: one operand's share of a stage in one CTA
constexpr int kStageBytes = 2 * kOpBytes;       // A then B
constexpr int kBox128Bytes = kBoxInner * 128 * 2;  // 16 KiB
constexpr int kBox64Bytes = kBoxInner * 64 * 2;    // 8 KiB
// Epilogue: two groups of four warps (one warp per TMEM lane quadrant each);
// group g takes the 32-column chunks g, g+2, ... of every tile, so each warp
// owns whole 32 x 32 blocks.  Each warp has 4 KiB of staging: two 32 x 32 bf16
// blocks in the 64-byte-swizzled layout of a 32 x 32 TMA store box.
constexpr int kEpiGroups = 2;
constexpr int kEpiBlockBytes = 32 * 32 * 2;               // 2 KiB
constexpr int kEpiWarpBytes = 2 * kEpiBlockBytes;         // 4 KiB
constexpr int kEpiBytes = kEpiWarps * kEpiWarpBytes;      // 32 KiB
constexpr int kWarpProducer = 0, kWarpMma = 1, kWarpEpi0 = 2;
// Producer warps: warp 0 and the warps after the epilogue; fill f of the
// stage ring goes to producer f mod kProducers.
#ifndef MUON_TC_PRODUCERS
#define MUON_TC_PRODUCERS 2
#endif
constexpr int kProducers = MUON_TC_PRODUCERS;
constexpr int kWarpProducer2 = kWarpEpi0 + kEpiWarps;  // first of the extra producer warps
constexpr int kThreads = 32 * (kWarpProducer2 + kProducers - 1);

// X-update input: per warp a ring of 2 buffers, each the 32 x 32 lo block
// (2 KiB) of the iterate, filled by cp.async two chunks ahead.  The a X term
// needs no hi block: the polynomial phase writes B' = B + a I, so the
// product B' hi already holds a hi and the epilogue adds a lo.
constexpr int kUpdBufs = 2;
constexpr int kUpdBufBytes = kEpiBlockBytes;

struct SmemLayout {
  static constexpr int kStages = 0;                                   // stage s at s * kStageBytes
  static constexpr int kUpdRing = kStagesUpd * kStageBytes;           // X update only
  static constexpr int kEpi = kStagesSym * kStageBytes;               // staging blocks
  static constexpr int kBar = kEpi + kEpiBytes;
  // full[S], empty[S], tfull[2], tempty[2], drain, never (nothing arrives on it)
  static constexpr int kNumBars = 2 * kStagesMax + 6;
  static constexpr int kMisc = kBar + kNumBars * 8;  // tmem base (u32), abort (int)
  static constexpr int kBytes = kMisc + 16;
};
static_assert(SmemLayout::kUpdRing + kEpiWarps * kUpdBufs * kUpdBufBytes <= SmemLayout::kEpi,
              "X-update ring overlaps the staging blocks");
static_assert(kStagesUpd * kStageBytes <= SmemLayout::kEpi, "stages overlap the staging blocks");
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

#ifndef MUON_TC_SUSPEND_NS
#define MUON_TC_SUSPEND_NS 2000
#endif
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
#if MUON_TC_SUSPEND_NS > 0
  // the waiting thread may sleep up to this long (it wakes when the phase completes)
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "n"(MUON_TC_SUSPEND_NS)
      : "memory");
#else
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
#endif
  return ok != 0u;
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for the phase with the given parity to complete; false after
// limit_ns or as soon as another role of this CTA raised `abort`.
__device__ __noinline__ bool wait_bounded_ns(uint32_t bar, uint32_t parity, const volatile int* abort_flag,
                                             unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0u) {
      if (abort_flag != nullptr && *abort_flag) return false;
      if (global_ns() - t0 > limit_ns) return false;
    }
  }
}

// try_wait without a suspend hint (returns at once)
__device__ __forceinline__ bool mbar_try_wait_spin(uint32_t bar, uint32_t parity) {
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
__device__ __noinline__ bool wait_spin_slow(uint32_t bar, uint32_t parity, const volatile int* abort_flag) {
  const unsigned long long t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_spin(bar, parity)) return true;
    if ((it & 255u) == 0u) {
      if (abort_flag != nullptr && *abort_flag) return false;
      if (global_ns() - t0 > kWaitLimitNs) return false;
    }
  }
}
// The waits on the operand ring's critical path (the producers on a free
// stage, the MMA issuer on a full one) spin, with the same bounds: a
// sleeping waiter wakes a few hundred cycles after the phase completes, and
// these three warps decide when the next stage is issued.  Sleeping there
// measured 1-3% slower on the MoE batch and the mixed-8 model; every other
// wait sleeps (the epilogue warps are most of the CTA).
__device__ __forceinline__ bool wait_hot(uint32_t bar, uint32_t parity, const volatile int* abort_flag) {
  if (mbar_try_wait_spin(bar, parity)) return true;
  return wait_spin_slow(bar, parity, abort_flag);
}

__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, const volatile int* abort_flag) {
  return wait_bounded_ns(bar, parity, abort_flag, kWaitLimitNs);
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

// Bring a tensor map into the TMA descriptor cache ahead of its first use.
__device__ __forceinline__ void prefetch_tensormap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// TMA bulk store of a staged box: shared::cta -> global, tracked by this
// thread's bulk async-groups.
__device__ __forceinline__ void tma_store_2d(const void* tmap, uint32_t src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(tmap), "r"(x),
               "r"(y), "r"(src)
               : "memory");
}
__device__ __forceinline__ void tma_store_3d(const void* tmap, uint32_t src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(tmap), "r"(x),
               "r"(y), "r"(z), "r"(src)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// wait until every committed bulk store of this thread has finished reading shared memory
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// wait until every committed bulk store of this thread has completed
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// make this thread's generic-proxy shared-memory writes visible to the async proxy (TMA)
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Arrive on a barrier (shared::cluster address) once all prior tcgen05 ops of
// this thread have completed.
__device__ __forceinline__ void tc_commit(uint32_t bar_cluster) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_cluster)
               : "memory");
}

// The same arrive on the barrier at this shared-memory offset in both CTAs of
// the pair (one instruction).
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(static_cast<uint16_t>(3))
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
// A stage holds each operand's 64-deep K slice in 16 KiB:
//   K-major : one box, K [0, 64) for up to 128 rows, one 128-byte row per MN
//             index; SBO = 1024 B between 8-row groups, LBO unused (16 B).
//   MN-major: box h (8 KiB) holds MN [64h, 64h+64) for the 64 k, one 128-byte
//             row per k; SBO = 1024 B between 8-k groups, LBO = 8 KiB between
//             boxes.
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
// One operand's per-CTA share of a stage: `nbox` boxes of `box_bytes` each,
// loaded from `tmap`.
struct Operand {
  const void* tmap;
  int mn;         // 1: MN-major (column-contiguous), 0: K-major
  int nbox;       // 1 or 2
  int box_bytes;  // kBox128Bytes or kBox64Bytes
};

struct TileCfg {
  int p, n_need, n_mma, half, nk, nch, skip, flags;
  int kb0, kpart;      // first K stage of this tile's part, and the part (split K)
  int r0, r1, c0, c1;  // see TcTile
  Operand a, b;
  __device__ __forceinline__ int arow(uint32_t rank) const { return rank ? r1 : r0; }
  __device__ __forceinline__ int brow(uint32_t rank) const { return rank ? c1 : c0; }
  // output column of accumulator column cc
  __device__ __forceinline__ int col(int cc) const { return cc < half ? c0 + cc : c1 + (cc - half); }
};

__device__ __forceinline__ const void* tmap_of(const GemmArgs& g, int p, int which) {
  return static_cast<const uint8_t*>(g.tmaps) + (static_cast<size_t>(p) * kMapsPerMat + which) * 128;
}

// Operand over the array with 128-row map `map128` (its 64-row map is
// map128 + 4) spanning `extent` MN indices in this CTA.
__device__ __forceinline__ Operand make_operand(const GemmArgs& g, int p, int map128, int mn, int extent) {
  Operand o;
  o.mn = mn;
  if (mn) {
    o.tmap = tmap_of(g, p, map128 + 4);
    o.nbox = extent > kBoxInner ? 2 : 1;
    o.box_bytes = kBox64Bytes;
  } else {
    const bool narrow = extent <= 64;
    o.tmap = tmap_of(g, p, narrow ? map128 + 4 : map128);
    o.nbox = 1;
    o.box_bytes = narrow ? kBox64Bytes : kBox128Bytes;
  }
  return o;
}

// What a role needs to know of a tile before it can work on it: the tile
// entry, its matrix's m, n and orientation, and whether the matrix is skipped
// (Y = 0) in this call.  Loaded ahead (see HeadPipe) so that the dependent
// global loads do not stall the producer or the MMA issuer between tiles.
struct TileHead {
  TcTile d;
  int m, n, tall;
  float s;
};

__device__ __forceinline__ TileCfg make_cfg(const GemmArgs& g, const TileHead& h) {
  TileCfg c;
  c.p = h.d.p;
  c.r0 = h.d.r0;
  c.r1 = h.d.r1;
  c.c0 = h.d.c0;
  c.c1 = h.d.c1;
  c.flags = h.d.flags;
  c.n_need = h.d.n_need;
  c.n_mma = tile_n_mma(c.n_need);
  c.half = c.n_mma >> 1;
  c.nch = (c.n_need + kEpiBoxCols - 1) / kEpiBoxCols;
  const int hi = kMapHi0 + g.cur;
  int K;
  if (g.phase == kPhaseGram) {
    K = h.n;
    c.a = make_operand(g, c.p, hi, h.tall, kHalfM);
    c.b = make_operand(g, c.p, hi, h.tall, c.half);
  } else if (g.phase == kPhasePoly) {
    K = h.m;
    c.a = make_operand(g, c.p, kMapA, 0, kHalfM);
    c.b = make_operand(g, c.p, kMapA, 0, c.half);
  } else {
    K = h.m;
    if (h.tall) {
      c.a = make_operand(g, c.p, hi, 0, kHalfM);
      c.b = make_operand(g, c.p, kMapB, 0, c.half);
    } else {
      c.a = make_operand(g, c.p, kMapB, 0, kHalfM);
      c.b = make_operand(g, c.p, hi, 1, c.half);
    }
  }
  const int nk_all = (K + kBK - 1) / kBK;
  c.kpart = h.d.kpart;
  if (g.split > 1 && g.phase != kPhaseUpdate) {
    // part k of `split` takes stages [k nk / split, (k + 1) nk / split)
    c.kb0 = (c.kpart * nk_all) / g.split;
    c.nk = ((c.kpart + 1) * nk_all) / g.split - c.kb0;
  } else {
    c.kb0 = 0;
    c.nk = nk_all;
  }
  c.skip = (h.s == 0.0f) ? 1 : 0;
  return c;
}

__device__ __forceinline__ TileHead load_head(const GemmArgs& g, const TcTile& d) {
  TileHead h;
  h.d = d;
  const MatInfo* mi = g.mats + d.p;
  h.m = mi->m;
  h.n = mi->n;
  h.tall = mi->tall;
  h.s = g.ws.s[d.p];
  return h;
}

__device__ __forceinline__ TileCfg decode_tile(const GemmArgs& g, int t) { return make_cfg(g, load_head(g, g.tiles[t])); }

// Two-deep prefetch of the tiles a pair visits (t, t + npairs, ...): while a
// role works on tile t, the entry of tile t + 2 npairs and the matrix fields
// of tile t + npairs are in flight, so advancing is free of load latency.
struct HeadPipe {
  TileHead cur, nxt;
  TcTile nn;
  int t, step, ntiles;

  __device__ __forceinline__ void start(const GemmArgs& g, int t0, int stride) {
    t = t0;
    step = stride;
    ntiles = g.ntiles;
    if (t < ntiles) cur = load_head(g, g.tiles[t]);
    if (t + step < ntiles) nxt = load_head(g, g.tiles[t + step]);
    if (t + 2 * step < ntiles) nn = g.tiles[t + 2 * step];
  }
  __device__ __forceinline__ bool valid() const { return t < ntiles; }
  __device__ __forceinline__ void advance(const GemmArgs& g) {
    t += step;
    cur = nxt;
    if (t + step < ntiles) nxt = load_head(g, nn);
    if (t + 2 * step < ntiles) nn = g.tiles[t + 2 * step];
  }
};

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

// This thread's row segment src[row * ld + col0 .. + 32), 64 contiguous bytes,
// through the read-only path (the array is not written during the launch).
__device__ __forceinline__ void load_row32(const __nv_bfloat16* src, int ld, int row, int col0, uint4 (&out)[4]) {
  const uint4* p = reinterpret_cast<const uint4*>(src + static_cast<size_t>(row) * ld + col0);
#pragma unroll
  for (int q = 0; q < 4; ++q) out[q] = __ldg(p + q);
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

// element q (0..31) of a packed 32-value bf16 row segment, as a float and as its bits
__device__ __forceinline__ float bf_at(const uint4 (&p)[4], int q) {
  const uint32_t w = reinterpret_cast<const uint32_t*>(&p[q >> 3])[(q & 7) >> 1];
  return __uint_as_float((q & 1) ? (w & 0xFFFF0000u) : (w << 16));
}
__device__ __forceinline__ unsigned short bf_bits(const uint4 (&p)[4], int q) {
  const uint32_t w = reinterpret_cast<const uint32_t*>(&p[q >> 3])[(q & 7) >> 1];
  return static_cast<unsigned short>((q & 1) ? (w >> 16) : (w & 0xFFFFu));
}

// bf16 pair (x in the low half, y in the high half) as one word
__device__ __forceinline__ uint32_t pack_bf2(float x, float y) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Staged transpose of a 32 x 32 bf16 block: row q, column t of `blk` gets
// element q of lane t's row (hw holds the row as 16 packed pairs).  Each
// pair of neighbouring lanes swaps a word, so that every lane stores whole
// words: an even lane t the pair (t, t + 1) of row q = 2u, an odd lane the
// pair (t - 1, t) of row 2u + 1; one store covers two rows, all 32 banks.
__device__ __forceinline__ void stage_transpose(uint8_t* blk, int lane, const uint32_t (&hw)[16]) {
  const int odd = lane & 1;
  const uint32_t sel = odd ? 0x3276u : 0x5410u;  // odd: high halves (nb, own); even: low halves (own, nb)
  const int le = lane & ~1;
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const uint32_t nb = __shfl_xor_sync(0xffffffffu, hw[u], 1);
    *reinterpret_cast<uint32_t*>(blk + swz64(2 * u + odd, le)) = __byte_perm(hw[u], nb, sel);
  }
}

// X-update row segment: val = alpha (a lo + acc) for the 32 columns of this
// thread's row (alpha = s when kScaled, else 1), split into hi = bf16(val) and
// lo = bf16(val - hi), staged in blk_hi / blk_lo
template <bool kScaled>
__device__ __forceinline__ void upd_stage_row(const uint32_t (&v)[32], const uint4 (&xa)[4], float a_c, float s,
                                              uint8_t* blk_hi, uint8_t* blk_lo, int lane) {
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) {
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int q = 8 * q4 + 2 * u;
      const uint32_t xw = reinterpret_cast<const uint32_t*>(&xa[q4])[u];  // lo of columns q, q + 1
      float v0 = fmaf(a_c, __uint_as_float(xw << 16), __uint_as_float(v[q]));
      float v1 = fmaf(a_c, __uint_as_float(xw & 0xFFFF0000u), __uint_as_float(v[q + 1]));
      if (kScaled) {
        v0 *= s;
        v1 *= s;
      }
      const uint32_t hb = pack_bf2(v0, v1);
      hw[u] = hb;
      lw[u] = pack_bf2(v0 - __uint_as_float(hb << 16), v1 - __uint_as_float(hb & 0xFFFF0000u));
    }
    *reinterpret_cast<uint4*>(blk_hi + chunk_off(lane, q4)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4*>(blk_lo + chunk_off(lane, q4)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  }
}

// ---------------------------------------------------------------- the kernel
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    ns_gemm_kernel(const __grid_constant__ GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + SmemLayout::kBar;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStagesMax + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * kStagesMax + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * kStagesMax + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * kStagesMax + 4);
  const uint32_t never_bar = bar0 + 8u * (2 * kStagesMax + 5);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SmemLayout::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SmemLayout::kMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cta_rank();
  const bool leader = (rank == 0);
  const int pair = static_cast<int>(cluster_id_x());
  const int npairs = static_cast<int>(num_clusters_x());
  const int nst = (g.phase == kPhaseUpdate) ? kStagesUpd : kStagesSym;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesMax; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 2 * kEpiWarps);
    }
    mbar_init(drain_bar, 1);
    mbar_init(never_bar, 1);
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
  // everything above touched only shared memory, TMEM and the kernel
  // parameters: with programmatic dependent launch it overlaps the previous
  // kernel's last CTAs; nothing below runs before that kernel has completed
  pdl_wait();
  pdl_trigger();

  if (g.test_wait_ns != 0) {
    // Failure-detection test (the same value in every CTA of the grid): one
    // thread per CTA waits, with the short limit, on a barrier that nothing
    // arrives at, then raises the abort flag of both CTAs of its pair and the
    // timeout status.  This happens before any role starts, so no operand
    // load or tensor-core instruction is ever issued and every role below
    // sees the flag and returns at once.
    if (warp == kWarpEpi0 && lane == 0) {
      if (!wait_bounded_ns(never_bar, 0u, nullptr, g.test_wait_ns)) {
        const uint32_t peer_abort = map_to_rank(smem_u32(const_cast<int*>(abort_flag)), rank ^ 1u);
        *abort_flag = 1;
        asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(peer_abort), "r"(1) : "memory");
        atomicOr(status, kStatusTimeout);
      }
    }
    cluster_sync();
  }

  if (warp == kWarpProducer || warp >= kWarpProducer2) {
    // ------------------------------------------------------------ TMA producers (both CTAs)
    // The producer warps take the fills in turn, so several stage fills are
    // being issued at any time (one thread issues about one TMA instruction
    // per few hundred ns; a second warp measured about 2% faster, a third no
    // better).  Within a warp, lane l < nbox_a loads A box l and the next
    // lanes the B boxes, all in one instruction; lane 0 owns the barriers.
    const int pp = (warp == kWarpProducer) ? 0 : warp - kWarpProducer2 + 1;
    long fills = 0;  // fills of all producers, in order
    int fstage = 0;        // stage of fill `fills`
    uint32_t fphase = 0;   // its ring pass parity
    const uint32_t full0 = map_to_rank(full_bar(0), 0);  // the leader's full barriers
    HeadPipe hp;
    for (hp.start(g, pair, npairs); hp.valid(); hp.advance(g)) {
      if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;
      const TileCfg c = make_cfg(g, hp.cur);
      if (c.skip) continue;
      const uint32_t bytes =
          static_cast<uint32_t>(2 * (c.a.nbox * c.a.box_bytes + c.b.nbox * c.b.box_bytes));
      const int arow = c.arow(rank);
      const int brow = c.brow(rank);
      if (lane == 0) prefetch_tensormap(c.a.tmap);
      if (lane == 1) prefetch_tensormap(c.b.tmap);
      bool ok = true;
      for (int kb = 0; kb < c.nk; ++kb, ++fills) {
        const int stage = fstage;
        const uint32_t phase = fphase;
        if (++fstage == nst) {
          fstage = 0;
          fphase ^= 1u;
        }
        if (static_cast<int>(fills % kProducers) != pp) continue;
        int ready = 0;
        if (lane == 0) {
          ready = wait_hot(empty_bar(stage), phase ^ 1u, abort_flag) ? 1 : 0;
          if (!ready) raise_abort(abort_flag, status);
          else if (leader) mbar_arrive_expect_tx(full_bar(stage), bytes);
        }
        ready = __shfl_sync(0xffffffffu, ready, 0);
        if (!ready) {
          ok = false;
          break;
        }
        const uint32_t fb = full0 + 8u * static_cast<uint32_t>(stage);
        const uint32_t sa = sbase + SmemLayout::kStages + stage * kStageBytes;
        const uint32_t sb = sa + kOpBytes;
        const int k0 = (c.kb0 + kb) * kBK;
        const bool is_a = lane < c.a.nbox;
        const Operand& o = is_a ? c.a : c.b;
        const int h = is_a ? lane : lane - c.a.nbox;
        if (lane < c.a.nbox + c.b.nbox) {
          const int mn0 = (is_a ? arow : brow) + h * kBoxInner;
          const uint32_t dst = (is_a ? sa : sb) + h * kBox64Bytes;
          tma_load_pair(dst, o.tmap, o.mn ? mn0 : k0, o.mn ? k0 : mn0 - h * kBoxInner, fb);
        }
      }
      if (!ok) break;
    }
    // Drain (leader): both CTAs' loads complete on the leader's barriers,
    // so each of this warp's fills among the last nst (the latest of its
    // stage) must have landed before exit.
    if (leader && lane == 0) {
      for (long f = fills > nst ? fills - nst : 0; f < fills; ++f) {
        if (f % kProducers != pp) continue;
        if (!wait_bounded(full_bar(static_cast<int>(f % nst)), static_cast<uint32_t>((f / nst) & 1), nullptr))
          atomicOr(status, kStatusTimeout);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer (leader CTA)
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool issued = false;
      HeadPipe hp;
      for (hp.start(g, pair, npairs); hp.valid() && !*abort_flag; hp.advance(g)) {
        const TileCfg c = make_cfg(g, hp.cur);
        if (c.skip) continue;
        if (!wait_bounded(tempty_bar(acc), acc_phase ^ 1u, abort_flag)) {
          raise_abort(abort_flag, status);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
        const uint32_t idesc = make_idesc(c.n_mma, c.a.mn, c.b.mn);
        const uint32_t a_lbo = c.a.mn ? kBox64Bytes : 16u, b_lbo = c.b.mn ? kBox64Bytes : 16u;
        // descriptor start-address fields advance by (byte offset >> 4); shared
        // addresses stay below 256 KiB, so the 14-bit field never carries
        const uint64_t a_desc0 = smem_desc(sbase + SmemLayout::kStages, a_lbo, 1024u);
        const uint64_t b_desc0 = smem_desc(sbase + SmemLayout::kStages + kOpBytes, b_lbo, 1024u);
        // byte offset of MMA k-step kk (16 deep) inside a stage: MN-major moves
        // down 16 rows of 128 B, K-major 32 B along the swizzled row
        auto koff = [](int mn, int kk) -> uint64_t {
          return static_cast<uint64_t>(mn ? kk * 2048 : kk * 32) >> 4;
        };
        bool ok = true;
        for (int kb = 0; kb < c.nk; ++kb) {
          if (!wait_hot(full_bar(stage), phase, abort_flag)) {
            raise_abort(abort_flag, status);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t so = static_cast<uint64_t>((stage * kStageBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk)
            tc_mma_pair(d_tmem, a_desc0 + so + koff(c.a.mn, kk), b_desc0 + so + koff(c.b.mn, kk), idesc,
                        (kb | kk) != 0 ? 1u : 0u);
          issued = true;
          // free the stage in both CTAs once these MMAs have read it
          tc_commit_pair(empty_bar(stage));
          if (++stage == nst) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair(tfull_bar(acc));  // accumulator complete, both halves
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
    // warp-private staging for the TMA stores: two 32 x 32 bf16 blocks
    uint8_t* blk0 = smem + SmemLayout::kEpi + ew * kEpiWarpBytes;
    uint8_t* blk1 = blk0 + kEpiBlockBytes;
    const uint32_t blk0_s = smem_u32(blk0), blk1_s = smem_u32(blk1);
    // the staging blocks may be rewritten once this warp's earlier bulk
    // stores have read them (lane 0 issues and tracks them)
    auto staging_free = [&]() {
      if (lane == 0) bulk_wait_read();
      __syncwarp();
    };
    // stage this thread's row of both blocks, then store them (lane 0)
    auto publish = [&](const void* map0, int x0, int y0, const void* map1, int x1, int y1) {
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(map0, blk0_s, x0, y0);
        tma_store_2d(map1, blk1_s, x1, y1);
        bulk_commit();
      }
    };
    int acc = 0;
    uint32_t acc_phase = 0;
    const float a_c = g.sc.a, b_c = g.sc.b, c_c = g.sc.c;
    const uint32_t tempty_leader0 = map_to_rank(tempty_bar(0), 0);
    const uint32_t tempty_leader1 = map_to_rank(tempty_bar(1), 0);
    for (int t = pair; t < g.ntiles; t += npairs) {
      if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;  // warp-uniform exit
      const TileCfg c = decode_tile(g, t);
      const MatInfo& mi = g.mats[c.p];
      if (c.skip) continue;  // Y == 0: nothing downstream reads this matrix
      const int i_lo = c.arow(rank) + quad * 32;  // first row of this warp
      const int i = i_lo + lane;
      const bool upd = (g.phase == kPhaseUpdate);
      const bool sym = !upd;
      // input the epilogue reads: A (polynomial) or the lo part of the iterate (X update)
      const __nv_bfloat16* in0 = upd ? g.ws.lo + mi.off_x : g.ws.A + mi.off_a;
      const int ld_in = upd ? mi.ld : mi.lda;
      const int rows_in = upd ? mi.rows : mi.m, cols_in = upd ? mi.cols : mi.m;
      // split K: this tile computes one part of the K range; its raw fp32
      // accumulator goes to ws.part and a reduction pass forms the product
      const bool splitk = sym && g.split > 1;
      const bool poly = (g.phase == kPhasePoly) && !splitk;
      // how chunk ch of this warp is written: always in the X update, by
      // sym_block_mode in a symmetric product (0 = not at all)
      auto mode = [&](int ch) { return sym ? sym_block_mode(c.flags, static_cast<int>(rank), i_lo, c.col(ch * kEpiBoxCols)) : 1; };
      auto needed = [&](int ch) { return mode(ch) != 0; };
      auto block_inside = [&](int ch) {
        return i_lo + 31 < rows_in && c.col(ch * kEpiBoxCols) + 32 <= cols_in;
      };
      // polynomial: prefetch of this thread's row of the next A block into
      // registers; pf_ch is the chunk whose row pf0 holds (a tile may skip
      // chunks and need later ones, so the next needed chunk is looked up,
      // not assumed)
      uint4 pf0[4];
      int pf_ch = -1;
      auto prefetch_from = [&](int from) {
        if (!poly) return;
        for (int nx = from; nx < c.nch; nx += kEpiGroups)
          if (needed(nx) && block_inside(nx)) {
            load_row32(in0, ld_in, i, c.col(nx * kEpiBoxCols), pf0);
            pf_ch = nx;
            return;
          }
      };
      // X update: ring of kUpdBufs lo buffers fed by cp.async; chunk k of
      // this warp lives in buffer k % kUpdBufs
      auto upd_buf = [&](int b) -> uint8_t* {
        return smem + SmemLayout::kUpdRing + (ew * kUpdBufs + b) * kUpdBufBytes;
      };
      int kc = 0;  // chunks of this warp in this tile
      for (int x = grp; x < c.nch; x += kEpiGroups) ++kc;
      int issued = 0;
      auto stage_chunk = [&](int k) {
        const int chh = grp + k * kEpiGroups;
        if (block_inside(chh)) {
          cp_block32(upd_buf(k % kUpdBufs), in0, ld_in, i_lo, c.col(chh * kEpiBoxCols), lane);
        }
        cp_async_commit();  // one group per chunk, empty for ragged chunks
      };
      int ch = grp;
      if (upd) {
        for (; issued < kc && issued < kUpdBufs; ++issued) stage_chunk(issued);
      } else {
        prefetch_from(ch);
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
        const int j0 = c.col(ch * kEpiBoxCols);
        const int md = mode(ch);
        if (md == 0) continue;
        const bool inside = block_inside(ch);
        uint32_t v[32];
        __syncwarp();
        tmem_ld32(t_row + static_cast<uint32_t>(ch * kEpiBoxCols), v);  // completes at tmem_ld_wait
        uint4 xa[4];  // this thread's row of the input (A, or lo), packed bf16
        if (upd) {
          if (inside) {
            cp_async_wait(issued - k - 1);
            __syncwarp();
            read_row32(upd_buf(k % kUpdBufs), lane, xa);
            __syncwarp();
          } else {
            load_row32_masked(in0, ld_in, rows_in, cols_in, i, j0, xa);
          }
          // this buffer is free again: fetch the chunk two ahead into it
          if (issued < kc) {
            stage_chunk(issued);
            ++issued;
          }
        } else if (poly) {
          if (inside) {
            if (pf_ch != ch) load_row32(in0, ld_in, i, j0, pf0);  // fallback; prefetch_from lands here
#pragma unroll
            for (int q = 0; q < 4; ++q) xa[q] = pf0[q];
          } else {
            load_row32_masked(in0, ld_in, rows_in, cols_in, i, j0, xa);
          }
          prefetch_from(ch + kEpiGroups);
        }
        tmem_ld_wait();
        if (splitk) {
          if (inside) {
            // this thread's row (128 bytes) into the 4 KiB staging pair,
            // 16-byte chunk q at q ^ (row & 7): the 128-byte swizzle of the
            // part map's 32 x 32 fp32 box
            staging_free();
#pragma unroll
            for (int q = 0; q < 8; ++q)
              *reinterpret_cast<uint4*>(blk0 + lane * 128 + ((q ^ (lane & 7)) << 4)) =
                  make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(tmap_of(g, c.p, kMapStPart), blk0_s, j0, i_lo, c.kpart);
              bulk_commit();
            }
          } else if (i < mi.m) {
            float* prow = g.ws.part + c.kpart * g.ws.part_stride + mi.off_a + static_cast<size_t>(i) * mi.lda;
#pragma unroll
            for (int q = 0; q < 32; ++q)
              if (j0 + q < mi.m) prow[j0 + q] = u2f(v[q]);
          }
          continue;
        }
        if (upd) {
          // X' = alpha (B' hi + a lo) = alpha (a X + B hi), split into the
          // new hi and lo; written 8 columns at a time so that only a
          // quarter of the row's outputs are live at once
          const float alpha = (g.iter == 0) ? s : 1.0f;
          if (inside) {
            staging_free();
            // two columns per step: their lo inputs share a word, and each
            // rounding to bf16 converts the pair at once
            if (g.iter == 0)
              upd_stage_row<true>(v, xa, a_c, s, blk0, blk1, lane);
            else
              upd_stage_row<false>(v, xa, a_c, s, blk0, blk1, lane);
            // blk1 follows blk0: one 3-D store writes the hi block and the lo block
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(tmap_of(g, c.p, kMapStHiLo0 + (g.cur ^ 1)), blk0_s, j0, i_lo, 0);
              bulk_commit();
            }
          } else if (i < mi.rows) {
            __nv_bfloat16* hout = g.ws.hi[g.cur ^ 1] + mi.off_x;
            __nv_bfloat16* lout = g.ws.lo + mi.off_x;
            const size_t wi = static_cast<size_t>(i) * mi.ld + j0;
#pragma unroll
            for (int q = 0; q < 32; ++q)
              if (j0 + q < mi.cols) {
                const float val = alpha * fmaf(a_c, bf_at(xa, q), u2f(v[q]));
                const __nv_bfloat16 h = __float2bfloat16_rn(val);
                hout[wi + q] = h;
                lout[wi + q] = __float2bfloat16_rn(val - __bfloat162float(h));
              }
          }
          continue;
        }
        float val[32];
        if (g.phase == kPhaseGram) {
          const bool first = (g.iter == 0);
#pragma unroll
          for (int q = 0; q < 32; ++q) val[q] = first ? (u2f(v[q]) * s) * s : u2f(v[q]);
        } else {
          // B' = b A + c A A + a I (the a X term of the update rides on B' hi);
          // only a block that starts on the diagonal holds diagonal elements
#pragma unroll
          for (int q = 0; q < 32; ++q) val[q] = fmaf(c_c, u2f(v[q]), b_c * bf_at(xa, q));
          if (j0 == i_lo) {
#pragma unroll
            for (int q = 0; q < 32; ++q)
              if (q == lane) val[q] += a_c;
          }
        }
        // symmetric products
        __align__(16) uint32_t hw[16];  // this thread's row, packed pairs
#pragma unroll
        for (int u = 0; u < 16; ++u) hw[u] = pack_bf2(val[2 * u], val[2 * u + 1]);
        __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(hw);
        if (inside && md == 1) {
          // off-diagonal block: stage it and its transpose, store both
          staging_free();
          write_row32(blk0, lane, h);
          stage_transpose(blk1, lane, hw);
          const void* map = tmap_of(g, c.p, g.phase == kPhaseGram ? kMapStA : kMapStB);
          publish(map, j0, i_lo, map, i_lo, j0);
        } else if (inside) {
          // diagonal block (j0 == i_lo): the diagonal and the part below it
          // from this thread's row, the part above from the transpose, so
          // the block is stored exactly symmetric, whole, in one bulk store
          staging_free();
          stage_transpose(blk1, lane, hw);
          __syncwarp();
          uint4 tr[4];  // row `lane` of the transpose: element q is (j0 + q, i)
          read_row32(blk1, lane, tr);
#pragma unroll
          for (int q = 0; q < 32; ++q)
            if (q > lane) h[q] = __ushort_as_bfloat16(bf_bits(tr, q));
          write_row32(blk0, lane, h);
          fence_proxy_async();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(tmap_of(g, c.p, g.phase == kPhaseGram ? kMapStA : kMapStB), blk0_s, j0, i_lo);
            bulk_commit();
          }
        } else {
          // ragged block (past the edge of the product): element-wise with
          // masks; below the diagonal it is written whole, with its mirror
          const bool whole = (md == 1);
          __nv_bfloat16* out = (g.phase == kPhaseGram ? g.ws.A : g.ws.B) + mi.off_a;
          __nv_bfloat16* row = out + static_cast<size_t>(i) * mi.lda;
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            const int j = j0 + q;
            if (i < mi.m && j < mi.m) {
              if (whole || j <= i) row[j] = h[q];
              if (whole || j < i) out[static_cast<size_t>(j) * mi.lda + i] = h[q];
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc == 0 ? tempty_leader0 : tempty_leader1);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    // nothing may still read or land in shared memory once the CTA exits
    if (lane == 0) bulk_wait_all();
    __syncwarp();
    asm volatile("cp.async.wait_all;" ::: "memory");
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
  return launch_pdl(kPdlGemm, ns_gemm_kernel, dim3(2 * npairs), dim3(kThreads), kSmemBytes, st, args);
}

}  // namespace muon
