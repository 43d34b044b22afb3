// Internal definitions shared by libmuon's kernels and host code.
//
// Data layout in HBM (all owned by the plan unless noted):
//   user W, M (fp32) and G (bf16/fp32): [R, C] row-major, the caller's buffers.
//   hi[2], lo (bf16): the Newton-Schulz iterate in the parameter's own
//       orientation [R, C] with row pitch `ld` (>= C, multiple of 8), stored as
//       a bf16 pair X = hi + lo.  hi is the tensor-core operand and is double
//       buffered (the X-update GEMM reads hi while its epilogue writes the
//       next one); lo is only touched by the epilogue of the tile that owns
//       the element and is updated in place.
//   A, B (bf16): symmetric [m, m] matrices (m = min(R, C)), pitch `lda`.
//   x32[2], a32, b32 (fp32): the same for the fp32 validation path.
// A matrix with R > C ("tall") is never transposed: its Gram matrix is
// Y^T Y, read with MN-major (column-contiguous) tensor-core operands, and its
// X update is Y B, so every buffer keeps the parameter's layout.
#pragma once

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <vector>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace muon {

// ---------------------------------------------------------------- tile shapes
// A tensor-core tile is 256 x 256 outputs computed by a pair of CTAs (a
// 2-CTA cluster on two SMs): each CTA stages 128 rows of the A operand and
// half of the B operand's N rows, and holds its 128 output rows in TMEM.
constexpr int kTileM = 256;     // output rows per tile (two CTAs x 128 TMEM lanes)
constexpr int kHalfM = 128;     // output rows per CTA
constexpr int kBN = 256;        // output columns per tile = max UMMA N
constexpr int kBK = 64;         // K per pipeline stage (one 128-byte swizzle atom of bf16)
constexpr int kUmmaK = 16;      // K of one tcgen05.mma kind::f16
constexpr int kBoxInner = 64;   // operand boxes: 64 contiguous bf16 (128 bytes) x 128 or 64 rows
constexpr int kEpiWarps = 8;    // epilogue warps per CTA (two per TMEM lane quadrant)
constexpr int kTmemCols = 512;  // two 256-column fp32 accumulators per CTA

constexpr int kChunkElems = 32768;  // elements per momentum/normalise chunk
constexpr int kEwThreads = 256;
constexpr int kT32 = 64;           // fp32 path tile edge
// TMA descriptors per matrix (128 bytes each):
//   kMapHi0..kMapB        operand boxes of 64 x 128 rows, 128-byte swizzle (K-major loads)
//   kMapHi0S..kMapBS      operand boxes of 64 x 64 rows, 128-byte swizzle (MN-major loads,
//                         and K-major loads of at most 64 rows)
//   kMapStHiLo0/1         epilogue store of a 32 x 32 block of hi[0/1] and the same block of
//                         lo in one 3-D box {32, 32, 2} (the third dimension steps from hi to
//                         lo), 64-byte swizzle
//   kMapStA, kMapStB      epilogue store boxes of 32 x 32, 64-byte swizzle
//   kMapStPart            split-K partial products (fp32): a 32 x 32 box of one
//                         part, 3-D {cols, rows, part}, 128-byte swizzle
enum MapIndex : int {
  kMapHi0 = 0, kMapHi1 = 1, kMapA = 2, kMapB = 3,
  kMapHi0S = 4, kMapHi1S = 5, kMapAS = 6, kMapBS = 7,
  kMapStHiLo0 = 8, kMapStHiLo1 = 9, kMapStA = 10, kMapStB = 11,
  kMapStPart = 12,
  kMapsPerMat = 13
};
constexpr int kMaxSplit = 4;  // split-K parts of a symmetric product
constexpr int kEpiBoxCols = 32;

// device status bits (sticky, cleared by muon_get_status)
constexpr uint32_t kStatusTimeout = 1u;
constexpr uint32_t kStatusNonFinite = 2u;

// bounded device waits: give up after this many nanoseconds of %globaltimer
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

enum Phase : int { kPhaseGram = 0, kPhasePoly = 1, kPhaseUpdate = 2 };
// what the update pass writes: the weight update (muon_step) or O itself (muon_orthogonalize)
enum FinalMode : int { kFinalWeight = 1, kFinalOut = 2 };
enum K1Mode : int { kK1Momentum = 0, kK1Copy = 1 };
// scaling of the update O (Sec. 3.1): Eq. 4, Eq. 5, Eq. 6
enum ScaleMode : int { kScaleMaxDim = 0, kScaleHidden = 1, kScaleUpdateNorm = 2 };

// Per-matrix description, built once by muon_init.
struct MatInfo {
  int32_t rows, cols;   // parameter shape [R, C]
  int32_t m, n;         // min(R, C), max(R, C)
  int32_t tall;         // R > C
  int32_t ld;           // pitch of [R, C] workspace arrays (elements)
  int32_t lda;          // pitch of [m, m] workspace arrays (elements)
  int32_t chunk_base;   // first chunk of this matrix in the chunk list
  int32_t nchunks;
  int32_t pad_;
  int64_t off_x;        // element offset of this matrix in hi/lo/x32
  int64_t off_a;        // element offset in A/B/a32/b32
};

// Per-call pointers of one matrix.
struct MatPtrs {
  float* W;             // muon_step: weights; muon_orthogonalize: O_out
  const void* G;        // gradient or X_in
  float* M;             // momentum (step only)
  int32_t g_dtype;      // 0 bf16, 1 fp32
  int32_t vec_ok;       // all three pointers 16-byte aligned and C % 8 == 0
};

// Host: a byte range [lo, hi) of a caller buffer, for the aliasing checks
struct ByteRange {
  uintptr_t lo, hi;
};

// Host: true if any two ranges of v intersect (sorts v)
inline bool any_overlap(std::vector<ByteRange>& v) {
  std::sort(v.begin(), v.end(), [](const ByteRange& a, const ByteRange& b) { return a.lo < b.lo; });
  for (size_t i = 1; i < v.size(); ++i)
    if (v[i].lo < v[i - 1].hi) return true;
  return false;
}

// Tile of the fp32 path's GEMM phases: .x matrix, .y row0, .z col0, .w unused.
using TileDesc = int4;

// Tile of the tensor-core path: a pair of CTAs computes rows [r0, r0 + 128)
// (CTA 0) and [r1, r1 + 128) (CTA 1) of the product against N <= 256 output
// columns; CTA k stages the B operand rows [ck, ck + N/2), and accumulator
// column c holds output column c0 + c (c < N/2) or c1 + c - N/2.  Rows and
// columns need not be contiguous: a symmetric product is tiled in 128-row
// blocks (see for_each_sym_tile).
struct TcTile {
  int32_t p;       // matrix
  int32_t n_need;  // accumulator columns that hold output (1..256)
  int32_t flags;   // kTileGhost1, kTileDiagOnly
  int32_t kpart;   // split-K part of the K range (0 unless the launch splits K)
  int32_t r0, r1;  // first output row of CTA 0 / CTA 1
  int32_t c0, c1;  // first B-operand row (output column) staged by CTA 0 / CTA 1
};
constexpr int32_t kTileGhost1 = 1;    // CTA 1 duplicates CTA 0's rows and writes nothing
constexpr int32_t kTileDiagOnly = 2;  // only the diagonal 128-blocks of the tile are outputs

// How a 32 x 32 block of a symmetric product, rows [i0, i0 + 32) and columns
// [j0, j0 + 32) (both multiples of 32), computed by CTA `rank` of a tile with
// `flags`, is written:
//   0 not at all (a duplicate, or the upper part of a diagonal 128-block);
//   1 with its mirror (a block strictly below the diagonal);
//   2 element-wise, (i, j) for j <= i and (j, i) for j < i (on the diagonal).
// No tile writes a block above the diagonal of its own: the tiling covers
// each pair of 128-blocks through the lower one.
__host__ __device__ __forceinline__ int sym_block_mode(int flags, int rank, int i0, int j0) {
  if (rank == 1 && (flags & kTileGhost1)) return 0;
  const int ib = i0 >> 7, jb = j0 >> 7;
  if (ib != jb) return (ib > jb && !(flags & kTileDiagOnly)) ? 1 : 0;
  if (j0 > i0) return 0;
  return j0 == i0 ? 2 : 1;
}

// Columns of a tile's accumulator: a multiple of 32 covering n_need.
__host__ __device__ __forceinline__ int tile_n_mma(int n_need) { return (n_need + 31) & ~31; }

// Tiles of a symmetric m x m product (X X^T, A A) over 128-row blocks
// 0 .. nb - 1, nb = ceil(m / 128); every element (i, j), j <= i, is written by
// exactly one tile (sym_block_mode).  With P = floor(nb / 2) pairs of blocks:
//   - rows {2i, 2i+1} x columns {2j, 2j+1}, j < i: four blocks below the diagonal;
//   - nb even: rows {2i, 2i+1} x columns {2i, 2i+1}: two diagonal blocks and
//     (2i+1, 2i); the block above the diagonal is skipped;
//   - nb odd, last block L = nb - 1: rows {2i+1, L} x columns {2i, 2i+1}: the
//     diagonal block 2i+1, (2i+1, 2i) and the two blocks of row L; then the
//     remaining diagonal blocks 0, 2, .., 2P-2, L two per tile (rows {a, b} x
//     columns {a, b}, diagonal blocks only), the last one alone if their count
//     is odd.
// For m = 1408 (11 blocks) that is 10 + 5 + 3 = 18 tiles of 256 columns,
// against 21 for square 256-blocks with the ragged block transposed.
template <class F>
inline void for_each_sym_tile(int m, F&& emit) {
  const int nb = (m + 127) / 128, P = nb / 2;
  const bool odd = (nb & 1) != 0;
  const int L = nb - 1;
  auto contiguous = [&](int r0, int r1, int c0, int flags) {
    const int need = m - c0 < 256 ? m - c0 : 256;
    const int half = tile_n_mma(need) / 2;
    emit(TcTile{0, need, flags, 0, r0, r1, c0, c0 + half});
  };
  for (int i = 0; i < P; ++i) {
    for (int j = 0; j < i; ++j) contiguous(256 * i, 256 * i + 128, 256 * j, 0);
    if (odd) emit(TcTile{0, 256, 0, 0, 256 * i + 128, 128 * L, 256 * i, 256 * i + 128});
    else contiguous(256 * i, 256 * i + 128, 256 * i, 0);
  }
  if (odd) {
    std::vector<int> d;
    for (int i = 0; i < P; ++i) d.push_back(2 * i);
    d.push_back(L);
    size_t k = 0;
    for (; k + 1 < d.size(); k += 2)
      emit(TcTile{0, 256, kTileDiagOnly, 0, 128 * d[k], 128 * d[k + 1], 128 * d[k], 128 * d[k + 1]});
    if (k < d.size()) contiguous(128 * d[k], 128 * d[k], 128 * d[k], kTileGhost1 | kTileDiagOnly);
  }
}

// A tile split along N into its first `half` columns (from c0) and the rest
// (from c1), each a tile of its own with the same rows and flags, `levels`
// times over.  The epilogue writes whole 32-column blocks, so only tiles
// whose half is a multiple of 32 columns are split (a ragged edge tile may
// stay whole), and tiles of 64 columns or fewer stay whole.  sym_block_mode
// decides the writes from the output block alone, so the pieces write the
// elements the whole tile wrote.  A piece is clipped to the product's
// `ncols` columns, and a piece with none is dropped (the second block of a
// diagonal pair may be the ragged last one).  Used for plans with too few
// tiles to give every CTA pair one.
template <class F>
inline void split_n(const TcTile& t, int levels, int ncols, F&& emit) {
  const int half = tile_n_mma(t.n_need) / 2;
  if (levels <= 0 || t.n_need <= 64 || half % 32 != 0) {
    emit(t);
    return;
  }
  int need_a = t.n_need < half ? t.n_need : half;
  if (need_a > ncols - t.c0) need_a = ncols - t.c0;
  if (need_a > 0)
    split_n(TcTile{t.p, need_a, t.flags, t.kpart, t.r0, t.r1, t.c0, t.c0 + tile_n_mma(need_a) / 2}, levels - 1,
            ncols, emit);
  int need_b = t.n_need - half;
  if (need_b > ncols - t.c1) need_b = ncols - t.c1;
  if (need_b > 0)
    split_n(TcTile{t.p, need_b, t.flags, t.kpart, t.r0, t.r1, t.c1, t.c1 + tile_n_mma(need_b) / 2}, levels - 1,
            ncols, emit);
}

// Tiles of a full [R, C] product (the X update): rows [r0, r0 + 256) on the
// pair, columns [c0, c0 + 256) contiguous.
template <class F>
inline void for_each_full_tile(int R, int C, F&& emit) {
  for (int r0 = 0; r0 < R; r0 += 256)
    for (int c0 = 0; c0 < C; c0 += 256) {
      const int need = C - c0 < 256 ? C - c0 : 256;
      emit(TcTile{0, need, 0, 0, r0, r0 + 128, c0, c0 + tile_n_mma(need) / 2});
    }
}

// Momentum/normalise chunk: .x matrix, .y first row, .z number of rows, .w slot
using ChunkDesc = int4;

struct Workspace {
  __nv_bfloat16* hi[2];
  __nv_bfloat16* lo;
  __nv_bfloat16* A;
  __nv_bfloat16* B;
  float* x32[2];
  float* a32;
  float* b32;
  float* s;             // per matrix: 1/||Y||_F, or 0 for a zero matrix
  double* norm_part;    // per chunk: sum of y^2
  unsigned* norm_count; // per matrix arrival counter (self-resetting)
  float* rms_part;      // per tile-warp / chunk: sum of O^2
  unsigned* status;
  float* unorm;         // per matrix: rms_scale / RMS(O) of the Eq. 6 update norm
  float* part;          // split-K partial products, part k at part + k * part_stride, A's layout
  int64_t part_stride;  // elements between parts
};

struct StepScalars {
  float lr, wd, mu, a, b, c, rms_scale;
  int nesterov;
  int scale_mode;       // ScaleMode
  float const_scale;    // rms_scale * sqrt(H) for kScaleHidden
};

// Factor of O in the weight update of matrix `n` = max(rows, cols) for
// kScaleMaxDim and kScaleHidden (kScaleUpdateNorm takes its per-matrix factor
// from Workspace::unorm).
__host__ __device__ __forceinline__ float update_scale_of(const StepScalars& sc, int n) {
  return sc.scale_mode == kScaleHidden ? sc.const_scale : sc.rms_scale * sqrtf(static_cast<float>(n));
}

// Arguments of the tensor-core GEMM kernel (one launch = one phase of one
// Newton-Schulz iteration over every matrix of the plan).
struct GemmArgs {
  const TcTile* tiles;
  int ntiles;
  int phase;            // Phase
  int iter;             // 0-based iteration index (iteration 0 folds in 1/||Y||_F)
  int cur;              // which hi buffer holds the current iterate (the X update writes the other)
  const MatInfo* mats;
  const MatPtrs* ptrs;
  const void* tmaps;    // CUtensorMap[kMapsPerMat * nmat], see MapIndex
  Workspace ws;
  StepScalars sc;
  unsigned long long test_wait_ns;  // 0; > 0 only for the failure-detection test (see muon_inject_wait_timeout)
  int split;            // > 1: this symmetric launch computes K in `split` parts into ws.part
};

// Arguments of the fp32 SIMT GEMM kernel.
struct Gemm32Args {
  const TileDesc* tiles;
  int ntiles;
  int phase, iter, cur;
  const MatInfo* mats;
  const MatPtrs* ptrs;
  Workspace ws;
  StepScalars sc;
};

// ---------------------------------------------------------------- launchers (host)
cudaError_t launch_k1(const ChunkDesc* chunks, int nchunks, const MatInfo* mats, const MatPtrs* ptrs,
                      Workspace ws, StepScalars sc, int mode, int fp32_path, cudaStream_t st);
// Weight update (or O output) from the iterate in hi[xbuf]/lo (x32[xbuf] on the
// fp32 path); O = s * X when mul_s (ns_steps = 0), else O = X.  Per-chunk
// sums of O^2 go to rms_part.
cudaError_t launch_apply_update(const ChunkDesc* chunks, int nchunks, const MatInfo* mats, const MatPtrs* ptrs,
                                Workspace ws, StepScalars sc, int final_mode, int fp32_path, int xbuf, int mul_s,
                                cudaStream_t st);
// Eq. 6: per matrix RMS(O) of the same iterate, unorm = rms_scale / RMS(O)
// (0 when O = 0), and RMS(O) into update_rms when it is not null.
cudaError_t launch_update_norm(const ChunkDesc* chunks, int nchunks, const MatInfo* mats, Workspace ws,
                               StepScalars sc, int fp32_path, int xbuf, int mul_s, float* update_rms,
                               cudaStream_t st);
// sqrt(mean(O^2)) per matrix from the per-chunk partial sums of the update pass
cudaError_t launch_rms_finalize(const MatInfo* mats, int nmat, const float* part, float* out, cudaStream_t st);
cudaError_t launch_gemm_tc(const GemmArgs& args, int npairs, cudaStream_t st);
// Encode the kMapsPerMat TMA descriptors of one matrix (host); false if the
// driver entry point is missing or rejects a descriptor.
bool encode_matrix_maps(void* maps, const MatInfo& mi, __nv_bfloat16* hi0, __nv_bfloat16* hi1, __nv_bfloat16* lo,
                        __nv_bfloat16* A, __nv_bfloat16* B, float* part = nullptr, int64_t part_stride = 0,
                        int nparts = 0);
// Sum the split-K parts of a symmetric product in part order, apply the
// phase's epilogue arithmetic (Gram: scale; polynomial: b A + c (.) + a I),
// round to bf16 and write the lower triangle and its mirror into A or B.
// blocks: (matrix, i0, j0, 0) for every 32 x 32 block with i0 >= j0.
cudaError_t launch_split_reduce(const int4* blocks, int nblocks, const MatInfo* mats, Workspace ws, StepScalars sc,
                                int phase, int iter, int split, cudaStream_t st);
int gemm_tc_max_pairs();
cudaError_t launch_gemm_f32(const Gemm32Args& args, cudaStream_t st);
int gemm_tc_smem_bytes();

// Programmatic dependent launch.  The step's kernels run back to back on one
// stream and each reads what the previous one wrote.  Launched with
// programmatic stream serialization, a kernel's CTAs may start (and run their
// set-up: barriers, TMEM allocation) while the previous kernel's last CTAs
// still run; every such kernel executes pdl_wait() before its first global
// memory access, which returns once the previous grid has completed and its
// writes are visible, and then pdl_trigger(), which lets the next kernel's
// CTAs be scheduled as SMs free up.  Both are no-ops for a kernel launched
// without the attribute.  The kernels are in two classes (the tensor-core
// products and the elementwise passes); MUON_PDL in the environment, read
// once per process, is a mask of the classes launched with the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
enum PdlClass : unsigned { kPdlGemm = 1u, kPdlElementwise = 2u };
bool pdl_enabled(unsigned cls);

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(unsigned cls, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled(cls) ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

}  // namespace muon
