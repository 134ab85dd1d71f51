// Launch-parameter layouts shared by the host planner and the kernels.
// Everything a kernel needs travels by value in its parameter block (up to a few
// tens of KB, allowed on sm_70+ since CUDA 12.1), so a step needs no host->device
// copies and the whole launch sequence can be captured in a CUDA graph.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <atomic>
#include <cstdint>

#include "../../include/nshb.h"

namespace nshb {

// A once-per-device fact of a launcher (a kernel attribute already set, the CTAs that fit
// at once): 0 until set.  Relaxed atomics, since threads that race compute the same value
// and a lost race only repeats the query; devices past kMaxDevices are never cached.
constexpr int kMaxDevices = 64;
struct PerDevice {
  std::atomic<int> v[kMaxDevices];
  int get(int dev) const { return dev >= 0 && dev < kMaxDevices ? v[dev].load(std::memory_order_relaxed) : 0; }
  void set(int dev, int x) {
    if (dev >= 0 && dev < kMaxDevices) v[dev].store(x, std::memory_order_relaxed);
  }
};

// Matrices per launch of a streaming kernel and GEMM problems per launch (the host splits
// larger sets).  224 keeps a whole 8B-width set (224 matrices) or Qwen3-style set (196) in
// one launch per phase while every parameter block stays under the 32,764-byte limit.
constexpr int kMaxMats = 224;
constexpr int kMaxProb = 224;
constexpr int kBlk = 64;        // streaming kernels work on 64 x 64 blocks

// Matrix flags.
constexpr int kTall = 1;        // rows > cols: the fp32 chain works on U^T (the wide side); the
                                // bf16 chain keeps X = U and takes the right Gram X^T X
constexpr int kVec = 2;         // 16-byte vector access is legal for W/G/M rows
constexpr int kWF32 = 4;        // W and G are fp32 (else bf16)
constexpr int kTiled = 8;       // Hierarchical Muon: X is a grid of T x T tiles
constexpr int kNsF32 = 16;      // NS in fp32, X row-major fp32 (else bf16 panel layout)
constexpr int kTileMajor = 32;  // block list enumerates tile by tile (momentum of tiled matrices)
constexpr int kFromP = 64;      // momentum kernel: take U from an fp32 row-major matrix (no momentum)
constexpr int kURow = 128;      // momentum kernel: write U as fp32 row-major only (Newton-Muon input)
constexpr int kNoX = 256;       // momentum kernel: the NS operand is already in place (Newton-Muon:
                                // the backward solve wrote P's hi / lo panels), only the norm

// Per-matrix record of a streaming launch (momentum, reductions, apply).
struct MatDesc {
  void *W;
  const void *G;
  float *M;
  void *O_out;
  int64_t x_off;     // workspace byte offset of X0 (where U is written)
  int64_t xlo_off;   // workspace byte offset of U's bf16 low part, or -1
  int64_t u_off;     // kURow / kFromP: workspace byte offset of the fp32 row-major m x n U / P
  int64_t o_off;     // workspace byte offset of the final O
  int32_t m, n, ld;  // W shape and leading dimension
  int32_t flags;
  int32_t ph;        // bf16: panel height of X (padded rows); fp32: row stride of X; tiled: T
  int32_t pr, pc;    // block domain of this launch in W coordinates (padded extents)
  int32_t blk_begin; // first 64x64 block of this matrix in the launch's block list
  int32_t seg_begin; // first norm segment (matrix, or first tile when tiled)
  int32_t tiles_c;   // tiled: tiles per tile-row of the padded grid
  int32_t mat;       // index of the matrix in the whole call
  int32_t rec_begin; // reduce: first (||O||^2, <W,O>, ||W||^2) record of this matrix
};

// Momentum + U + ||U||^2 partials, one per warp of every block (kK1PartsPerBlock per block).
constexpr int kK1PartsPerBlock = 8;
struct MomentumParams {
  char *ws;
  double *partials;  // kK1PartsPerBlock per block of the launch
  uint32_t *status;
  float beta;
  int32_t nesterov;
  int32_t nmat, total_blocks;
  MatDesc mats[kMaxMats];
};

// Per-segment ||U||^2 -> scale 1 / (sqrt(nu) + eps).
struct NormFinParams {
  const double *partials;
  float *scales;
  double *nus;
  uint32_t *status;
  float ns_eps;
  int32_t nmat;
  int32_t seg_begin[kMaxMats + 1];  // segment prefix (segments of one matrix are contiguous)
  int32_t blk_begin[kMaxMats];      // index of each matrix's first partial record
  int32_t bps[kMaxMats];            // partial records per segment
};

// Per-matrix scalars kept in the workspace between the reduce, finalize and apply kernels.
struct MatScalars {
  double omega, delta, pi;  // ||O||^2, <W, O>, ||W||^2
  double t;                 // eta / ||O|| (Hyperball) or lr * shape scale (RadialBrake)
  float alpha, beta;        // W_new = alpha W + beta O
  int32_t need_exact;       // closed-form ||W - t O|| lost too many digits; recompute it
  int32_t pad_;
  double vv;                // exact ||W - t O||^2 when need_exact
  double pad2_;
};

// Reductions over (W, O) blocks and the streaming update W <- alpha W + beta O.
enum ApplyOp { kOpMuon = 0, kOpHyperball = 1, kOpBrake = 2, kOpNorms = 3, kOpRelative = 4 };
struct ApplyParams {
  char *ws;
  double *partials;        // reduce: 3 doubles per record (MatDesc::rec_begin + local block);
                           // exact norm: 1 double per block of the launch
  MatScalars *scal;        // indexed by MatDesc::mat
  uint32_t *status;
  int32_t op;
  int32_t nmat, total_blocks;
  MatDesc mats[kMaxMats];
};
struct ApplyFinParams {
  const double *partials;  // stage 0: 3-double records; stage 1: exact-norm block sums
  const double *xpartials;
  MatScalars *scal;
  uint32_t *status;
  const float *rho;        // device radii or NULL
  float *norms_out;        // kOpNorms: ||W|| per matrix
  int32_t op, stage;       // stage 0: after the reduce; stage 1: after the exact-norm pass
  float lr, weight_decay, eta, hb_eps, brake_out, brake_in;
  int32_t nmat;
  int32_t rec_begin[kMaxMats + 1];  // stage 0: records of matrix k (contiguous)
  int32_t blk_begin[kMaxMats + 1];  // stage 1: exact-norm blocks of matrix k
  int32_t mat[kMaxMats];
  int32_t m[kMaxMats], n[kMaxMats];
};

// AdamH first pass: Adam moments, the direction U~ (kept in the matrix's dtype where the
// apply kernels read O: bf16 panels, or fp32 row-major with kNsF32) and the
// (||U~||^2, <W, U~>, ||W||^2) partials of every block.
struct AdamParams {
  char *ws;
  double *partials;        // 3 doubles per block
  uint32_t *status;
  float beta1, beta2, eps;
  float bc1, bc2;          // 1 / (1 - beta1^t), 1 / (1 - beta2^t)
  int32_t nmat, total_blocks;
  MatDesc mats[kMaxMats];  // o_off: U~; M: first moment
  float *V[kMaxMats];      // second moments (same ld as W)
};

// One bf16 GEMM problem of a Newton-Schulz phase (possibly a batch of equal problems).
// Operands live in the workspace in the panel layout (see panel_chunk_off); every operand
// of a problem has the same batch stride.  An operand is K-major (its rows are the M or N
// index, k runs along the panel rows) or MN-major (M or N runs along the panel rows, k down
// the rows), which lets the chain run on a tall matrix as stored: its Gram X^T X takes both
// operands MN-major, its update X B both K-major.
constexpr int kAMn = 1;   // GemmProb::major: A MN-major
constexpr int kBMn = 2;   // B MN-major
// The operand is a symmetric matrix of which only the 256 x 256 tiles on and below the
// diagonal are stored: a block above the diagonal is read as the transpose of its mirror
// (the same rows of the stored matrix, taken MN-major instead of K-major).
constexpr int kASym = 4;
constexpr int kBSym = 8;
struct GemmProb {
  int64_t a_off, b_off, c_off, d_off;  // byte offsets of batch 0
  int64_t c_lo, d_lo;                  // kUpdate: bf16 low parts of C (read) / D (written), or -1
  int64_t bs;                          // byte stride between batches (every operand)
  int32_t a_ph, b_ph, d_ph;            // panel heights (padded rows) of A, B and C / D
  int32_t major;                       // kAMn | kBMn | kASym | kBSym
  int32_t mt, nt, kt;                  // 256-row tiles, BN-column tiles, 64-deep k blocks
  int32_t batch, tiles_per_batch, tile_begin;
  int32_t scale_idx;                   // scale of batch 0 in GemmParams::scales, or -1
  // Hyperball partials of the last update (kUpdate with GemmParams::partials): the caller's
  // weight W (rows w_m x w_n, leading dimension w_ld) read in the epilogue next to O.
  const void *w;                       // NULL: no partials for this problem
  int32_t w_m, w_n, w_ld;
  int32_t w_flags;                     // kPwTiled | kPwVec (W is bf16; X has W's orientation)
  int32_t w_tiles_c;                   // kPwTiled: tiles per tile-row (batch b = tile (b / tc, b % tc))
  int32_t part_begin;                  // first partial record of this problem (16 per tile)
};
constexpr int kPwTiled = 4;  // batch b is the T x T tile (b / w_tiles_c, b % w_tiles_c) of W
constexpr int kPwVec = 8;    // W rows may be read with 16-byte loads
constexpr int kPartsPerTile = 16;   // partial records per 256 x 256 tile (one per epilogue warp)
enum GemmMode { kGram = 0, kPoly = 1, kUpdate = 2, kGramF32 = 5 };
struct GemmHead {
  CUtensorMap tmap;       // 2-SM kernel: the workspace seen as rows of 128 bytes (64 bf16),
                          // 64-row boxes, no swizzle (the data is stored pre-swizzled)
  char *ws;
  const float *scales;
  uint32_t *status;
  double *partials;       // kUpdate: (||O||^2, <W,O>, ||W||^2) records of problems with w, or NULL
  long long wait_limit;   // clock cycles a role may wait on one mbarrier phase
  int32_t mode;           // kGram: D = s^2 acc (tiles on and below the diagonal)
                          // kPoly: D = cb C + cc acc (tiles on and below the diagonal)
                          // kUpdate: D = s (ca C + acc), B operand MN-major; C may be a
                          //          hi + lo pair and D may be written as one
                          // kGramF32: D = acc in fp32 (tiles on and below the diagonal)
  float ca, cb, cc;
  int32_t nprob, total_tiles;
  int32_t test_stall;     // tests only: the MMA warp withholds its first accumulator commit,
                          // so the epilogue's bounded wait runs out (NSHB_DEV_TIMEOUT)
};
struct GemmParams : GemmHead {
  GemmProb prob[kMaxProb];
};
// The Gram S = Z Z^T of the Newton-Muon layer inputs, read straight from the caller's
// row-major bf16 Z (d x n): problem i's A and B operands come through zmap[i] (128-byte
// swizzled boxes of 64 columns x 128 rows, zeros outside Z), the fp32 result goes to the
// workspace (c_off / d_off) as in kGramF32.
constexpr int kMaxZMaps = 64;
struct SyrkParams : GemmHead {
  GemmProb prob[kMaxZMaps];
  CUtensorMap zmap[kMaxZMaps];
};

// Tile-resident Hierarchical Muon (T = 256): one record per tiled matrix; its tiles are
// consecutive T x T panel matrices (128 KB each) from x0 on.
struct HmProb {
  int64_t x0;              // X0 of tile 0 (read once per tile)
  int64_t xo;              // where the final O of tile 0 is written
  int64_t xl0, xl1;        // low parts of X0 / X1 (compensated iterations), or -1
  int32_t tile_begin;      // first tile of this matrix in the launch
  int32_t ntiles;
  int32_t seg_begin;       // scale of tile 0 in scales
  int32_t w_tiles_c;       // tiles per tile-row of the matrix (tile t = (t / w_tiles_c, t % w_tiles_c))
  // Hyperball partials (HmParams::partials): the caller's W read next to the final O.
  const void *w;           // NULL: no partials for this matrix
  int32_t w_m, w_n, w_ld;
  int32_t w_flags;         // kPwVec (W is bf16)
  int32_t part_begin;      // first record (one per epilogue warp and tile)
  int32_t pad_;
};
struct HmParams {
  CUtensorMap tmap;        // the workspace as 128-byte rows, 128-row boxes (see GemmParams)
  char *ws;
  const float *scales;
  uint32_t *status;
  double *partials;        // (||O||^2, <W,O>, ||W||^2) records, or NULL
  long long wait_limit;
  int32_t ns_steps, comp, nprob, total_tiles;
  int32_t test_stall;      // tests only: the MMA warp withholds the first Gram commit of its
                           // first tile, so the epilogues' bounded wait runs out
  int32_t pad_;
  float coef[32][3];       // (a, b, c) of every iteration
  HmProb prob[kMaxProb];
};

// fp32 SIMT GEMM problem (row-major fp32 operands in the workspace).
constexpr int kF32Tile = 128;   // output tile of the fp32 GEMM (kF32Tile x kF32Tile)
struct F32Prob {
  int64_t a_off, b_off, c_off, d_off;
  int32_t M, N, K;
  int32_t lda, ldb, ldc;   // ldd = ldc
  int32_t b_trans;         // 1: B element (k, j) at b[j * ldb + k]; 0: at b[k * ldb + j]
  int32_t tiles_n, tile_begin;
  int32_t scale_idx;
};
struct F32Params {
  char *ws;
  const float *scales;
  int32_t mode;            // as GemmMode (no symmetry exploited)
  float ca, cb, cc;
  int32_t nprob, total_tiles;
  F32Prob prob[kMaxProb];
};

// Newton-Muon helpers.
struct CholParams {          // the ridge of a batch of layer-input Gram matrices
  char *ws;
  uint32_t *status;
  int64_t s_off[kMaxMats];   // fp32 row-major S (ld = ld[i], padded size)
  int32_t ld[kMaxMats], d[kMaxMats];
  float ridge_rel;
  int32_t n;
};

// Checks of one matrix that every entry point makes, in this order: sizes, limits, pointers,
// dtype, element alignment (W, G, O_out to their element; M and, when given, V to 4 bytes).
// w_only: only W is read (the norm entry points), so G, M and V are not looked at.
nshb_status check_matrix(const nshb_matrix &d, const float *V = nullptr, bool need_v = false, bool w_only = false);
// Records a CUDA error for nshb_last_cuda_error (per calling thread) and clears it.
void record_cuda_error(cudaError_t e);

// Split-precision (bf16 x 3) products of the Newton-Muon preconditioner (newton_tc.cu):
// D = A B^T (B K-major), D = A B (B MN-major) or D = C - A B^(T), over 256 x 256 tiles of
// one M x N region, with A = A_hi + A_lo and B = B_hi + B_lo held as bf16 panel matrices.
constexpr int kNwBMn = 1;     // B MN-major
constexpr int kNwNeg = 2;     // D = -A B (no C)
constexpr int kMaxNwProb = 200;
struct NwProb {
  int64_t a_hi, a_lo, b_hi, b_lo;  // panel matrices of A and B (workspace byte offsets of panel 0)
  int64_t c32, d32;                // fp32 row-major C / D: byte offset of the region's (0, 0), or -1
  int64_t dhi, dlo;                // panel matrices of D (hi, lo), or -1
  int32_t a_ph, b_ph, d_ph;        // panel heights
  int32_t a_r0, a_k0;              // A region: first row, first k (multiple of 64)
  int32_t b_r0, b_k0;              // B region: first n (row if K-major, column if MN-major), first k
  int32_t d_r0, d_c0;              // D region within D's panels
  int32_t ld32;                    // row stride (elements) of the fp32 C and D
  int32_t m_valid, n_valid;        // rows / columns of the fp32 D region that exist
  int32_t mt, nt, kt;              // 256-row tiles, 256-column tiles, 64-deep k panels (even)
  int32_t flags;                   // kNwBMn | kNwNeg
  int32_t tile_begin;
};
struct NwParams {
  CUtensorMap tmap;                // the workspace as 128-byte rows (see GemmParams)
  char *ws;
  uint32_t *status;
  long long wait_limit;
  int32_t nprob, total_tiles;
  int32_t late_wait;               // 1: the inputs were complete when the previous kernel let this
                                   // one start, so it runs beside that kernel and waits for it at the end
  int32_t pad_;
  NwProb prob[kMaxNwProb];
};

// fp32 row-major regions -> bf16 hi/lo panel matrices (and optionally an fp32 copy with
// another leading dimension), zero outside the source region up to the padded extents.
struct SplitItem {
  int64_t src32;                   // workspace byte offset of the source's (0, 0)
  int64_t dst32;                   // fp32 copy's (0, 0), or -1
  int64_t dhi, dlo;                // panel matrices (panel 0)
  int32_t src_ld, dst_ld;          // elements
  int32_t rows, cols;              // source extent
  int32_t prow, pcol;              // padded extent written (multiples of 64)
  int32_t d_ph, d_r0, d_c0;        // destination panels: height, region origin
  int32_t blk_begin;               // first 64 x 64 block of this item in the launch
};
struct SplitParams {
  char *ws;
  int32_t n, total_blocks;
  SplitItem item[kMaxMats];
};

// Cholesky factor and inverse of one 256 x 256 diagonal block per layer input (column
// block k), written as bf16 hi/lo panels into the stack of the 512 x 512 diagonal blocks'
// inverses (Dp x 512): block k at rows 256 k, columns 256 (k % 2); an even block also
// zeroes columns 256 .. 511 of its rows.
struct DiagParams {
  char *ws;
  uint32_t *status;
  int32_t n, k;
  int64_t s32[kMaxMats];           // fp32 S (row-major, ld[i])
  int64_t dhi[kMaxMats], dlo[kMaxMats];
  int32_t ld[kMaxMats];            // S row stride = panel height of the inverse stack
};

// Launchers (defined in the .cu files); each returns cudaGetLastError().
cudaError_t launch_momentum(const MomentumParams &p, cudaStream_t s);
cudaError_t launch_norm_finalize(const NormFinParams &p, int nseg_total, cudaStream_t s);
cudaError_t launch_reduce(const ApplyParams &p, cudaStream_t s);
cudaError_t launch_exact_norm(const ApplyParams &p, cudaStream_t s);
cudaError_t launch_apply_finalize(const ApplyFinParams &p, cudaStream_t s);
cudaError_t launch_apply(const ApplyParams &p, cudaStream_t s);
cudaError_t launch_adam(const AdamParams &p, cudaStream_t s);
// 2-SM (CTA pair) form: 256 x 256 tiles, tcgen05.mma.cta_group::2; p.tmap must be encoded.
cudaError_t launch_gemm_tc2(const GemmParams &p, int num_sms, cudaStream_t s);
cudaError_t launch_gemm_syrk(const SyrkParams &p, int num_sms, cudaStream_t s);
// Tile-resident Hierarchical Muon for T = 256 (all iterations of a tile on one CTA pair).
cudaError_t launch_himuon_tile(const HmParams &p, int num_sms, cudaStream_t s);
// The same for T = 128, one tile per CTA, two CTAs per SM.
cudaError_t launch_himuon_tile128(const HmParams &p, int num_sms, cudaStream_t s);
// Encodes p.tmap for a workspace of `bytes` bytes at `ws` (host; driver entry point).
cudaError_t encode_ws_tensor_map(CUtensorMap *map, void *ws, size_t bytes);
// Row-major bf16 d x n (n a multiple of 64, 16-byte aligned): 64 x 128 boxes, 128-byte swizzle.
cudaError_t encode_z_tensor_map(CUtensorMap *map, const void *z, int64_t d, int64_t n);
cudaError_t launch_gemm_f32(const F32Params &p, cudaStream_t s);
cudaError_t launch_ridge(const CholParams &p, cudaStream_t s);
// reserve_pairs: SM pairs left to a kernel that runs beside this one (the grid is that much
// smaller, so that every CTA pair is resident from the start).
cudaError_t launch_newton_gemm(const NwParams &p, int num_sms, cudaStream_t s, int reserve_pairs = 0);
cudaError_t launch_split(const SplitParams &p, cudaStream_t s);
cudaError_t launch_potrf_diag(const DiagParams &p, cudaStream_t s);

constexpr size_t kMaxParamBytes = 32764;   // kernel parameter limit (CUDA 12.1+, sm_70+)
static_assert(sizeof(MomentumParams) <= kMaxParamBytes, "MomentumParams");
static_assert(sizeof(NormFinParams) <= kMaxParamBytes, "NormFinParams");
static_assert(sizeof(ApplyParams) <= kMaxParamBytes, "ApplyParams");
static_assert(sizeof(ApplyFinParams) <= kMaxParamBytes, "ApplyFinParams");
static_assert(sizeof(AdamParams) <= kMaxParamBytes, "AdamParams");
static_assert(sizeof(GemmParams) <= kMaxParamBytes, "GemmParams");
static_assert(sizeof(HmParams) <= kMaxParamBytes, "HmParams");
static_assert(sizeof(F32Params) <= kMaxParamBytes, "F32Params");
static_assert(sizeof(SyrkParams) <= kMaxParamBytes, "SyrkParams");
static_assert(sizeof(CholParams) <= kMaxParamBytes, "CholParams");
static_assert(sizeof(NwParams) <= kMaxParamBytes, "NwParams");
static_assert(sizeof(SplitParams) <= kMaxParamBytes, "SplitParams");
static_assert(sizeof(DiagParams) <= kMaxParamBytes, "DiagParams");

}  // namespace nshb
