// C ABI of the optimizer step: argument validation, workspace planning and the launch
// sequence.  Host code only; every step of the path runs in the kernels of this library.
//
// Launch sequence of a step (all on the caller's stream, no host synchronisation):
//   memset(status) -> momentum -> norm finalize -> K x {Gram, Poly, Update} GEMMs
//   -> [reduce -> finalize -> exact norm -> finalize] -> apply
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/nshb.h"
#include "nshb_internal.h"

namespace nshb {

thread_local int g_last_cuda_error = 0;   // last CUDA error seen by this thread's calls

namespace {

constexpr size_t kAlign = 256;
constexpr long long kWaitLimit = 4000000000LL;  // ~2 s of SM clock per mbarrier phase
constexpr long long kWaitLimitTest = 2000000LL; // ~1 ms (debug_flags bit 0)
constexpr float kKeller[3] = {3.4445f, -4.7750f, 2.0315f};

size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }
// Matrices whose wide side has fewer rows than this run their NS in fp32 even on the bf16
// path: the tensor-core chain would pad them to 256-row panels, and with so few singular
// values the bf16 rounding of B (amplified by the a + B cancellation near sigma = 1) is not
// averaged over a spectrum (a rank-1 input is 5 % off in bf16).
constexpr int64_t kSmallNsF32 = 32;
int64_t round_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

struct MatPlan {
  int64_t m = 0, n = 0, ld = 0;
  bool tall = false;
  int64_t r = 0, s = 0;          // wide-side dims of X
  int64_t Rp = 0, Sp = 0;        // bf16: padded X dims (panel height, columns)
  int flags = 0;
  int64_t x0 = 0, x1 = 0, a = 0, b = 0;   // workspace offsets
  int64_t xl0 = -1, xl1 = -1;             // bf16 low parts of X0 / X1 (compensated iterations)
  bool f32 = false;              // NS in fp32 (CUDA cores) for this matrix
  int T = 0, tiles_r = 0, tiles_c = 0, ntiles = 0;
  int seg_begin = 0, nseg = 0;
  int pr = 0, pc = 0;            // momentum block domain (W coordinates)
  int k1_blocks = 0, k1_begin = 0;
  int w_blocks = 0, w_begin = 0;
  // (||O||^2, <W,O>, ||W||^2) records: from the last NS update's epilogue (fused: one per
  // epilogue warp and output tile) or from the reduce pass (one per 64 x 64 block of W)
  bool fused = false;
  int rec_begin = 0, rec_count = 0;
};

struct Plan {
  int op = 0;
  bool f32ns = false;
  bool tiled = false;
  int bn = 256;
  int comp = 0;                  // compensated (hi/lo) iterations of the bf16 chain
  std::vector<MatPlan> mp;
  // Newton-Muon: per layer input Z (d rows, padded to Dp = a multiple of 256)
  struct ZPlan {
    int64_t d = 0, Dp = 0;
    const void *src = nullptr;
    int64_t s = 0;                    // S = Z Z^T + lambda I, fp32 Dp x Dp, updated in place
    int64_t sh = 0, sl = 0;           // bf16 hi / lo panels of S (operands of the panel products)
    int64_t lh = 0, ll = 0;           // bf16 hi / lo panels of the Cholesky factor L
    int64_t dh = 0, dl = 0;           // hi / lo panels of the stacked inverses of the 512 x 512 diagonal
                                      // blocks (Dp x 512): rows 512 j .. +511 hold the inverse of
                                      // L's diagonal block j of 512 (block k of 256 at columns 256 (k % 2))
  };
  std::vector<ZPlan> zp;
  int64_t n_tokens = 0;
  std::vector<int64_t> r_off;         // per matrix: fp32 m x n, U (momentum) and then P
  std::vector<int64_t> y32, yh, yl;   // per matrix: fp32 Mp x Dp U -> Y, and its hi / lo panels
  std::vector<int64_t> ph, plo;       // per matrix: hi / lo panels of P (Mp x Dp), the backward's operand
  std::vector<int64_t> mpad;          // per matrix: rows padded to 256
  std::vector<int> zidx;
  size_t scal_off = 0, scale_off = 0, nu_off = 0, k1part_off = 0, wpart_off = 0, xpart_off = 0, total = 0;
  int nseg = 0, k1_total = 0, w_total = 0, rec_total = 0;
};

// Steps whose update rule needs (||O||^2, <W,O>, ||W||^2).
bool needs_partials(int op) {
  return op == NSHB_OP_HYPERBALL || op == NSHB_OP_RADIAL_BRAKE || op == NSHB_OP_RELATIVE_UPDATE ||
         op == NSHB_OP_HIMUON || op == NSHB_OP_NEWTON_MUON;
}

nshb_status plan_step(const nshb_matrix *mats, int n_mats, const nshb_params *p, int op, Plan &pl) {
  if (!p) return NSHB_ERR_NULL;
  if (n_mats < 0) return NSHB_ERR_SHAPE;
  if (n_mats > 0 && !mats) return NSHB_ERR_NULL;
  if (op < NSHB_OP_MUON || op > NSHB_OP_RELATIVE_UPDATE) return NSHB_ERR_PARAM;
  if (!(p->beta >= 0.f && p->beta < 1.f)) return NSHB_ERR_PARAM;
  if (p->ns_steps < 1 || p->ns_steps > 32) return NSHB_ERR_PARAM;
  if (!(p->ns_eps > 0.f) || !std::isfinite(p->ns_eps)) return NSHB_ERR_PARAM;
  if (!(p->hb_eps > 0.f) || !std::isfinite(p->hb_eps)) return NSHB_ERR_PARAM;
  if (!std::isfinite(p->lr) || !std::isfinite(p->weight_decay) || !std::isfinite(p->eta) || p->eta < 0.f)
    return NSHB_ERR_PARAM;
  if (op == NSHB_OP_RADIAL_BRAKE) {
    if (!(p->brake_out >= 0.f && p->brake_out <= 1.f && p->brake_in >= 0.f && p->brake_in <= 1.f))
      return NSHB_ERR_PARAM;
    if (p->weight_decay != 0.f) return NSHB_ERR_PARAM;
  }
  if (p->ns_precision != NSHB_BF16 && p->ns_precision != NSHB_F32) return NSHB_ERR_DTYPE;
  if (p->ns_compensated < 0 || p->ns_compensated > 32) return NSHB_ERR_PARAM;
  if (p->coeffs)
    for (int i = 0; i < 3 * p->ns_steps; ++i)
      if (!std::isfinite(p->coeffs[i])) return NSHB_ERR_PARAM;
  if ((uintptr_t)p->rho % sizeof(float)) return NSHB_ERR_PARAM;
  pl.op = op;
  pl.f32ns = p->ns_precision == NSHB_F32;
  pl.tiled = op == NSHB_OP_HIMUON;
  pl.comp = pl.f32ns ? 0 : std::min(p->ns_compensated, p->ns_steps);
  if (pl.tiled) {
    if (pl.f32ns) return NSHB_ERR_UNSUPPORTED;
    if (p->tile != 128 && p->tile != 256 && p->tile != 512) return NSHB_ERR_PARAM;
    pl.bn = p->tile == 128 ? 128 : 256;
  }
  if (op == NSHB_OP_NEWTON_MUON) {
    if (!(p->ridge_rel >= 0.f) || !std::isfinite(p->ridge_rel)) return NSHB_ERR_PARAM;
  }
  pl.mp.resize(n_mats);
  for (int i = 0; i < n_mats; ++i) {
    const nshb_matrix &d = mats[i];
    MatPlan &m = pl.mp[i];
    const nshb_status ce = check_matrix(d);
    if (ce != NSHB_OK) return ce;
    m.m = d.rows;
    m.n = d.cols;
    m.ld = d.ld;
    const bool wf32 = d.w_dtype == NSHB_F32;
    const size_t esz = wf32 ? 4 : 2;
    const bool vec = ((uintptr_t)d.W % 16 == 0) && ((uintptr_t)d.G % 16 == 0) && ((uintptr_t)d.M % 16 == 0) &&
                     ((d.ld * esz) % 16 == 0) && ((d.ld * 4) % 16 == 0);
    m.f32 = pl.f32ns || (!pl.tiled && std::min(d.rows, d.cols) < kSmallNsF32);
    m.flags = (vec ? kVec : 0) | (wf32 ? kWF32 : 0) | (m.f32 ? kNsF32 : 0);
    if (pl.tiled) {
      m.flags |= kTiled;
      m.T = p->tile;
      m.tiles_r = (int)((m.m + m.T - 1) / m.T);
      m.tiles_c = (int)((m.n + m.T - 1) / m.T);
      m.ntiles = m.tiles_r * m.tiles_c;
      m.pr = m.tiles_r * m.T;
      m.pc = m.tiles_c * m.T;
      m.nseg = m.ntiles;
    } else {
      m.tall = m.m > m.n;
      if (m.tall) m.flags |= kTall;
      m.r = m.tall ? m.n : m.m;
      m.s = m.tall ? m.m : m.n;
      if (m.f32) {
        m.pr = (int)round_up(m.m, kBlk);
        m.pc = (int)round_up(m.n, kBlk);
      } else {
        m.Rp = round_up(m.r, 256);
        m.Sp = round_up(m.s, 256);
        m.pr = (int)(m.tall ? m.Sp : m.Rp);
        m.pc = (int)(m.tall ? m.Rp : m.Sp);
      }
      m.nseg = 1;
    }
    m.k1_blocks = (m.pr / kBlk) * (m.pc / kBlk);
    m.w_blocks = (int)(((m.m + kBlk - 1) / kBlk) * ((m.n + kBlk - 1) / kBlk));
    // The partials come from the epilogue that writes the final O wherever the NS runs on
    // the tensor cores: the pair GEMM's last update (one record per epilogue warp and 256 x
    // 256 output tile) or the tile-resident Hierarchical-Muon kernels (one per epilogue warp
    // and tile: 16 for T = 256, 4 for T = 128).  The fp32 chain and fp32 weights leave them
    // to the reduce pass.
    m.fused = needs_partials(op) && !m.f32 && !wf32;
    if (m.fused) {
      int64_t recs;
      if (!pl.tiled) recs = (m.Rp / 256) * (m.Sp / 256) * kPartsPerTile;
      else if (m.T == 512) recs = (int64_t)m.ntiles * 4 * kPartsPerTile;
      else recs = (int64_t)m.ntiles * (m.T == 256 ? kPartsPerTile : 4);
      m.rec_count = (int)recs;
    } else {
      m.rec_count = m.w_blocks;
    }
  }
  // Workspace layout.
  size_t off = kAlign;  // [0, 256): device status word
  pl.scal_off = off;
  off = align_up(off + sizeof(MatScalars) * (size_t)n_mats);
  pl.nseg = 0;
  pl.k1_total = 0;
  pl.w_total = 0;
  pl.rec_total = 0;
  for (auto &m : pl.mp) {
    m.seg_begin = pl.nseg;
    pl.nseg += m.nseg;
    m.k1_begin = pl.k1_total;
    pl.k1_total += m.k1_blocks;
    m.w_begin = pl.w_total;
    pl.w_total += m.w_blocks;
    m.rec_begin = pl.rec_total;
    pl.rec_total += m.rec_count;
  }
  pl.scale_off = off;
  off = align_up(off + sizeof(float) * (size_t)pl.nseg);
  pl.nu_off = off;
  off = align_up(off + sizeof(double) * (size_t)pl.nseg);
  pl.k1part_off = off;
  off = align_up(off + kK1PartsPerBlock * sizeof(double) * (size_t)pl.k1_total);
  pl.wpart_off = off;
  off = align_up(off + 3 * sizeof(double) * (size_t)pl.rec_total);
  pl.xpart_off = off;
  off = align_up(off + sizeof(double) * (size_t)pl.w_total);
  for (auto &m : pl.mp) {
    size_t xb, ab;
    if (pl.tiled) {
      xb = (size_t)m.ntiles * m.T * m.T * 2;
      ab = xb;
    } else if (m.f32) {
      xb = (size_t)m.r * m.s * 4;
      ab = (size_t)m.r * m.r * 4;
    } else {
      xb = (size_t)m.Rp * m.Sp * 2;
      ab = (size_t)m.Rp * m.Rp * 2;
    }
    m.x0 = off; off = align_up(off + xb);
    m.x1 = off; off = align_up(off + xb);
    m.a = off;  off = align_up(off + ab);
    m.b = off;  off = align_up(off + ab);
    if (pl.comp > 0 && !m.f32) {
      m.xl0 = off; off = align_up(off + xb);
      if (pl.comp > 1) { m.xl1 = off; off = align_up(off + xb); }
    }
  }
  pl.total = off;
  return NSHB_OK;
}

// Extends a plan with the Newton-Muon buffers (layer inputs, Gram / Cholesky factors, the
// fp32 right-hand sides of the triangular solves).
nshb_status plan_newton(const nshb_matrix *mats, int n_mats, const void *const *Z, const int64_t *z_rows, int n_z,
                        int64_t n_tokens, Plan &pl) {
  if (n_z <= 0 || n_z > kMaxMats || !z_rows) return n_z <= 0 || !z_rows ? NSHB_ERR_NULL : NSHB_ERR_UNSUPPORTED;
  if (n_tokens <= 0 || n_tokens % 64 != 0 || n_tokens > (1LL << 24)) return NSHB_ERR_SHAPE;
  if (pl.f32ns) return NSHB_ERR_UNSUPPORTED;
  pl.n_tokens = n_tokens;
  pl.zp.resize(n_z);
  size_t off = pl.total;
  for (int j = 0; j < n_z; ++j) {
    Plan::ZPlan &z = pl.zp[j];
    z.d = z_rows[j];
    if (z.d <= 0 || z.d % 64 != 0 || z.d > 16384) return NSHB_ERR_SHAPE;
    z.src = Z ? Z[j] : nullptr;
    if (Z && (!z.src || (uintptr_t)z.src % 16 != 0)) return !z.src ? NSHB_ERR_NULL : NSHB_ERR_SHAPE;
    z.Dp = round_up(z.d, 256);
    const size_t sq = (size_t)z.Dp * z.Dp;
    z.s = off;  off = align_up(off + sq * 4);
    z.sh = off; off = align_up(off + sq * 2);
    z.sl = off; off = align_up(off + sq * 2);
    z.lh = off; off = align_up(off + sq * 2);
    z.ll = off; off = align_up(off + sq * 2);
    z.dh = off; off = align_up(off + (size_t)z.Dp * 512 * 2);
    z.dl = off; off = align_up(off + (size_t)z.Dp * 512 * 2);
  }
  pl.r_off.resize(n_mats);
  pl.y32.resize(n_mats);
  pl.yh.resize(n_mats);
  pl.yl.resize(n_mats);
  pl.ph.resize(n_mats);
  pl.plo.resize(n_mats);
  pl.mpad.resize(n_mats);
  pl.zidx.resize(n_mats);
  for (int i = 0; i < n_mats; ++i) {
    const int zi = mats[i].z_index;
    if (zi < 0 || zi >= n_z) return NSHB_ERR_PARAM;
    if (pl.zp[zi].d != mats[i].cols) return NSHB_ERR_SHAPE;
    pl.zidx[i] = zi;
    const int64_t Mp = round_up(mats[i].rows, 256), Dp = pl.zp[zi].Dp;
    pl.mpad[i] = Mp;
    pl.r_off[i] = off; off = align_up(off + (size_t)mats[i].rows * mats[i].cols * 4);
    pl.y32[i] = off;   off = align_up(off + (size_t)Mp * Dp * 4);
    pl.yh[i] = off;    off = align_up(off + (size_t)Mp * Dp * 2);
    pl.yl[i] = off;    off = align_up(off + (size_t)Mp * Dp * 2);
  }
  // The backward solve writes P's hi / lo panels (Mp x Dp) straight into X0 and its low part
  // when they are the NS operand's layout (bf16 panels of height round_up(m, 256) and width
  // round_up(n, 256), either orientation).  A matrix whose NS runs in fp32 (fewer than 32 rows)
  // gets panels of its own, and the pass after the solve writes its X0 from the fp32 P.
  for (int i = 0; i < n_mats; ++i) {
    const MatPlan &m = pl.mp[i];
    const int64_t Mp = pl.mpad[i], Dp = pl.zp[pl.zidx[i]].Dp;
    const bool in_place = !m.f32 && m.pr == Mp && m.pc == Dp;
    pl.ph[i] = in_place ? m.x0 : -1;
    pl.plo[i] = in_place ? m.xl0 : -1;
    if (pl.ph[i] < 0) {
      pl.ph[i] = off;
      off = align_up(off + (size_t)Mp * Dp * 2);
    }
    if (pl.plo[i] < 0) {   // also when no compensated NS iteration keeps a low part of X0
      pl.plo[i] = off;
      off = align_up(off + (size_t)Mp * Dp * 2);
    }
  }
  pl.total = off;
  return NSHB_OK;
}

MatDesc make_desc(const nshb_matrix &d, const MatPlan &m, int idx, int64_t o_off, int blk_begin, bool k1) {
  MatDesc r;
  std::memset(&r, 0, sizeof(r));
  r.W = d.W;
  r.G = d.G;
  r.M = d.M;
  r.O_out = d.O_out;
  r.x_off = m.x0;
  r.xlo_off = m.xl0;
  r.u_off = 0;
  r.o_off = o_off;
  r.m = (int)m.m;
  r.n = (int)m.n;
  r.ld = (int)m.ld;
  r.flags = m.flags;
  if (m.flags & kTiled) r.ph = m.T;
  else if (m.flags & kNsF32) r.ph = (int)m.s;
  else r.ph = (int)(m.tall ? m.Sp : m.Rp);   // bf16 X = U as stored: m rows, padded
  if (k1) {
    r.pr = m.pr;
    r.pc = m.pc;
    if (m.flags & kTiled) r.flags |= kTileMajor;  // momentum blocks walk tile by tile
  } else {
    r.pr = (int)round_up(m.m, kBlk);
    r.pc = (int)round_up(m.n, kBlk);
  }
  r.blk_begin = blk_begin;
  r.seg_begin = m.seg_begin;
  r.tiles_c = m.tiles_c;
  r.mat = idx;
  r.rec_begin = m.rec_begin;
  return r;
}

// Output tiles of one GEMM problem: all mt x nt tiles, or for the symmetric phases only
// those that touch the lower triangle (BM-row block mi needs the BN-wide column tiles
// that start at or before its last row).
int gemm_tiles(int mode, int mt, int nt, int bm, int bn) {
  if (mode == kUpdate) return mt * nt;
  int cnt = 0;
  for (int mi = 0; mi < mt; ++mi) cnt += std::min(nt, (bm * mi + bm - 1) / bn + 1);
  return cnt;
}

int device_sms() {
  static PerDevice cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  int v = cache.get(dev);
  if (!v) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    cache.set(dev, v);
  }
  return v;
}

#define NSHB_CHECK_CUDA(x)                 \
  do {                                     \
    cudaError_t e_ = (x);                  \
    if (e_ != cudaSuccess) {               \
      g_last_cuda_error = (int)e_;         \
      (void)cudaGetLastError();            \
      return NSHB_ERR_CUDA;                \
    }                                      \
  } while (0)


// ---------------------------------------------------------------- phase timing
// Opt-in measurement aid: when enabled, every kernel launch of a step is bracketed by two
// CUDA events on the caller's stream; nshb_profile_read sums the elapsed times per kind.
struct Profiler {
  std::mutex mu;
  std::atomic<bool> on{false};   // read without the lock on every launch
  struct Rec {
    cudaEvent_t a, b;
    int kind;
  };
  std::vector<Rec> recs;
  std::vector<cudaEvent_t> pool;
  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }
};
Profiler &prof() {
  static Profiler p;
  return p;
}
struct ProfScope {
  cudaEvent_t a = nullptr;
  int kind;
  cudaStream_t st;
  ProfScope(int k, cudaStream_t s) : kind(k), st(s) {
    Profiler &p = prof();
    if (!p.on) return;
    std::lock_guard<std::mutex> g(p.mu);
    a = p.get();
    if (a) cudaEventRecord(a, st);
  }
  ~ProfScope() {
    if (!a) return;
    Profiler &p = prof();
    std::lock_guard<std::mutex> g(p.mu);
    cudaEvent_t b = p.get();
    if (!b) return;
    cudaEventRecord(b, st);
    p.recs.push_back({a, b, kind});
  }
};

#define NSHB_LAUNCH(kind, call)   \
  do {                            \
    ProfScope ps_(kind, st);      \
    NSHB_CHECK_CUDA(call);        \
  } while (0)

// momentum + per-segment norms
nshb_status run_momentum(const nshb_matrix *mats, const Plan &pl, const nshb_params *p, char *ws,
                         cudaStream_t st, bool from_p = false) {
  const int n = (int)pl.mp.size();
  double *k1part = reinterpret_cast<double *>(ws + pl.k1part_off);
  for (int c0 = 0; c0 < n; c0 += kMaxMats) {
    const int c1 = std::min(n, c0 + kMaxMats);
    MomentumParams mp;
    std::memset(&mp, 0, sizeof(mp));
    mp.ws = ws;
    mp.partials = k1part + kK1PartsPerBlock * (int64_t)pl.mp[c0].k1_begin;
    mp.status = reinterpret_cast<uint32_t *>(ws);
    mp.beta = p->beta;
    mp.nesterov = p->nesterov ? 1 : 0;
    mp.nmat = c1 - c0;
    int nb = 0;
    for (int i = c0; i < c1; ++i) {
      mp.mats[i - c0] = make_desc(mats[i], pl.mp[i], i, 0, nb, true);
      if (from_p) {
        // Where the backward solve wrote P's hi / lo panels into X0 they already are the
        // operand, and the pass only forms the norm; otherwise it writes X0 from the fp32 P.
        mp.mats[i - c0].flags |= kFromP | (pl.ph[i] == pl.mp[i].x0 ? kNoX : 0);
        mp.mats[i - c0].u_off = pl.r_off[i];
      }
      nb += pl.mp[i].k1_blocks;
    }
    mp.total_blocks = nb;
    NSHB_LAUNCH(NSHB_PROF_MOMENTUM, launch_momentum(mp, st));

    NormFinParams nf;
    std::memset(&nf, 0, sizeof(nf));
    nf.partials = k1part + kK1PartsPerBlock * (int64_t)pl.mp[c0].k1_begin;
    const int seg0 = pl.mp[c0].seg_begin;
    nf.scales = reinterpret_cast<float *>(ws + pl.scale_off) + seg0;
    nf.nus = reinterpret_cast<double *>(ws + pl.nu_off) + seg0;
    nf.status = reinterpret_cast<uint32_t *>(ws);
    nf.ns_eps = p->ns_eps;
    nf.nmat = c1 - c0;
    int segs = 0, blks = 0;
    for (int i = c0; i < c1; ++i) {
      const MatPlan &m = pl.mp[i];
      nf.seg_begin[i - c0] = segs;
      nf.blk_begin[i - c0] = kK1PartsPerBlock * blks;             // partial records
      nf.bps[i - c0] = kK1PartsPerBlock * (m.k1_blocks / m.nseg);  // records per segment
      segs += m.nseg;
      blks += m.k1_blocks;
    }
    nf.seg_begin[c1 - c0] = segs;
    NSHB_LAUNCH(NSHB_PROF_NORM, launch_norm_finalize(nf, segs, st));
  }
  return NSHB_OK;
}

void coeffs_for(const nshb_params *p, int it, float &a, float &b, float &c) {
  if (p->coeffs) {
    a = p->coeffs[3 * it];
    b = p->coeffs[3 * it + 1];
    c = p->coeffs[3 * it + 2];
  } else {
    a = kKeller[0];
    b = kKeller[1];
    c = kKeller[2];
  }
}

// Hierarchical Muon with T = 256 or 128: every tile's whole chain in a tile-resident kernel.
nshb_status run_himuon_tile(const nshb_matrix *mats, const Plan &pl, const nshb_params *p, char *ws,
                            cudaStream_t st) {
  const int n = (int)pl.mp.size();
  for (int c0 = 0; c0 < n; c0 += kMaxProb) {
    const int c1 = std::min(n, c0 + kMaxProb);
    HmParams hp;
    std::memset(&hp, 0, sizeof(hp));
    hp.ws = ws;
    hp.scales = reinterpret_cast<const float *>(ws + pl.scale_off);
    hp.status = reinterpret_cast<uint32_t *>(ws);
    hp.wait_limit = (p->debug_flags & 1u) ? kWaitLimitTest : kWaitLimit;
    hp.ns_steps = p->ns_steps;
    hp.comp = pl.comp;
    hp.test_stall = (p->debug_flags & 2u) ? 1 : 0;
    for (int it = 0; it < p->ns_steps; ++it) coeffs_for(p, it, hp.coef[it][0], hp.coef[it][1], hp.coef[it][2]);
    int tiles = 0;
    for (int i = c0; i < c1; ++i) {
      const MatPlan &m = pl.mp[i];
      HmProb &q = hp.prob[i - c0];
      q.x0 = m.x0;
      q.xo = (p->ns_steps % 2 == 0) ? m.x0 : m.x1;
      q.xl0 = m.xl0;
      q.xl1 = m.xl1;
      q.tile_begin = tiles;
      q.ntiles = m.ntiles;
      q.seg_begin = m.seg_begin;
      q.w_tiles_c = m.tiles_c;
      q.w = nullptr;
      if (m.fused) {
        const nshb_matrix &d = mats[i];
        q.w = d.W;
        q.w_m = (int)m.m;
        q.w_n = (int)m.n;
        q.w_ld = (int)m.ld;
        q.w_flags = (uintptr_t)d.W % 16 == 0 && (d.ld * 2) % 16 == 0 ? kPwVec : 0;   // bf16 W
        q.part_begin = m.rec_begin;
        hp.partials = reinterpret_cast<double *>(ws + pl.wpart_off);
      }
      tiles += m.ntiles;
    }
    hp.nprob = c1 - c0;
    hp.total_tiles = tiles;
    NSHB_CHECK_CUDA(encode_ws_tensor_map(&hp.tmap, ws, pl.total / 128 * 128));
    if (p->tile == 128) NSHB_LAUNCH(NSHB_PROF_GRAM, launch_himuon_tile128(hp, device_sms(), st));
    else NSHB_LAUNCH(NSHB_PROF_GRAM, launch_himuon_tile(hp, device_sms(), st));
  }
  return NSHB_OK;
}

// K iterations of the three NS phases.  Returns the offset of each matrix's O in `o_off`.
nshb_status run_ns(const nshb_matrix *mats, const Plan &pl, const nshb_params *p, char *ws, cudaStream_t st,
                   std::vector<int64_t> &o_off) {
  const int n = (int)pl.mp.size();
  o_off.resize(n);
  const float *scales = reinterpret_cast<const float *>(ws + pl.scale_off);
  uint32_t *status = reinterpret_cast<uint32_t *>(ws);
  const long long limit = (p->debug_flags & 1u) ? kWaitLimitTest : kWaitLimit;
  if (pl.tiled && (p->tile == 256 || p->tile == 128)) {
    const nshb_status e = run_himuon_tile(mats, pl, p, ws, st);
    if (e != NSHB_OK) return e;
    for (int i = 0; i < n; ++i) o_off[i] = (p->ns_steps % 2 == 0) ? pl.mp[i].x0 : pl.mp[i].x1;
    return NSHB_OK;
  }
  std::vector<int> f32_idx, bf_idx;   // matrices whose NS runs in fp32 / on the bf16 tensor cores
  for (int i = 0; i < n; ++i) (pl.mp[i].f32 ? f32_idx : bf_idx).push_back(i);
  for (int it = 0; it < p->ns_steps; ++it) {
    float ca, cb, cc;
    coeffs_for(p, it, ca, cb, cc);
    for (int phase = 0; phase < 3; ++phase) {
      const int mode = phase == 0 ? kGram : phase == 1 ? kPoly : kUpdate;
      {
        const int nf = (int)f32_idx.size();
        for (int c0 = 0; c0 < nf; c0 += kMaxProb) {
          const int c1 = std::min(nf, c0 + kMaxProb);
          F32Params fp;
          std::memset(&fp, 0, sizeof(fp));
          fp.ws = ws;
          fp.scales = scales;
          fp.mode = mode;
          fp.ca = ca; fp.cb = cb; fp.cc = cc;
          int tiles = 0;
          for (int ii = c0; ii < c1; ++ii) {
            const MatPlan &m = pl.mp[f32_idx[ii]];
            const int64_t xin = (it % 2 == 0) ? m.x0 : m.x1, xout = (it % 2 == 0) ? m.x1 : m.x0;
            F32Prob &q = fp.prob[ii - c0];
            if (mode == kGram) {
              q.a_off = xin; q.b_off = xin; q.c_off = m.a; q.d_off = m.a;
              q.M = (int)m.r; q.N = (int)m.r; q.K = (int)m.s;
              q.lda = (int)m.s; q.ldb = (int)m.s; q.ldc = (int)m.r; q.b_trans = 1;
            } else if (mode == kPoly) {
              q.a_off = m.a; q.b_off = m.a; q.c_off = m.a; q.d_off = m.b;
              q.M = (int)m.r; q.N = (int)m.r; q.K = (int)m.r;
              q.lda = (int)m.r; q.ldb = (int)m.r; q.ldc = (int)m.r; q.b_trans = 0;
            } else {
              q.a_off = m.b; q.b_off = xin; q.c_off = xin; q.d_off = xout;
              q.M = (int)m.r; q.N = (int)m.s; q.K = (int)m.r;
              q.lda = (int)m.r; q.ldb = (int)m.s; q.ldc = (int)m.s; q.b_trans = 0;
            }
            q.scale_idx = (it == 0 && mode != kPoly) ? m.seg_begin : -1;
            q.tiles_n = (q.N + kF32Tile - 1) / kF32Tile;
            q.tile_begin = tiles;
            tiles += ((q.M + kF32Tile - 1) / kF32Tile) * q.tiles_n;
          }
          fp.nprob = c1 - c0;
          fp.total_tiles = tiles;
          NSHB_LAUNCH(NSHB_PROF_F32GEMM, launch_gemm_f32(fp, st));
        }
      }
      {
        const int nb = (int)bf_idx.size();
        for (int c0 = 0; c0 < nb; c0 += kMaxProb) {
          const int c1 = std::min(nb, c0 + kMaxProb);
          GemmParams gp;
          std::memset(&gp, 0, sizeof(gp));
          gp.ws = ws;
          gp.scales = scales;
          gp.status = status;
          gp.wait_limit = limit;
          gp.test_stall = (p->debug_flags & 2u) ? 1 : 0;
          gp.mode = mode;
          gp.ca = ca; gp.cb = cb; gp.cc = cc;
          const bool last_update = mode == kUpdate && it + 1 == p->ns_steps;
          gp.partials = nullptr;
          // Longest-k problems first, so the static tile walk ends evenly.
          std::vector<std::pair<int64_t, int>> ord;
          for (int ii = c0; ii < c1; ++ii) {
            const int i = bf_idx[ii];
            const MatPlan &m = pl.mp[i];
            const int64_t kext = pl.tiled ? m.T : (mode == kGram ? m.Sp : m.Rp);
            ord.push_back({-kext, i});
          }
          std::stable_sort(ord.begin(), ord.end());
          int tiles = 0, k = 0;
          for (auto &e : ord) {
            const int i = e.second;
            const MatPlan &m = pl.mp[i];
            const int64_t xin = (it % 2 == 0) ? m.x0 : m.x1, xout = (it % 2 == 0) ? m.x1 : m.x0;
            GemmProb &q = gp.prob[k++];
            int64_t R, S;
            int batch;
            if (pl.tiled) {
              R = m.T; S = m.T; batch = m.ntiles;
            } else {
              R = m.Rp; S = m.Sp; batch = 1;
            }
            q.batch = batch;
            // X, A and B of a tile share one stride (T x T bf16); a whole matrix is one batch
            q.bs = pl.tiled ? (int64_t)m.T * m.T * 2 : 0;
            // A tall matrix keeps X = U (S rows, R columns): its Gram X^T X reads X MN-major on
            // both sides, its update X B reads X and B K-major.  Everything else is R rows.
            const bool tall = !pl.tiled && m.tall;
            const int64_t xph = tall ? S : R;
            q.w = nullptr;
            if (last_update && m.fused) {
              const nshb_matrix &d = mats[i];
              const bool wvec = (uintptr_t)d.W % 16 == 0 && (d.ld * 2) % 16 == 0;   // bf16 W
              q.w = d.W;
              q.w_m = (int)m.m;
              q.w_n = (int)m.n;
              q.w_ld = (int)m.ld;
              q.w_flags = (pl.tiled ? kPwTiled : 0) | (wvec ? kPwVec : 0);
              q.w_tiles_c = m.tiles_c;
              q.part_begin = m.rec_begin;
              gp.partials = reinterpret_cast<double *>(ws + pl.wpart_off);
            }
            q.c_lo = -1;
            q.d_lo = -1;
            if (mode == kUpdate && it < pl.comp) {
              q.c_lo = (it % 2 == 0) ? m.xl0 : m.xl1;
              if (it + 1 < pl.comp) q.d_lo = (it % 2 == 0) ? m.xl1 : m.xl0;
            }
            if (mode == kGram) {
              q.a_off = xin; q.b_off = xin; q.c_off = m.a; q.d_off = m.a;
              q.a_ph = q.b_ph = (int)xph; q.d_ph = (int)R;
              q.major = tall ? (kAMn | kBMn) : 0;
              q.mt = (int)(R / 256); q.nt = (int)(R / pl.bn); q.kt = (int)(S / 64);
            } else if (mode == kPoly) {
              // A is stored on and below the diagonal only (as is every symmetric result)
              q.a_off = m.a; q.b_off = m.a; q.c_off = m.a; q.d_off = m.b;
              q.a_ph = q.b_ph = q.d_ph = (int)R;
              q.major = kASym | kBSym;
              q.mt = (int)(R / 256); q.nt = (int)(R / pl.bn); q.kt = (int)(R / 64);
            } else if (!tall) {
              // X' = s (a X + B X): A = B (K-major, lower triangle stored), B operand = X (MN-major)
              q.a_off = m.b; q.b_off = xin; q.c_off = xin; q.d_off = xout;
              q.a_ph = q.b_ph = q.d_ph = (int)R;
              q.major = kBMn | kASym;
              q.mt = (int)(R / 256); q.nt = (int)(S / pl.bn); q.kt = (int)(R / 64);
            } else {
              // X' = s (a X + X B): A = X (K-major, S rows), B operand = B (symmetric, K-major,
              // lower triangle stored)
              q.a_off = xin; q.b_off = m.b; q.c_off = xin; q.d_off = xout;
              q.a_ph = q.d_ph = (int)S; q.b_ph = (int)R;
              q.major = kBSym;
              q.mt = (int)(S / 256); q.nt = (int)(R / pl.bn); q.kt = (int)(R / 64);
            }
            q.tiles_per_batch = gemm_tiles(mode, q.mt, q.nt, 256, pl.bn);
            q.scale_idx = (it == 0 && mode != kPoly) ? m.seg_begin : -1;
            q.tile_begin = tiles;
            tiles += q.tiles_per_batch * q.batch;
          }
          gp.nprob = k;
          gp.total_tiles = tiles;
          NSHB_CHECK_CUDA(encode_ws_tensor_map(&gp.tmap, ws, pl.total / 128 * 128));
          NSHB_LAUNCH(NSHB_PROF_GRAM + mode, launch_gemm_tc2(gp, device_sms(), st));
        }
      }
    }
  }
  for (int i = 0; i < n; ++i) o_off[i] = (p->ns_steps % 2 == 0) ? pl.mp[i].x0 : pl.mp[i].x1;
  return NSHB_OK;
}

nshb_status run_apply(const nshb_matrix *mats, const Plan &pl, const nshb_params *p, int apply_op, char *ws,
                      cudaStream_t st, const std::vector<int64_t> &o_off, float *norms_out,
                      bool have_partials = false) {
  const int n = (int)pl.mp.size();
  MatScalars *scal = reinterpret_cast<MatScalars *>(ws + pl.scal_off);
  double *wpart = reinterpret_cast<double *>(ws + pl.wpart_off);
  double *xpart = reinterpret_cast<double *>(ws + pl.xpart_off);
  uint32_t *status = reinterpret_cast<uint32_t *>(ws);
  for (int c0 = 0; c0 < n; c0 += kMaxMats) {
    const int c1 = std::min(n, c0 + kMaxMats);
    ApplyParams ap;
    std::memset(&ap, 0, sizeof(ap));
    ap.ws = ws;
    ap.scal = scal;
    ap.status = status;
    ap.op = apply_op;
    ap.nmat = c1 - c0;
    // The reduce pass covers only the matrices whose records the NS epilogue did not write.
    ApplyParams rp = ap;
    rp.nmat = 0;
    rp.partials = wpart;
    ApplyFinParams fp;
    std::memset(&fp, 0, sizeof(fp));
    fp.scal = scal;
    fp.status = status;
    fp.rho = p->rho;
    fp.norms_out = norms_out;
    fp.op = apply_op;
    fp.lr = p->lr;
    fp.weight_decay = p->weight_decay;
    fp.eta = p->eta;
    fp.hb_eps = p->hb_eps;
    fp.brake_out = p->brake_out;
    fp.brake_in = p->brake_in;
    fp.nmat = c1 - c0;
    int nb = 0, rb = 0;
    for (int i = c0; i < c1; ++i) {
      const MatPlan &m = pl.mp[i];
      ap.mats[i - c0] = make_desc(mats[i], m, i, o_off.empty() ? 0 : o_off[i], nb, false);
      if (!m.fused) {
        rp.mats[rp.nmat] = make_desc(mats[i], m, i, o_off.empty() ? 0 : o_off[i], rb, false);
        rp.nmat++;
        rb += m.w_blocks;
      }
      fp.rec_begin[i - c0] = m.rec_begin;
      fp.blk_begin[i - c0] = nb;
      fp.mat[i - c0] = i;
      fp.m[i - c0] = (int)m.m;
      fp.n[i - c0] = (int)m.n;
      nb += m.w_blocks;
    }
    fp.rec_begin[c1 - c0] = pl.mp[c1 - 1].rec_begin + pl.mp[c1 - 1].rec_count;
    fp.blk_begin[c1 - c0] = nb;
    ap.total_blocks = nb;
    rp.total_blocks = rb;
    fp.partials = wpart;                                   // records: absolute indices
    ap.partials = xpart + pl.mp[c0].w_begin;               // exact-norm sums: one per block
    fp.xpartials = ap.partials;
    if (apply_op != kOpMuon && !have_partials && rp.nmat > 0) {
      NSHB_LAUNCH(NSHB_PROF_REDUCE, launch_reduce(rp, st));
    }
    fp.stage = 0;
    NSHB_LAUNCH(NSHB_PROF_FINALIZE, launch_apply_finalize(fp, st));
    if (apply_op == kOpNorms) continue;
    if (apply_op == kOpHyperball || apply_op == kOpBrake) {
      NSHB_LAUNCH(NSHB_PROF_EXACT, launch_exact_norm(ap, st));
      fp.stage = 1;
      NSHB_LAUNCH(NSHB_PROF_FINALIZE, launch_apply_finalize(fp, st));
    }
    NSHB_LAUNCH(NSHB_PROF_APPLY, launch_apply(ap, st));
  }
  return NSHB_OK;
}

NwProb nw_prob() {
  NwProb q;
  std::memset(&q, 0, sizeof(q));
  q.c32 = q.d32 = q.dhi = q.dlo = -1;
  q.kt = 4;                        // every product is 256 deep (one block column)
  return q;
}

// Launches the split-precision products of `probs` (in launches of kMaxNwProb).
nshb_status run_nw(NwParams &np, const std::vector<NwProb> &probs, cudaStream_t st, int reserve_pairs = 0) {
  for (size_t c0 = 0; c0 < probs.size(); c0 += kMaxNwProb) {
    const size_t c1 = std::min(probs.size(), c0 + (size_t)kMaxNwProb);
    int tiles = 0;
    for (size_t i = c0; i < c1; ++i) {
      NwProb q = probs[i];
      q.tile_begin = tiles;
      tiles += q.mt * q.nt;
      np.prob[i - c0] = q;
    }
    np.nprob = (int)(c1 - c0);
    np.total_tiles = tiles;
    NSHB_LAUNCH(NSHB_PROF_NEWTON, launch_newton_gemm(np, device_sms(), st, reserve_pairs));
  }
  return NSHB_OK;
}

// fp32 -> bf16 hi / lo panels for a list of regions (in launches of kMaxMats).
nshb_status run_split(const std::vector<SplitItem> &items, char *ws, cudaStream_t st) {
  for (size_t c0 = 0; c0 < items.size(); c0 += kMaxMats) {
    const size_t c1 = std::min(items.size(), c0 + (size_t)kMaxMats);
    SplitParams sp;
    std::memset(&sp, 0, sizeof(sp));
    sp.ws = ws;
    int nb = 0;
    for (size_t i = c0; i < c1; ++i) {
      SplitItem it = items[i];
      it.blk_begin = nb;
      nb += (it.prow / 64) * (it.pcol / 64);
      sp.item[i - c0] = it;
    }
    sp.n = (int)(c1 - c0);
    sp.total_blocks = nb;
    NSHB_LAUNCH(NSHB_PROF_NEWTON, launch_split(sp, st));
  }
  return NSHB_OK;
}

// P = U (Z Z^T + lambda I)^-1 for every matrix; leaves P (fp32, m x n) at pl.r_off[i].
nshb_status run_newton_precond(const nshb_matrix *mats, const Plan &pl, const nshb_params *p, char *ws,
                               cudaStream_t st) {
  const int n = (int)pl.mp.size(), nz = (int)pl.zp.size();
  uint32_t *status = reinterpret_cast<uint32_t *>(ws);
  const long long limit = (p->debug_flags & 1u) ? kWaitLimitTest : kWaitLimit;
  // 1. momentum, U in fp32 row-major
  for (int c0 = 0; c0 < n; c0 += kMaxMats) {
    const int c1 = std::min(n, c0 + kMaxMats);
    MomentumParams mp;
    std::memset(&mp, 0, sizeof(mp));
    mp.ws = ws;
    mp.partials = reinterpret_cast<double *>(ws + pl.k1part_off);
    mp.status = status;
    mp.beta = p->beta;
    mp.nesterov = p->nesterov ? 1 : 0;
    mp.nmat = c1 - c0;
    int nb = 0;
    for (int i = c0; i < c1; ++i) {
      MatDesc d = make_desc(mats[i], pl.mp[i], i, 0, nb, false);
      d.flags = (d.flags & (kVec | kWF32)) | kURow;
      d.u_off = pl.r_off[i];
      mp.mats[i - c0] = d;
      nb += pl.mp[i].w_blocks;
    }
    mp.total_blocks = nb;
    NSHB_LAUNCH(NSHB_PROF_MOMENTUM, launch_momentum(mp, st));
  }
  // 2. S = Z Z^T on the tensor cores (fp32 out), its operands read straight from each Z
  for (int c0 = 0; c0 < nz; c0 += kMaxZMaps) {
    const int c1 = std::min(nz, c0 + kMaxZMaps);
    SyrkParams gp;
    std::memset(&gp, 0, sizeof(gp));
    gp.ws = ws;
    gp.status = status;
    gp.wait_limit = limit;
    gp.test_stall = 0;
    gp.mode = kGramF32;
    int tiles = 0, k = 0;
    for (int j = c0; j < c1; ++j) {
      const Plan::ZPlan &z = pl.zp[j];
      NSHB_CHECK_CUDA(encode_z_tensor_map(&gp.zmap[k], z.src, z.d, pl.n_tokens));
      GemmProb &q = gp.prob[k++];
      q.a_off = q.b_off = 0;
      q.c_off = q.d_off = z.s;
      q.c_lo = q.d_lo = -1;
      q.a_ph = q.b_ph = q.d_ph = (int)z.Dp;
      q.major = 0;
      q.bs = 0;
      q.w = nullptr;
      q.mt = (int)(z.Dp / 256);
      q.nt = (int)(z.Dp / 256);
      q.kt = (int)(pl.n_tokens / 64);
      q.batch = 1;
      const int cnt = gemm_tiles(kGramF32, q.mt, q.nt, 256, 256);
      q.tiles_per_batch = cnt;
      q.tile_begin = tiles;
      q.scale_idx = -1;
      tiles += cnt;
    }
    gp.nprob = k;
    gp.total_tiles = tiles;
    NSHB_CHECK_CUDA(encode_ws_tensor_map(&gp.tmap, ws, pl.total / 128 * 128));
    NSHB_LAUNCH(NSHB_PROF_NEWTON, launch_gemm_syrk(gp, device_sms(), st));
  }
  // 3. ridge (and a unit diagonal on the padding), then the operands of the first step as
  //    bf16 hi / lo panels: S's first column block and every U (with an fp32 copy padded to
  //    Mp x Dp, the running Y of the forward solve)
  for (int c0 = 0; c0 < nz; c0 += kMaxMats) {
    const int c1 = std::min(nz, c0 + kMaxMats);
    CholParams cp;
    std::memset(&cp, 0, sizeof(cp));
    cp.ws = ws;
    cp.status = status;
    cp.ridge_rel = p->ridge_rel;
    cp.n = c1 - c0;
    for (int j = c0; j < c1; ++j) {
      cp.s_off[j - c0] = pl.zp[j].s;
      cp.ld[j - c0] = (int)pl.zp[j].Dp;
      cp.d[j - c0] = (int)pl.zp[j].d;
    }
    NSHB_LAUNCH(NSHB_PROF_NEWTON, launch_ridge(cp, st));
  }
  {
    std::vector<SplitItem> items;
    for (auto &z : pl.zp) {
      SplitItem it;
      std::memset(&it, 0, sizeof(it));
      it.src32 = z.s;
      it.dst32 = -1;
      it.dhi = z.sh;
      it.dlo = z.sl;
      it.src_ld = (int)z.Dp;
      it.rows = it.prow = (int)z.Dp;
      it.cols = it.pcol = 256;
      it.d_ph = (int)z.Dp;
      items.push_back(it);
    }
    for (int i = 0; i < n; ++i) {
      const Plan::ZPlan &z = pl.zp[pl.zidx[i]];
      SplitItem it;
      std::memset(&it, 0, sizeof(it));
      it.src32 = pl.r_off[i];
      it.dst32 = pl.y32[i];
      it.dhi = pl.yh[i];
      it.dlo = pl.yl[i];
      it.src_ld = (int)pl.mp[i].n;
      it.dst_ld = (int)z.Dp;
      it.rows = (int)pl.mp[i].m;
      it.cols = (int)pl.mp[i].n;
      it.prow = (int)pl.mpad[i];
      it.pcol = (int)z.Dp;
      it.d_ph = (int)pl.mpad[i];
      items.push_back(it);
    }
    nshb_status e = run_split(items, ws, st);
    if (e != NSHB_OK) return e;
  }
  NwParams np;
  std::memset(&np, 0, sizeof(np));
  np.ws = ws;
  np.status = status;
  np.wait_limit = limit;
  NSHB_CHECK_CUDA(encode_ws_tensor_map(&np.tmap, ws, pl.total / 128 * 128));
  int64_t dmax = 0;
  for (auto &z : pl.zp) dmax = std::max(dmax, z.Dp);
  const int nb = (int)(dmax / 256);
  // 4. forward, left-looking by block columns of 256.  Block column k of S is brought up to
  //    date by products over every earlier column of L, T = S[k0:, k] - L[k0:, :k] L[k, :k]^T;
  //    its diagonal block is factored and inverted (D_k); the panel L[k1:, k] = T[k1:] D_k^T
  //    follows.  The rows of every U are carried along the same way: V = U[:, k] - Y[:, :k]
  //    L[k, :k]^T, Y[:, k] = V D_k^T.  Every fp32 element of S and U is read and written about
  //    once (a right-looking order rewrites the whole trailing matrix at every step).  Only the
  //    last term of T, from column k - 1, waits for the previous panel: the rest of column k's
  //    update runs beside step k - 1's diagonal blocks, with the update of U's column (both
  //    need only earlier columns; that launch starts without waiting and waits for the
  //    diagonal blocks at its end).  Launches per step: T's last term (k > 0), diagonal blocks,
  //    [V and the next column's early terms], panel.
  auto run_diag = [&](int k) -> nshb_status {
    const int64_t k0 = 256LL * k;
    for (int c0 = 0; c0 < nz; c0 += kMaxMats) {
      const int c1 = std::min(nz, c0 + kMaxMats);
      DiagParams dp;
      std::memset(&dp, 0, sizeof(dp));
      dp.ws = ws;
      dp.status = status;
      dp.k = k;
      for (int j = c0; j < c1; ++j) {
        if (pl.zp[j].Dp <= k0) continue;
        dp.s32[dp.n] = pl.zp[j].s;
        dp.dhi[dp.n] = pl.zp[j].dh;
        dp.dlo[dp.n] = pl.zp[j].dl;
        dp.ld[dp.n] = (int)pl.zp[j].Dp;
        dp.n++;
      }
      if (dp.n) NSHB_LAUNCH(NSHB_PROF_NEWTON, launch_potrf_diag(dp, st));
    }
    return NSHB_OK;
  };
  // 5. backward, P L = Y by block columns of 512 from the last, left-looking as well:
  //    W = Y[:, K] - P[:, K1:] L[K1:, K] (one product over every later column of P; only its
  //    hi / lo panels are kept, in place of Y[:, K]), then P[:, K] = W E_K with E_K the inverse
  //    of L's 512 x 512 diagonal block K (fp32 into the m x n buffer the momentum pass reads, and
  //    hi / lo panels of P).  E_K = [D_a 0; X D_b] for the 256-blocks a = 2j, b = 2j + 1, with
  //    X = -D_b L_ba D_a formed during the forward sweep; a last block of 256 has E = D.  A
  //    matrix whose layer input has G blocks of 512 runs 2G - 1 stages (solve G-1, column
  //    G-2, solve G-2, ..., solve 0); its stages start as soon as its forward sweep is over,
  //    one per launch, so the matrices of narrow layer inputs finish theirs inside the forward
  //    sweep of the wide ones (in the launches beside the diagonal blocks) and the rest
  //    continue after it.
  auto n_super = [&](const Plan::ZPlan &z) { return (int)((z.Dp / 256 + 1) / 2); };
  auto bwd_stage = [&](int i, int s, std::vector<NwProb> &out) {
    const Plan::ZPlan &z = pl.zp[pl.zidx[i]];
    const int G = n_super(z);
    const int jj = G - 1 - (s + 1) / 2;
    const int64_t K0 = 512LL * jj, wj = std::min<int64_t>(512, z.Dp - K0), K1 = K0 + wj;
    if (s % 2 == 1) {
      NwProb t = nw_prob();
      t.a_hi = pl.ph[i]; t.a_lo = pl.plo[i]; t.a_ph = (int)pl.mpad[i]; t.a_r0 = 0; t.a_k0 = (int)K1;
      t.b_hi = z.lh; t.b_lo = z.ll; t.b_ph = (int)z.Dp; t.b_r0 = (int)K0; t.b_k0 = (int)K1;
      t.kt = (int)((z.Dp - K1) / 64);
      t.flags = kNwBMn;
      t.c32 = pl.y32[i] + K0 * 4; t.ld32 = (int)z.Dp;
      t.m_valid = (int)pl.mpad[i]; t.n_valid = (int)wj;
      t.dhi = pl.yh[i]; t.dlo = pl.yl[i]; t.d_ph = (int)pl.mpad[i]; t.d_r0 = 0; t.d_c0 = (int)K0;
      t.mt = (int)(pl.mpad[i] / 256); t.nt = (int)(wj / 256);
      out.push_back(t);
    } else {
      const int d = (int)pl.mp[i].n, m = (int)pl.mp[i].m;
      NwProb q = nw_prob();
      q.a_hi = pl.yh[i]; q.a_lo = pl.yl[i]; q.a_ph = (int)pl.mpad[i]; q.a_r0 = 0; q.a_k0 = (int)K0;
      q.b_hi = z.dh; q.b_lo = z.dl; q.b_ph = (int)z.Dp; q.b_r0 = 0; q.b_k0 = (int)K0;
      q.kt = (int)(wj / 64);
      q.flags = kNwBMn;
      q.d32 = pl.r_off[i] + K0 * 4; q.ld32 = d; q.m_valid = m; q.n_valid = (int)std::max<int64_t>(0, d - K0);
      q.dhi = pl.ph[i]; q.dlo = pl.plo[i]; q.d_ph = (int)pl.mpad[i]; q.d_r0 = 0; q.d_c0 = (int)K0;
      q.mt = (int)(pl.mpad[i] / 256); q.nt = (int)(wj / 256);
      out.push_back(q);
    }
  };
  // A matrix whose forward sweep ends well before the last step (g + 2G - 2 < nb - 1) may start
  // its stages up to R - 1 steps late.  The delays are chosen greedily, largest matrices first,
  // to even out the work of the launches beside the diagonal blocks: each launch's estimated
  // cost (per 256 x 256 tile, its k panels times the three products plus an epilogue's worth)
  // starts from the early terms of the next S column and the update of U's column, and every
  // matrix takes the delay that leaves the largest launch its stages touch the smallest.
  auto tile_cost = [](int64_t tiles, int64_t kt) { return (double)tiles * (double)(3 * kt + 24); };
  std::vector<double> load(nb > 0 ? nb : 1, 0.0);
  for (int k = 1; k < nb; ++k) {
    const int64_t k0 = 256LL * k, k1 = k0 + 256;
    for (auto &z : pl.zp)
      if (z.Dp > k1) load[k] += tile_cost((z.Dp - k1) / 256, k0 / 64);
    for (int i = 0; i < n; ++i)
      if (pl.zp[pl.zidx[i]].Dp > k0) load[k] += tile_cost(pl.mpad[i] / 256, k0 / 64);
  }
  auto stage_cost = [&](int i, int s) {
    const Plan::ZPlan &z = pl.zp[pl.zidx[i]];
    const int G = n_super(z), jj = G - 1 - (s + 1) / 2;
    const int64_t K0 = 512LL * jj, wj = std::min<int64_t>(512, z.Dp - K0), K1 = K0 + wj;
    const int64_t tiles = (pl.mpad[i] / 256) * (wj / 256);
    return s % 2 == 1 ? tile_cost(tiles, (z.Dp - K1) / 64) : tile_cost(tiles, wj / 64);
  };
  std::vector<int> bwd_off(n, 0), order;
  for (int i = 0; i < n; ++i) {
    const Plan::ZPlan &z = pl.zp[pl.zidx[i]];
    const int g = (int)(z.Dp / 256);
    if (nb - g - 2 * n_super(z) + 2 > 1) order.push_back(i);
  }
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return pl.mpad[a] > pl.mpad[b]; });
  for (int i : order) {
    const Plan::ZPlan &z = pl.zp[pl.zidx[i]];
    const int g = (int)(z.Dp / 256), ns = 2 * n_super(z) - 1;
    const int R = std::min(8, nb - g - ns + 1);
    int best = 0;
    double best_peak = 0.0;
    for (int o = 0; o < R; ++o) {
      double peak = 0.0;
      for (int st = 0; st < ns; ++st) peak = std::max(peak, load[g + o + st] + stage_cost(i, st));
      if (o == 0 || peak < best_peak) { best = o; best_peak = peak; }
    }
    bwd_off[i] = best;
    for (int st = 0; st < ns; ++st) load[g + best + st] += stage_cost(i, st);
  }
  // stage k - g - off of every matrix whose g block columns of 256 are done by step k
  // (0 <= k - g - off <= 2G - 2)
  auto bwd_stages = [&](int k, std::vector<NwProb> &out) {
    for (int i = 0; i < n; ++i) {
      const Plan::ZPlan &z = pl.zp[pl.zidx[i]];
      const int g = (int)(z.Dp / 256), s = k - g - bwd_off[i];
      if (s >= 0 && s <= 2 * n_super(z) - 2) bwd_stage(i, s, out);
    }
  };
  for (int k = 0; k < nb; ++k) {
    const int64_t k0 = 256LL * k, k1 = k0 + 256;
    const int dcol = (k & 1) * 256;       // column of D_k in the stack of 512-wide inverses
    std::vector<NwProb> col_s, col_u, panel;
    int ndiag = 0;
    for (auto &z : pl.zp) {
      if (z.Dp <= k0) continue;
      ++ndiag;
      if (k & 1) {
        // the lower-left block X = -D_k L[k0:k1, k-1] D_{k-1} of the inverse of the 512 x 512
        // diagonal block (k-1, k), in two products over the columns 0 .. 255 of block row k of
        // the stack: T = L[k0:k1, k-1] D_{k-1} beside the diagonal blocks (both factors are
        // done), then X = -D_k T after them (one tile, so T is read before X replaces it)
        NwProb t = nw_prob();
        t.a_hi = z.lh; t.a_lo = z.ll; t.a_ph = (int)z.Dp; t.a_r0 = (int)k0; t.a_k0 = (int)(k0 - 256);
        t.b_hi = z.dh; t.b_lo = z.dl; t.b_ph = (int)z.Dp; t.b_r0 = 0; t.b_k0 = (int)(k0 - 256);
        t.flags = kNwBMn;
        t.dhi = z.dh; t.dlo = z.dl; t.d_ph = (int)z.Dp; t.d_r0 = (int)k0; t.d_c0 = 0;
        t.mt = 1; t.nt = 1;
        col_u.push_back(t);
        NwProb x = nw_prob();
        x.a_hi = z.dh; x.a_lo = z.dl; x.a_ph = (int)z.Dp; x.a_r0 = (int)k0; x.a_k0 = 256;
        x.b_hi = z.dh; x.b_lo = z.dl; x.b_ph = (int)z.Dp; x.b_r0 = 0; x.b_k0 = (int)k0;
        x.flags = kNwBMn | kNwNeg;
        x.dhi = z.dh; x.dlo = z.dl; x.d_ph = (int)z.Dp; x.d_r0 = (int)k0; x.d_c0 = 0;
        x.mt = 1; x.nt = 1;
        panel.push_back(x);
      }
      if (k > 0) {
        // T = S[k0:, k] - L[k0:, k-1] L[k0:k1, k-1]^T, the last term of the column's update
        // (the others were applied beside the previous step's diagonal blocks), fp32 in place
        // and as hi / lo panels
        NwProb t = nw_prob();
        t.a_hi = z.lh; t.a_lo = z.ll; t.a_ph = (int)z.Dp; t.a_r0 = (int)k0; t.a_k0 = (int)(k0 - 256);
        t.b_hi = z.lh; t.b_lo = z.ll; t.b_ph = (int)z.Dp; t.b_r0 = (int)k0; t.b_k0 = (int)(k0 - 256);
        t.c32 = t.d32 = z.s + (k0 * z.Dp + k0) * 4; t.ld32 = (int)z.Dp;
        t.m_valid = (int)(z.Dp - k0); t.n_valid = 256;
        t.dhi = z.sh; t.dlo = z.sl; t.d_ph = (int)z.Dp; t.d_r0 = (int)k0; t.d_c0 = (int)k0;
        t.mt = (int)((z.Dp - k0) / 256); t.nt = 1;
        col_s.push_back(t);
      }
      if (z.Dp <= k1) continue;
      if (k > 0) {
        // beside the diagonal blocks: S[k1:, k + 1] -= L[k1:, :k] L[k1:k1+256, :k]^T (fp32 only)
        NwProb t = nw_prob();
        t.a_hi = z.lh; t.a_lo = z.ll; t.a_ph = (int)z.Dp; t.a_r0 = (int)k1; t.a_k0 = 0;
        t.b_hi = z.lh; t.b_lo = z.ll; t.b_ph = (int)z.Dp; t.b_r0 = (int)k1; t.b_k0 = 0;
        t.kt = (int)(k0 / 64);
        t.c32 = t.d32 = z.s + (k1 * z.Dp + k1) * 4; t.ld32 = (int)z.Dp;
        t.m_valid = (int)(z.Dp - k1); t.n_valid = 256;
        t.mt = (int)((z.Dp - k1) / 256); t.nt = 1;
        col_u.push_back(t);
      }
      // L[k1:, k] = T[k1:] D_k^T
      NwProb q = nw_prob();
      q.a_hi = z.sh; q.a_lo = z.sl; q.a_ph = (int)z.Dp; q.a_r0 = (int)k1; q.a_k0 = (int)k0;
      q.b_hi = z.dh; q.b_lo = z.dl; q.b_ph = (int)z.Dp; q.b_r0 = (int)k0; q.b_k0 = dcol;
      q.dhi = z.lh; q.dlo = z.ll; q.d_ph = (int)z.Dp; q.d_r0 = (int)k1; q.d_c0 = (int)k0;
      q.mt = (int)((z.Dp - k1) / 256); q.nt = 1;
      panel.push_back(q);
    }
    for (int i = 0; i < n; ++i) {
      const Plan::ZPlan &z = pl.zp[pl.zidx[i]];
      if (z.Dp <= k0) continue;
      if (k > 0) {
        // V = U[:, k] - Y[:, :k] L[k0:k1, :k]^T, fp32 in place and as hi / lo panels
        NwProb t = nw_prob();
        t.a_hi = pl.yh[i]; t.a_lo = pl.yl[i]; t.a_ph = (int)pl.mpad[i]; t.a_r0 = 0; t.a_k0 = 0;
        t.b_hi = z.lh; t.b_lo = z.ll; t.b_ph = (int)z.Dp; t.b_r0 = (int)k0; t.b_k0 = 0;
        t.kt = (int)(k0 / 64);
        t.c32 = t.d32 = pl.y32[i] + k0 * 4; t.ld32 = (int)z.Dp;
        t.m_valid = (int)pl.mpad[i]; t.n_valid = 256;
        t.dhi = pl.yh[i]; t.dlo = pl.yl[i]; t.d_ph = (int)pl.mpad[i]; t.d_r0 = 0; t.d_c0 = (int)k0;
        t.mt = (int)(pl.mpad[i] / 256); t.nt = 1;
        col_u.push_back(t);
      }
      // Y[:, k] = V D_k^T
      NwProb q = nw_prob();
      q.a_hi = pl.yh[i]; q.a_lo = pl.yl[i]; q.a_ph = (int)pl.mpad[i]; q.a_r0 = 0; q.a_k0 = (int)k0;
      q.b_hi = z.dh; q.b_lo = z.dl; q.b_ph = (int)z.Dp; q.b_r0 = (int)k0; q.b_k0 = dcol;
      q.d32 = pl.y32[i] + k0 * 4; q.ld32 = (int)z.Dp; q.m_valid = (int)pl.mpad[i]; q.n_valid = 256;
      q.dhi = pl.yh[i]; q.dlo = pl.yl[i]; q.d_ph = (int)pl.mpad[i]; q.d_r0 = 0; q.d_c0 = (int)k0;
      q.mt = (int)(pl.mpad[i] / 256); q.nt = 1;
      panel.push_back(q);
    }
    nshb_status e = run_nw(np, col_s, st);
    if (e != NSHB_OK) return e;
    e = run_diag(k);
    if (e != NSHB_OK) return e;
    // beside the diagonal blocks: one SM per block is taken, and a few pairs more for the SMs
    // that the pairing leaves single.  When that would take more than a quarter of the pairs,
    // nothing is reserved: the pairs that find no SM start when the diagonal blocks end, which
    // costs what running the two in turn costs.
    int reserve = (ndiag + 1) / 2 + 4;
    if (4 * reserve > device_sms() / 2) reserve = 0;
    bwd_stages(k, col_u);                 // backward stages of the matrices already done
    np.late_wait = 1;
    e = run_nw(np, col_u, st, reserve);
    np.late_wait = 0;
    if (e != NSHB_OK) return e;
    e = run_nw(np, panel, st);
    if (e != NSHB_OK) return e;
  }
  // the remaining backward stages, one launch per stage index
  int k_end = 0;
  for (int i = 0; i < n; ++i) {
    const Plan::ZPlan &z = pl.zp[pl.zidx[i]];
    k_end = std::max(k_end, (int)(z.Dp / 256) + bwd_off[i] + 2 * n_super(z) - 2);
  }
  for (int k = nb; k <= k_end; ++k) {
    std::vector<NwProb> stage;
    bwd_stages(k, stage);
    nshb_status e = run_nw(np, stage, st);
    if (e != NSHB_OK) return e;
  }
  return NSHB_OK;
}

nshb_status check_ws(const Plan &pl, void *ws, size_t ws_bytes) {
  if (!ws) return NSHB_ERR_NULL;
  if ((uintptr_t)ws % kAlign != 0) return NSHB_ERR_WORKSPACE;
  if (ws_bytes < pl.total) return NSHB_ERR_WORKSPACE;
  return NSHB_OK;
}

// keep_status: a later chunk of one chunked call, which adds its flags to the status word
// the earlier chunks set (only the exact-pass counter starts again from zero).
nshb_status do_step(const nshb_matrix *mats, int n_mats, const nshb_params *p, int op, void *ws, size_t ws_bytes,
                    cudaStream_t st, bool keep_status = false) {
  Plan pl;
  nshb_status e = plan_step(mats, n_mats, p, op, pl);
  if (e != NSHB_OK) return e;
  if (n_mats == 0) return NSHB_OK;
  e = check_ws(pl, ws, ws_bytes);
  if (e != NSHB_OK) return e;
  char *w = static_cast<char *>(ws);
  if (keep_status)
    NSHB_CHECK_CUDA(cudaMemsetAsync(w + sizeof(uint32_t), 0, sizeof(uint32_t), st));  // exact-pass counter
  else
    NSHB_CHECK_CUDA(cudaMemsetAsync(w, 0, 2 * sizeof(uint32_t), st));  // status word, exact-pass counter
  e = run_momentum(mats, pl, p, w, st);
  if (e != NSHB_OK) return e;
  std::vector<int64_t> o_off;
  e = run_ns(mats, pl, p, w, st, o_off);
  if (e != NSHB_OK) return e;
  const int aop = op == NSHB_OP_MUON              ? kOpMuon
                  : op == NSHB_OP_RADIAL_BRAKE    ? kOpBrake
                  : op == NSHB_OP_RELATIVE_UPDATE ? kOpRelative
                                                  : kOpHyperball;
  return run_apply(mats, pl, p, aop, w, st, o_off, nullptr);
}

// AdamH: no NS.  Per matrix the Adam direction U~ in the layout the apply kernels read as O
// (bf16 panels of round_up(rows, 64) rows, or fp32 row-major), block partials and the
// per-matrix scalars.
nshb_status plan_adamh(const nshb_matrix *mats, int n_mats, float *const *V, const nshb_adam_params *a,
                       const nshb_params *p, Plan &pl) {
  if (!p || !a) return NSHB_ERR_NULL;
  if (n_mats < 0) return NSHB_ERR_SHAPE;
  if (n_mats > 0 && (!mats || !V)) return NSHB_ERR_NULL;
  if (!(a->beta1 >= 0.f && a->beta1 < 1.f) || !(a->beta2 >= 0.f && a->beta2 < 1.f)) return NSHB_ERR_PARAM;
  if (!(a->eps > 0.f) || !std::isfinite(a->eps) || a->step < 1) return NSHB_ERR_PARAM;
  if (!(p->hb_eps > 0.f) || !std::isfinite(p->hb_eps) || !std::isfinite(p->eta) || p->eta < 0.f)
    return NSHB_ERR_PARAM;
  if ((uintptr_t)p->rho % sizeof(float)) return NSHB_ERR_PARAM;
  pl.op = NSHB_OP_ADAMH;
  pl.mp.resize(n_mats);
  size_t off = kAlign;  // [0, 256): device status word
  pl.scal_off = off;
  off = align_up(off + sizeof(MatScalars) * (size_t)n_mats);
  pl.w_total = 0;
  for (int i = 0; i < n_mats; ++i) {
    const nshb_matrix &d = mats[i];
    MatPlan &m = pl.mp[i];
    const nshb_status ce = check_matrix(d, V[i], /*need_v=*/true);
    if (ce != NSHB_OK) return ce;
    const bool wf32 = d.w_dtype == NSHB_F32;
    const size_t esz = wf32 ? 4 : 2;
    const bool vec = ((uintptr_t)d.W % 16 == 0) && ((uintptr_t)d.G % 16 == 0) && ((uintptr_t)d.M % 16 == 0) &&
                     ((uintptr_t)V[i] % 16 == 0) && ((d.ld * esz) % 16 == 0) && ((d.ld * 4) % 16 == 0);
    m.m = d.rows;
    m.n = d.cols;
    m.ld = d.ld;
    m.flags = (vec ? kVec : 0) | (wf32 ? (kWF32 | kNsF32) : 0);   // never transposed
    m.Rp = round_up(m.m, kBlk);   // bf16 U~: panel height
    m.s = m.n;                    // fp32 U~: row stride
    m.w_blocks = (int)(((m.m + kBlk - 1) / kBlk) * ((m.n + kBlk - 1) / kBlk));
    m.w_begin = pl.w_total;
    pl.w_total += m.w_blocks;
    m.rec_begin = m.w_begin;      // adam_kernel writes one record per block
    m.rec_count = m.w_blocks;
  }
  pl.rec_total = pl.w_total;
  pl.wpart_off = off;
  off = align_up(off + 3 * sizeof(double) * (size_t)pl.w_total);
  pl.xpart_off = off;
  off = align_up(off + sizeof(double) * (size_t)pl.w_total);
  for (auto &m : pl.mp) {
    m.x0 = off;
    const size_t ub = (m.flags & kWF32) ? (size_t)m.m * m.n * 4 : (size_t)m.Rp * round_up(m.n, kBlk) * 2;
    off = align_up(off + ub);
  }
  pl.total = off;
  return NSHB_OK;
}

nshb_status run_adam(const nshb_matrix *mats, const Plan &pl, float *const *V, const nshb_adam_params *a,
                     char *ws, cudaStream_t st) {
  const int n = (int)pl.mp.size();
  double *wpart = reinterpret_cast<double *>(ws + pl.wpart_off);
  for (int c0 = 0; c0 < n; c0 += kMaxMats) {
    const int c1 = std::min(n, c0 + kMaxMats);
    AdamParams ap;
    std::memset(&ap, 0, sizeof(ap));
    ap.ws = ws;
    ap.partials = wpart + 3 * (int64_t)pl.mp[c0].w_begin;
    ap.status = reinterpret_cast<uint32_t *>(ws);
    ap.beta1 = a->beta1;
    ap.beta2 = a->beta2;
    ap.eps = a->eps;
    ap.bc1 = (float)(1.0 / (1.0 - std::pow((double)a->beta1, (double)a->step)));
    ap.bc2 = (float)(1.0 / (1.0 - std::pow((double)a->beta2, (double)a->step)));
    ap.nmat = c1 - c0;
    int nb = 0;
    for (int i = c0; i < c1; ++i) {
      ap.mats[i - c0] = make_desc(mats[i], pl.mp[i], i, pl.mp[i].x0, nb, false);
      ap.V[i - c0] = V[i];
      nb += pl.mp[i].w_blocks;
    }
    ap.total_blocks = nb;
    NSHB_LAUNCH(NSHB_PROF_ADAM, launch_adam(ap, st));
  }
  return NSHB_OK;
}

}  // namespace
}  // namespace nshb

namespace nshb {

nshb_status check_matrix(const nshb_matrix &d, const float *V, bool need_v, bool w_only) {
  if (d.rows <= 0 || d.cols <= 0 || d.ld < d.cols) return NSHB_ERR_SHAPE;
  if (d.rows > (1LL << 20) || d.cols > (1LL << 20) || d.ld > (1LL << 30)) return NSHB_ERR_UNSUPPORTED;
  if (!d.W) return NSHB_ERR_NULL;
  if (!w_only && (!d.G || !d.M || (need_v && !V))) return NSHB_ERR_NULL;
  if (d.w_dtype != NSHB_BF16 && d.w_dtype != NSHB_F32) return NSHB_ERR_DTYPE;
  const size_t esz = d.w_dtype == NSHB_F32 ? 4 : 2;
  if ((uintptr_t)d.W % esz) return NSHB_ERR_SHAPE;
  if (w_only) return NSHB_OK;
  if (d.O_out && ((uintptr_t)d.O_out % esz) != 0) return NSHB_ERR_SHAPE;
  if ((uintptr_t)d.G % esz || (uintptr_t)d.M % 4 || (uintptr_t)V % 4) return NSHB_ERR_SHAPE;
  return NSHB_OK;
}

void record_cuda_error(cudaError_t e) {
  g_last_cuda_error = (int)e;
  (void)cudaGetLastError();
}

}  // namespace nshb

using namespace nshb;

extern "C" {

nshb_status nshb_default_params(nshb_params *p) {
  if (!p) return NSHB_ERR_NULL;
  std::memset(p, 0, sizeof(*p));
  p->beta = 0.95f;
  p->nesterov = 1;
  p->ns_steps = 5;
  p->ns_precision = NSHB_BF16;
  p->coeffs = nullptr;
  p->ns_eps = 1e-7f;
  p->lr = 0.02f;
  p->weight_decay = 0.f;
  p->eta = 0.02f;
  p->rho = nullptr;
  p->hb_eps = 1e-8f;
  p->brake_out = 0.5f;
  p->brake_in = 1.0f;
  p->tile = 256;
  p->ridge_rel = 1e-3f;
  p->ns_compensated = 2;
  p->debug_flags = 0;
  return NSHB_OK;
}

nshb_status nshb_workspace_size(const nshb_matrix *mats, int32_t n_mats, const nshb_params *p, int32_t op,
                                const int64_t *z_rows, int32_t n_z, int64_t n_tokens, size_t *bytes) {
  if (!bytes) return NSHB_ERR_NULL;
  Plan pl;
  if (op == NSHB_OP_ADAMH) {
    // The moments' pointers do not change the size: plan with stand-ins for V.
    nshb_adam_params a;
    nshb_default_adam_params(&a);
    if (!p) return NSHB_ERR_NULL;
    std::vector<float *> vs((size_t)std::max(n_mats, 1), reinterpret_cast<float *>(uintptr_t(256)));
    nshb_status e = plan_adamh(mats, n_mats, vs.data(), &a, p, pl);
    if (e != NSHB_OK) return e;
    *bytes = pl.total;
    return NSHB_OK;
  }
  nshb_status e = plan_step(mats, n_mats, p, op, pl);
  if (e != NSHB_OK) return e;
  if (op == NSHB_OP_NEWTON_MUON && n_mats > 0) {
    e = plan_newton(mats, n_mats, nullptr, z_rows, n_z, n_tokens, pl);
    if (e != NSHB_OK) return e;
  }
  *bytes = pl.total;
  return NSHB_OK;
}

nshb_status muon_step(const nshb_matrix *mats, int32_t n_mats, const nshb_params *p, void *ws, size_t ws_bytes,
                      nshb_stream stream) {
  return do_step(mats, n_mats, p, NSHB_OP_MUON, ws, ws_bytes, (cudaStream_t)stream);
}

nshb_status relative_update_step(const nshb_matrix *mats, int32_t n_mats, const nshb_params *p, void *ws,
                                 size_t ws_bytes, nshb_stream stream) {
  return do_step(mats, n_mats, p, NSHB_OP_RELATIVE_UPDATE, ws, ws_bytes, (cudaStream_t)stream);
}

nshb_status nshb_default_adam_params(nshb_adam_params *a) {
  if (!a) return NSHB_ERR_NULL;
  a->beta1 = 0.9f;
  a->beta2 = 0.999f;
  a->eps = 1e-8f;
  a->step = 1;
  return NSHB_OK;
}

nshb_status adamh_step(const nshb_matrix *mats, int32_t n_mats, float *const *V, const nshb_adam_params *a,
                       const nshb_params *p, void *ws, size_t ws_bytes, nshb_stream stream) {
  Plan pl;
  nshb_status e = plan_adamh(mats, n_mats, V, a, p, pl);
  if (e != NSHB_OK) return e;
  if (n_mats == 0) return NSHB_OK;
  e = check_ws(pl, ws, ws_bytes);
  if (e != NSHB_OK) return e;
  char *w = static_cast<char *>(ws);
  cudaStream_t st = (cudaStream_t)stream;
  NSHB_CHECK_CUDA(cudaMemsetAsync(w, 0, 2 * sizeof(uint32_t), st));  // status word, exact-pass counter
  e = run_adam(mats, pl, V, a, w, st);
  if (e != NSHB_OK) return e;
  std::vector<int64_t> u_off(n_mats);
  for (int i = 0; i < n_mats; ++i) u_off[i] = pl.mp[i].x0;
  return run_apply(mats, pl, p, kOpHyperball, w, st, u_off, nullptr, /*have_partials=*/true);
}

nshb_status hyperball_step(const nshb_matrix *mats, int32_t n_mats, const nshb_params *p, void *ws,
                           size_t ws_bytes, nshb_stream stream) {
  return do_step(mats, n_mats, p, NSHB_OP_HYPERBALL, ws, ws_bytes, (cudaStream_t)stream);
}

nshb_status radial_brake_step(const nshb_matrix *mats, int32_t n_mats, const nshb_params *p, void *ws,
                              size_t ws_bytes, nshb_stream stream) {
  return do_step(mats, n_mats, p, NSHB_OP_RADIAL_BRAKE, ws, ws_bytes, (cudaStream_t)stream);
}

nshb_status himuon_step(const nshb_matrix *mats, int32_t n_mats, const nshb_params *p, void *ws, size_t ws_bytes,
                        nshb_stream stream) {
  return do_step(mats, n_mats, p, NSHB_OP_HIMUON, ws, ws_bytes, (cudaStream_t)stream);
}

nshb_status newton_muon_step(const nshb_matrix *mats, int32_t n_mats, const void *const *Z, const int64_t *z_rows,
                             int32_t n_z, int64_t n_tokens, const nshb_params *p, void *ws, size_t ws_bytes,
                             nshb_stream stream) {
  Plan pl;
  nshb_status e = plan_step(mats, n_mats, p, NSHB_OP_NEWTON_MUON, pl);
  if (e != NSHB_OK) return e;
  if (n_mats == 0) return NSHB_OK;
  if (!Z) return NSHB_ERR_NULL;
  e = plan_newton(mats, n_mats, Z, z_rows, n_z, n_tokens, pl);
  if (e != NSHB_OK) return e;
  e = check_ws(pl, ws, ws_bytes);
  if (e != NSHB_OK) return e;
  char *w = static_cast<char *>(ws);
  cudaStream_t st = (cudaStream_t)stream;
  NSHB_CHECK_CUDA(cudaMemsetAsync(w, 0, 2 * sizeof(uint32_t), st));  // status word, exact-pass counter
  e = run_newton_precond(mats, pl, p, w, st);
  if (e != NSHB_OK) return e;
  e = run_momentum(mats, pl, p, w, st, /*from_p=*/true);
  if (e != NSHB_OK) return e;
  std::vector<int64_t> o_off;
  e = run_ns(mats, pl, p, w, st, o_off);
  if (e != NSHB_OK) return e;
  return run_apply(mats, pl, p, kOpHyperball, w, st, o_off, nullptr);
}

static bool chunkable_op(int32_t op) {
  return op == NSHB_OP_MUON || op == NSHB_OP_HYPERBALL || op == NSHB_OP_RADIAL_BRAKE || op == NSHB_OP_HIMUON ||
         op == NSHB_OP_RELATIVE_UPDATE;
}

nshb_status nshb_workspace_size_min(const nshb_matrix *mats, int32_t n_mats, const nshb_params *p, int32_t op,
                                    size_t *bytes) {
  if (!bytes) return NSHB_ERR_NULL;
  if (!chunkable_op(op)) return NSHB_ERR_PARAM;
  size_t best = 0;
  for (int i = 0; i < n_mats; ++i) {
    Plan pl;
    const nshb_status e = plan_step(mats + i, 1, p, op, pl);
    if (e != NSHB_OK) return e;
    best = std::max(best, pl.total);
  }
  if (n_mats == 0) {
    Plan pl;
    const nshb_status e = plan_step(mats, 0, p, op, pl);
    if (e != NSHB_OK) return e;
  }
  *bytes = best;
  return NSHB_OK;
}

nshb_status nshb_step_chunked(int32_t op, const nshb_matrix *mats, int32_t n_mats, const nshb_params *p, void *ws,
                              size_t ws_bytes, nshb_stream stream, int32_t *n_chunks) {
  if (!chunkable_op(op)) return NSHB_ERR_PARAM;
  Plan all;
  nshb_status e = plan_step(mats, n_mats, p, op, all);   // validates every argument before any launch
  if (e != NSHB_OK) return e;
  if (!ws) return NSHB_ERR_NULL;
  if ((uintptr_t)ws % kAlign != 0) return NSHB_ERR_WORKSPACE;
  // Chunk boundaries first (host only), so that a workspace too small for some matrix
  // is reported before anything is queued.
  std::vector<int> starts;
  auto fits = [&](int i, int k) {
    Plan pl;
    return plan_step(mats + i, k, p, op, pl) == NSHB_OK && pl.total <= ws_bytes;
  };
  for (int i = 0; i < n_mats;) {
    if (!fits(i, 1)) return NSHB_ERR_WORKSPACE;
    int lo = 1, hi = 1;                        // largest k with fits(i, k): doubling, then bisection
    while (i + hi < n_mats && fits(i, std::min(2 * hi, n_mats - i))) hi = std::min(2 * hi, n_mats - i);
    if (i + hi < n_mats) {
      lo = hi;
      int up = std::min(2 * hi, n_mats - i);   // fits(i, up) is false
      while (up - lo > 1) {
        const int mid = (lo + up) / 2;
        if (fits(i, mid)) lo = mid; else up = mid;
      }
      hi = lo;
    }
    starts.push_back(i);
    i += hi;
  }
  starts.push_back(n_mats);
  if (n_chunks) *n_chunks = (int32_t)starts.size() - 1;
  for (size_t c = 0; c + 1 < starts.size(); ++c) {
    const int i = starts[c], k = starts[c + 1] - starts[c];
    nshb_params pc = *p;
    if (p->rho) pc.rho = p->rho + i;           // the radii of this chunk's matrices
    e = do_step(mats + i, k, &pc, op, ws, ws_bytes, (cudaStream_t)stream, /*keep_status=*/c > 0);
    if (e != NSHB_OK) return e;
  }
  return NSHB_OK;
}

nshb_status nshb_fro_norms(const nshb_matrix *mats, int32_t n_mats, float *out, void *ws, size_t ws_bytes,
                           nshb_stream stream) {
  if (!out && n_mats > 0) return NSHB_ERR_NULL;
  if ((uintptr_t)out % sizeof(float)) return NSHB_ERR_SHAPE;
  nshb_params p;
  nshb_default_params(&p);
  Plan pl;
  nshb_status e = plan_step(mats, n_mats, &p, NSHB_OP_MUON, pl);
  if (e != NSHB_OK) return e;
  if (n_mats == 0) return NSHB_OK;
  e = check_ws(pl, ws, ws_bytes);
  if (e != NSHB_OK) return e;
  char *w = static_cast<char *>(ws);
  cudaStream_t st = (cudaStream_t)stream;
  NSHB_CHECK_CUDA(cudaMemsetAsync(w, 0, 2 * sizeof(uint32_t), st));  // status word, exact-pass counter
  std::vector<int64_t> none;
  return run_apply(mats, pl, &p, kOpNorms, w, st, none, out);
}

nshb_status nshb_device_status(const void *ws, nshb_stream stream, uint32_t *flags) {
  if (!ws || !flags) return NSHB_ERR_NULL;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaStreamSynchronize(st) != cudaSuccess) {
    (void)cudaGetLastError();
    return NSHB_ERR_CUDA;
  }
  uint32_t v = 0;
  if (cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) {
    (void)cudaGetLastError();
    return NSHB_ERR_CUDA;
  }
  *flags = v;
  return NSHB_OK;
}

const char *nshb_status_string(int32_t s) {
  switch (s) {
    case NSHB_OK: return "NSHB_OK";
    case NSHB_ERR_NULL: return "NSHB_ERR_NULL";
    case NSHB_ERR_SHAPE: return "NSHB_ERR_SHAPE";
    case NSHB_ERR_DTYPE: return "NSHB_ERR_DTYPE";
    case NSHB_ERR_PARAM: return "NSHB_ERR_PARAM";
    case NSHB_ERR_WORKSPACE: return "NSHB_ERR_WORKSPACE";
    case NSHB_ERR_CUDA: return "NSHB_ERR_CUDA";
    case NSHB_ERR_DEVICE_TIMEOUT: return "NSHB_ERR_DEVICE_TIMEOUT";
    case NSHB_ERR_NONFINITE: return "NSHB_ERR_NONFINITE";
    case NSHB_ERR_ZERO_NORM: return "NSHB_ERR_ZERO_NORM";
    case NSHB_ERR_UNSUPPORTED: return "NSHB_ERR_UNSUPPORTED";
    default: return "NSHB_ERR_UNKNOWN";
  }
}

nshb_status nshb_profile_enable(int32_t on) {
  Profiler &p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  p.on = on != 0;
  return NSHB_OK;
}

nshb_status nshb_profile_read(int32_t n_kinds, float *ms, int32_t *launches) {
  if (n_kinds < 0 || (n_kinds > 0 && (!ms || !launches))) return NSHB_ERR_NULL;
  Profiler &p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  for (int k = 0; k < n_kinds; ++k) {
    ms[k] = 0.f;
    launches[k] = 0;
  }
  nshb_status st = NSHB_OK;
  for (auto &r : p.recs) {
    float t = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) {
      (void)cudaGetLastError();
      st = NSHB_ERR_CUDA;
    }
    if (r.kind >= 0 && r.kind < n_kinds) {
      ms[r.kind] += t;
      launches[r.kind] += 1;
    }
    p.pool.push_back(r.a);
    p.pool.push_back(r.b);
  }
  p.recs.clear();
  return st;
}

int32_t nshb_last_cuda_error(void) { return g_last_cuda_error; }

int32_t nshb_version(void) { return 200; }   // 0.2.0: AdamH, RelativeUpdate, chunked steps, alignment checks

}  // extern "C"
