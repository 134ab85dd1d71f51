// HBM-bound kernels of the optimizer step.
//
//  momentum_kernel   M <- beta M + (1-beta) G ; U = (1-beta) G + beta M (Nesterov) ;
//                    writes U straight into the NS operand layout (bf16 panels, transposed
//                    for tall matrices, or fp32 row-major) and one ||U||^2 partial per
//                    64x64 block.  ("Muon: the orthogonalized optimizer explained",
//                    momentum recap note and Muon.step code.)
//  norm_finalize     ||U||^2 per matrix (or per Hierarchical-Muon tile) in fixed order,
//                    scale = 1 / (||U|| + eps)  (newton_schulz5 normalisation).
//  reduce_kernel     ||O||^2, <W, O>, ||W||^2 partials per block.
//  apply_finalize    per-matrix coefficients of the update rule (Hyperball Method,
//                    PR #224 RadialBrake, Muon.step) in fp64.
//  exact_norm        ||W - t O||^2 computed element-wise for the rare matrices whose
//                    closed form cancels (an update that nearly equals W).
//  apply_kernel      W <- alpha W + beta O, one read of W and O, one write of W.
//
// Every kernel works on 64x64 blocks with 256 threads: thread t owns row t/4 and the 16
// columns 16*(t%4) .. +15 of its block.  Reductions use fixed-order trees in fp64.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cmath>

#include "nshb_device.cuh"
#include "nshb_internal.h"

namespace nshb {
namespace {

constexpr int kThreads = 256;

template <typename P>
__device__ __forceinline__ int find_mat(const P &p, int blk) {
  int lo = 0, hi = p.nmat - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (p.mats[mid].blk_begin <= blk) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Origin (W coordinates) of local block `lb` of a matrix.  Tiled matrices enumerate
// their blocks tile by tile so that the partials of one tile are contiguous.
__device__ __forceinline__ void block_origin(const MatDesc &d, int lb, int &r0, int &c0) {
  if (d.flags & kTileMajor) {
    const int tb = d.ph / kBlk;
    const int per = tb * tb;
    const int tl = lb / per, l = lb % per;
    r0 = (tl / d.tiles_c) * d.ph + (l / tb) * kBlk;
    c0 = (tl % d.tiles_c) * d.ph + (l % tb) * kBlk;
  } else {
    const int bc = d.pc / kBlk;
    r0 = (lb / bc) * kBlk;
    c0 = (lb % bc) * kBlk;
  }
}

// Load 16 consecutive W-or-G values of row i starting at column j (bounds-checked).
__device__ __forceinline__ void load16(const void *base, int64_t ld, int i, int j, int m, int n, bool f32,
                                       bool vec, float (&v)[16]) {
  if (i >= m) {
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] = 0.f;
    return;
  }
  if (f32) {
    const float *row = static_cast<const float *>(base) + (int64_t)i * ld;
    if (vec && j + 15 < n) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float4 t = *reinterpret_cast<const float4 *>(row + j + 4 * q);
        v[4 * q] = t.x; v[4 * q + 1] = t.y; v[4 * q + 2] = t.z; v[4 * q + 3] = t.w;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) v[e] = (j + e < n) ? row[j + e] : 0.f;
    }
  } else {
    const __nv_bfloat16 *row = static_cast<const __nv_bfloat16 *>(base) + (int64_t)i * ld;
    if (vec && j + 15 < n) {
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint4 t = *reinterpret_cast<const uint4 *>(row + j + 8 * q);
        v[8 * q + 0] = bf16lo(t.x); v[8 * q + 1] = bf16hi(t.x);
        v[8 * q + 2] = bf16lo(t.y); v[8 * q + 3] = bf16hi(t.y);
        v[8 * q + 4] = bf16lo(t.z); v[8 * q + 5] = bf16hi(t.z);
        v[8 * q + 6] = bf16lo(t.w); v[8 * q + 7] = bf16hi(t.w);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) v[e] = (j + e < n) ? __bfloat162float(row[j + e]) : 0.f;
    }
  }
}

__device__ __forceinline__ void store16(void *base, int64_t ld, int i, int j, int m, int n, bool f32, bool vec,
                                        const float (&v)[16]) {
  if (i >= m) return;
  if (f32) {
    float *row = static_cast<float *>(base) + (int64_t)i * ld;
    if (vec && j + 15 < n) {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<float4 *>(row + j + 4 * q) = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e)
        if (j + e < n) row[j + e] = v[e];
    }
  } else {
    __nv_bfloat16 *row = static_cast<__nv_bfloat16 *>(base) + (int64_t)i * ld;
    if (vec && j + 15 < n) {
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint4 t;
        t.x = pack_bf16(v[8 * q + 0], v[8 * q + 1]);
        t.y = pack_bf16(v[8 * q + 2], v[8 * q + 3]);
        t.z = pack_bf16(v[8 * q + 4], v[8 * q + 5]);
        t.w = pack_bf16(v[8 * q + 6], v[8 * q + 7]);
        *reinterpret_cast<uint4 *>(row + j + 8 * q) = t;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e)
        if (j + e < n) row[j + e] = __float2bfloat16_rn(v[e]);
    }
  }
}

// Momentum buffer: always fp32.
__device__ __forceinline__ void loadM(const float *M, int64_t ld, int i, int j, int m, int n, bool vec,
                                      float (&v)[16]) {
  load16(M, ld, i, j, m, n, true, vec, v);
}

// Address of X element block for the tiled layout: tile (tr, tc) is a T x T panel matrix.
__device__ __forceinline__ char *tile_base(char *xbase, const MatDesc &d, int r, int c) {
  const int64_t T = d.ph;
  const int64_t tl = (int64_t)(r / T) * d.tiles_c + (c / T);
  return xbase + tl * T * T * 2;
}

// Writes 16 values of X row xr, columns xc..xc+15, into the NS operand storage.
__device__ __forceinline__ void store_x16(char *xbase, const MatDesc &d, int xr, int xc, const float (&v)[16]) {
  if (d.flags & kNsF32) {
    // fp32 row-major, unpadded: r x s with row stride ph.
    const bool tall = d.flags & kTall;
    const int rr = tall ? d.n : d.m, ss = tall ? d.m : d.n;
    if (xr >= rr) return;
    float *row = reinterpret_cast<float *>(xbase) + (int64_t)xr * d.ph;
#pragma unroll
    for (int e = 0; e < 16; ++e)
      if (xc + e < ss) row[xc + e] = v[e];
    return;
  }
  char *base = xbase;
  int64_t ph = d.ph;
  int lr = xr, lc = xc;
  if (d.flags & kTiled) {
    base = tile_base(xbase, d, xr, xc);
    lr = xr % d.ph;
    lc = xc % d.ph;
  }
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    uint4 t;
    t.x = pack_bf16(v[8 * q + 0], v[8 * q + 1]);
    t.y = pack_bf16(v[8 * q + 2], v[8 * q + 3]);
    t.z = pack_bf16(v[8 * q + 4], v[8 * q + 5]);
    t.w = pack_bf16(v[8 * q + 6], v[8 * q + 7]);
    *reinterpret_cast<uint4 *>(base + panel_chunk_off(lr, lc + 8 * q, ph)) = t;
  }
}

// Reads 16 values of X row xr, columns xc..xc+15 (zero outside an fp32 X).
__device__ __forceinline__ void load_x16(const char *xbase, const MatDesc &d, int xr, int xc, float (&v)[16]) {
  if (d.flags & kNsF32) {
    const bool tall = d.flags & kTall;
    const int rr = tall ? d.n : d.m, ss = tall ? d.m : d.n;
    const float *row = reinterpret_cast<const float *>(xbase) + (int64_t)xr * d.ph;
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] = (xr < rr && xc + e < ss) ? row[xc + e] : 0.f;
    return;
  }
  const char *base = xbase;
  int lr = xr, lc = xc;
  if (d.flags & kTiled) {
    base = tile_base(const_cast<char *>(xbase), d, xr, xc);
    lr = xr % d.ph;
    lc = xc % d.ph;
  }
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    uint4 t = *reinterpret_cast<const uint4 *>(base + panel_chunk_off(lr, lc + 8 * q, d.ph));
    v[8 * q + 0] = bf16lo(t.x); v[8 * q + 1] = bf16hi(t.x);
    v[8 * q + 2] = bf16lo(t.y); v[8 * q + 3] = bf16hi(t.y);
    v[8 * q + 4] = bf16lo(t.z); v[8 * q + 5] = bf16hi(t.z);
    v[8 * q + 6] = bf16lo(t.w); v[8 * q + 7] = bf16hi(t.w);
  }
}

// ------------------------------------------------------------------------- momentum
__global__ void __launch_bounds__(kThreads) momentum_kernel(const __grid_constant__ MomentumParams p) {
  __shared__ float sT[kBlk][kBlk + 1];   // transpose staging (tall matrices), hi then lo
  __shared__ double red[kThreads / 32];
  const int blk = blockIdx.x;
  const MatDesc &d = p.mats[find_mat(p, blk)];
  int r0, c0;
  block_origin(d, blk - d.blk_begin, r0, c0);
  const int t = threadIdx.x, rr = t >> 2, cg = (t & 3) * 16;
  const int i = r0 + rr, j = c0 + cg;
  const bool f32 = d.flags & kWF32, vec = d.flags & kVec;
  const bool round_bf16 = !(d.flags & (kNsF32 | kURow));
  const bool lo_part = round_bf16 && d.xlo_off >= 0;

  float g[16], mm[16], u[16], ul[16];
  const bool from_p = d.flags & kFromP;
  if (from_p) {
    // U is given (the Newton-Muon preconditioned update), fp32 row-major m x n.
    load16(p.ws + d.u_off, d.n, i, j, d.m, d.n, true, (d.n % 4) == 0, g);
  } else {
    load16(d.G, d.ld, i, j, d.m, d.n, f32, vec, g);
    loadM(d.M, d.ld, i, j, d.m, d.n, vec, mm);
  }
  const float beta = p.beta, omb = 1.0f - p.beta;
  float acc = 0.f;
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    float uf;
    if (from_p) {
      uf = g[e];
    } else {
      const float mnew = fmaf(beta, mm[e], omb * g[e]);
      mm[e] = mnew;
      uf = p.nesterov ? fmaf(omb, g[e], beta * mnew) : mnew;
    }
    if (!(i < d.m && j + e < d.n)) uf = 0.f;
    const float uh = round_bf16 ? bf16_round(uf) : uf;
    u[e] = uh;
    ul[e] = uf - uh;                       // exact in fp32; stored as bf16 when kept
    const float un = lo_part ? uf : uh;    // the norm of what the first iteration reads
    acc = fmaf(un, un, acc);
  }
  if (!from_p) store16(d.M, d.ld, i, j, d.m, d.n, true, vec, mm);
  if (d.flags & kURow) {
    // Newton-Muon: U goes to an fp32 row-major buffer for the triangular solves.
    store16(p.ws + d.u_off, d.n, i, j, d.m, d.n, true, (d.n % 4) == 0, u);
    return;
  }

  char *xbase = p.ws + d.x_off;
  char *lbase = lo_part ? p.ws + d.xlo_off : nullptr;
  if (d.flags & kTall && !(d.flags & kTiled)) {
    // X = U^T: stage the block and write it transposed (hi, then lo through the same tile).
#pragma unroll
    for (int e = 0; e < 16; ++e) sT[rr][cg + e] = u[e];
    __syncthreads();
    float v[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] = sT[cg + e][rr];
    store_x16(xbase, d, c0 + rr, r0 + cg, v);
    if (lo_part) {
      __syncthreads();
#pragma unroll
      for (int e = 0; e < 16; ++e) sT[rr][cg + e] = ul[e];
      __syncthreads();
#pragma unroll
      for (int e = 0; e < 16; ++e) v[e] = sT[cg + e][rr];
      store_x16(lbase, d, c0 + rr, r0 + cg, v);
    }
  } else {
    store_x16(xbase, d, i, j, u);
    if (lo_part) store_x16(lbase, d, i, j, ul);
  }

  double s[1] = {(double)acc};
  block_sum<1>(s, red);
  if (t == 0) p.partials[blk] = s[0];
}

// ---------------------------------------------------------------- norm finalize
__global__ void norm_finalize_kernel(const __grid_constant__ NormFinParams p, int nseg_total) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= nseg_total) return;
  int lo = 0, hi = p.nmat - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (p.seg_begin[mid] <= warp) lo = mid; else hi = mid - 1;
  }
  const int bps = p.bps[lo];
  const double *src = p.partials + p.blk_begin[lo] + (int64_t)(warp - p.seg_begin[lo]) * bps;
  double s = 0.0;
  for (int k = lane; k < bps; k += 32) s += src[k];
  s = warp_sum(s);
  if (lane == 0) {
    if (!isfinite(s)) set_status(p.status, 0x2u);
    p.nus[warp] = s;
    p.scales[warp] = (float)(1.0 / (sqrt(s) + (double)p.ns_eps));
  }
}

// This thread's 16 O values of W row r0 + t/4, columns c0 + 16 (t%4) .. +15.  Matrices
// whose NS ran on the transpose go through the shared tile sO; the others read their
// 16 values straight from the panel layout (two 16-byte chunks, no block barrier).
__device__ __forceinline__ void load_o_block(const ApplyParams &p, const MatDesc &d, int r0, int c0,
                                             float (&sO)[kBlk][kBlk + 1]);
__device__ __forceinline__ void load_o16(const ApplyParams &p, const MatDesc &d, int r0, int c0,
                                         float (&sO)[kBlk][kBlk + 1], float (&o)[16]) {
  const int t = threadIdx.x, rr = t >> 2, cg = (t & 3) * 16;
  const bool tr = (d.flags & kTall) && !(d.flags & kTiled);
  if (!tr) {
    load_x16(p.ws + d.o_off, d, r0 + rr, c0 + cg, o);
    return;
  }
  load_o_block(p, d, r0, c0, sO);
#pragma unroll
  for (int e = 0; e < 16; ++e) o[e] = sO[rr][cg + e];
}

// Loads the O block of W block (r0, c0) into sO[w_row][w_col] (zero outside W).
__device__ __forceinline__ void load_o_block(const ApplyParams &p, const MatDesc &d, int r0, int c0,
                                             float (&sO)[kBlk][kBlk + 1]) {
  const int t = threadIdx.x, rr = t >> 2, cg = (t & 3) * 16;
  const char *xbase = p.ws + d.o_off;
  float v[16];
  const bool tr = (d.flags & kTall) && !(d.flags & kTiled);
  if (tr) {
    load_x16(xbase, d, c0 + rr, r0 + cg, v);          // X row = W column
#pragma unroll
    for (int e = 0; e < 16; ++e) sO[cg + e][rr] = v[e];
  } else {
    load_x16(xbase, d, r0 + rr, c0 + cg, v);
#pragma unroll
    for (int e = 0; e < 16; ++e) sO[rr][cg + e] = v[e];
  }
  __syncthreads();
}

// ------------------------------------------------------------ (W, O) reductions
__global__ void __launch_bounds__(kThreads) reduce_kernel(const __grid_constant__ ApplyParams p) {
  __shared__ float sO[kBlk][kBlk + 1];
  __shared__ double red[3 * kThreads / 32];
  const int blk = blockIdx.x;
  const MatDesc &d = p.mats[find_mat(p, blk)];
  int r0, c0;
  block_origin(d, blk - d.blk_begin, r0, c0);
  const int t = threadIdx.x, rr = t >> 2, cg = (t & 3) * 16;
  const int i = r0 + rr, j = c0 + cg;
  float w[16];
  load16(d.W, d.ld, i, j, d.m, d.n, d.flags & kWF32, d.flags & kVec, w);
  float om = 0.f, de = 0.f, pi = 0.f;
  if (p.op != kOpNorms) {
    float ov[16];
    load_o16(p, d, r0, c0, sO, ov);
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float o = (i < d.m && j + e < d.n) ? ov[e] : 0.f;
      om = fmaf(o, o, om);
      de = fmaf(w[e], o, de);
    }
  }
#pragma unroll
  for (int e = 0; e < 16; ++e) pi = fmaf(w[e], w[e], pi);
  double s[3] = {(double)om, (double)de, (double)pi};
  block_sum<3>(s, red);
  if (t == 0) {
    p.partials[3 * (int64_t)blk + 0] = s[0];
    p.partials[3 * (int64_t)blk + 1] = s[1];
    p.partials[3 * (int64_t)blk + 2] = s[2];
  }
}

// ||W - t O||^2 for matrices flagged need_exact; a persistent grid walks their blocks.
__global__ void __launch_bounds__(kThreads) exact_norm_kernel(const __grid_constant__ ApplyParams p) {
  __shared__ float sO[kBlk][kBlk + 1];
  __shared__ double red[kThreads / 32];
  const int t = threadIdx.x, rr = t >> 2, cg = (t & 3) * 16;
  if (*(volatile uint32_t *)(p.status + 1) == 0) return;  // no matrix of this call needs it
  for (int mi = 0; mi < p.nmat; ++mi) {
    const MatDesc &d = p.mats[mi];
    const MatScalars &sc = p.scal[d.mat];
    if (!sc.need_exact) continue;
    const int nb = (mi + 1 < p.nmat ? p.mats[mi + 1].blk_begin : p.total_blocks) - d.blk_begin;
    const float tt = (float)sc.t;
    for (int lb = blockIdx.x; lb < nb; lb += gridDim.x) {
      int r0, c0;
      block_origin(d, lb, r0, c0);
      const int i = r0 + rr, j = c0 + cg;
      float w[16];
      load16(d.W, d.ld, i, j, d.m, d.n, d.flags & kWF32, d.flags & kVec, w);
      float ov[16];
      load_o16(p, d, r0, c0, sO, ov);
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float o = (i < d.m && j + e < d.n) ? ov[e] : 0.f;
        const float v = fmaf(-tt, o, w[e]);
        acc = fmaf(v, v, acc);
      }
      double s[1] = {(double)acc};
      block_sum<1>(s, red);
      if (t == 0) p.partials[d.blk_begin + lb] = s[0];
    }
  }
}

// --------------------------------------------------------------- apply finalize
__device__ void hyperball_coeffs(MatScalars &s, double q, double rho, double hb_eps, double pi, uint32_t *status) {
  if (q >= hb_eps) {
    s.alpha = (float)(rho / q);
    s.beta = (float)(-rho * s.t / q);
  } else {
    // ||W - eta U_hat|| is a numerical zero: keep W on its sphere, skip the step.
    set_status(status, 0x1u);
    const double nw = sqrt(pi);
    if (nw >= hb_eps) {
      s.alpha = (float)(rho / nw);
      s.beta = 0.f;
    } else {
      set_status(status, 0x8u);
      s.alpha = 1.f;
      s.beta = 0.f;
    }
  }
}

__device__ void brake_coeffs(MatScalars &s, double vv, double pi, const ApplyFinParams &p) {
  const double nn = sqrt(fmax(vv, 0.0)), np = sqrt(pi);
  if (nn < (double)p.hb_eps) {
    s.alpha = 1.f;
    s.beta = (float)(-s.t);
    return;
  }
  const double delta = nn - np;
  const double sf = delta > 0.0 ? (double)p.brake_out : (double)p.brake_in;
  const double f = (np + sf * delta) / nn;
  s.alpha = (float)f;
  s.beta = (float)(-f * s.t);
}

// One warp per matrix: the lanes sum the block partials in a fixed order, lane 0 derives
// the coefficients.
__global__ void apply_finalize_kernel(const __grid_constant__ ApplyFinParams p) {
  const int k = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (k >= p.nmat) return;
  MatScalars &s = p.scal[p.mat[k]];
  const int m = p.m[k], n = p.n[k];
  const double sshape = sqrt(fmax(1.0, (double)m / (double)n));
  if (p.op == kOpMuon) {
    if (lane == 0) {
      s.alpha = (float)(1.0 - (double)p.lr * (double)p.weight_decay);
      s.beta = (float)(-(double)p.lr * sshape);
      s.need_exact = 0;
    }
    return;
  }
  double om = 0.0, de = 0.0, pi = 0.0, ex = 0.0;
  if (p.stage == 0) {
    for (int b = p.blk_begin[k] + lane; b < p.blk_begin[k + 1]; b += 32) {
      om += p.partials[3 * (int64_t)b];
      de += p.partials[3 * (int64_t)b + 1];
      pi += p.partials[3 * (int64_t)b + 2];
    }
    om = warp_sum(om);
    de = warp_sum(de);
    pi = warp_sum(pi);
  } else if (s.need_exact) {
    for (int b = p.blk_begin[k] + lane; b < p.blk_begin[k + 1]; b += 32) ex += p.partials[b];
    ex = warp_sum(ex);
  }
  if (lane != 0) return;
  if (p.stage == 0) {
    s.omega = om; s.delta = de; s.pi = pi;
    s.need_exact = 0;
    if (p.op == kOpNorms) {
      p.norms_out[p.mat[k]] = (float)sqrt(pi);
      if (!isfinite(pi)) set_status(p.status, 0x2u);
      return;
    }
    if (!isfinite(om) || !isfinite(de) || !isfinite(pi)) {
      set_status(p.status, 0x2u);
      s.alpha = 1.f; s.beta = 0.f;
      return;
    }
    if (p.op == kOpHyperball) {
      const double nO = fmax(sqrt(om), (double)p.hb_eps);
      s.t = (double)p.eta / nO;
    } else {
      s.t = (double)p.lr * sshape;
    }
    const double tw = s.t * s.t * om;
    const double vv = pi - 2.0 * s.t * de + tw;
    // Below 1% of (||W||^2 + ||tO||^2) the closed form has lost about two digits of the
    // fp32-accumulated partials; recompute ||W - tO||^2 element-wise instead.
    if (vv < 1e-2 * (pi + tw)) {
      s.need_exact = 1;
      atomicAdd(p.status + 1, 1u);   // tells the exact-norm pass that it has work
      return;
    }
    s.vv = vv;
  } else {
    if (!s.need_exact) return;
    s.vv = ex;
    s.need_exact = 0;
  }
  if (p.op == kOpHyperball) {
    double rho = p.rho ? (double)p.rho[p.mat[k]] : 0.0;
    if (!(rho > 0.0)) {
      rho = sqrt(s.pi);
      if (rho < (double)p.hb_eps) {
        set_status(p.status, 0x8u);
        s.alpha = 1.f; s.beta = 0.f;
        return;
      }
    }
    hyperball_coeffs(s, sqrt(fmax(s.vv, 0.0)), rho, (double)p.hb_eps, s.pi, p.status);
  } else {
    brake_coeffs(s, s.vv, s.pi, p);
  }
}

// ------------------------------------------------------------------------ apply
__global__ void __launch_bounds__(kThreads) apply_kernel(const __grid_constant__ ApplyParams p) {
  __shared__ float sO[kBlk][kBlk + 1];
  const int blk = blockIdx.x;
  const MatDesc &d = p.mats[find_mat(p, blk)];
  int r0, c0;
  block_origin(d, blk - d.blk_begin, r0, c0);
  const int t = threadIdx.x, rr = t >> 2, cg = (t & 3) * 16;
  const int i = r0 + rr, j = c0 + cg;
  const bool f32 = d.flags & kWF32, vec = d.flags & kVec;
  float o[16];
  load_o16(p, d, r0, c0, sO, o);
  if (d.O_out) {
    const bool vo = ((uintptr_t)d.O_out % 16 == 0) && (d.n % (f32 ? 4 : 8) == 0);
    store16(d.O_out, d.n, i, j, d.m, d.n, f32, vo, o);
  }
  const MatScalars &s = p.scal[d.mat];
  const float a = s.alpha, b = s.beta;
  if (a == 1.f && b == 0.f) return;
  float w[16];
  load16(d.W, d.ld, i, j, d.m, d.n, f32, vec, w);
#pragma unroll
  for (int e = 0; e < 16; ++e) w[e] = fmaf(a, w[e], b * o[e]);
  store16(d.W, d.ld, i, j, d.m, d.n, f32, vec, w);
}

}  // namespace

cudaError_t launch_momentum(const MomentumParams &p, cudaStream_t s) {
  if (p.total_blocks > 0) momentum_kernel<<<p.total_blocks, kThreads, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_norm_finalize(const NormFinParams &p, int nseg_total, cudaStream_t s) {
  if (nseg_total > 0) norm_finalize_kernel<<<(nseg_total + 7) / 8, 256, 0, s>>>(p, nseg_total);
  return cudaGetLastError();
}
cudaError_t launch_reduce(const ApplyParams &p, cudaStream_t s) {
  if (p.total_blocks > 0) reduce_kernel<<<p.total_blocks, kThreads, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_exact_norm(const ApplyParams &p, cudaStream_t s) {
  if (p.total_blocks > 0) exact_norm_kernel<<<296, kThreads, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_apply_finalize(const ApplyFinParams &p, cudaStream_t s) {
  if (p.nmat > 0) apply_finalize_kernel<<<(p.nmat + 3) / 4, 128, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_apply(const ApplyParams &p, cudaStream_t s) {
  if (p.total_blocks > 0) apply_kernel<<<p.total_blocks, kThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace nshb
