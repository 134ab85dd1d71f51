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
// The work unit is a 64x64 block; thread t of 256 owns the 8 consecutive columns
// 8 (t%8) .. +7 of the block rows t/8 and t/8 + 32, so one warp access covers four whole
// 128-byte bf16 row segments (or four 128-byte panel rows of X).  The streaming kernels
// are persistent: a grid of (SMs x resident CTAs) walks the block list with a stride of
// the grid size, and every CTA issues the loads of its next block before it processes the
// current one, so loads stay in flight through the block's arithmetic, its stores and its
// reduction.  Partial sums are still one per block (fixed-order trees in fp64), so the
// results do not depend on the grid size.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cmath>

#include "nshb_device.cuh"
#include "nshb_internal.h"

namespace nshb {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
static_assert(kWarps == kK1PartsPerBlock, "one ||U||^2 partial per warp of a momentum block");

template <typename P>
__device__ __forceinline__ int find_mat(const P &p, int blk) {
  int lo = 0, hi = p.nmat - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (p.mats[mid].blk_begin <= blk) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// The block list is walked in increasing order, so the owning matrix only moves forward.
template <typename P>
__device__ __forceinline__ int advance_mat(const P &p, int mi, int blk) {
  while (mi + 1 < p.nmat && p.mats[mi + 1].blk_begin <= blk) ++mi;
  return mi;
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

// Eight values of one row as loaded from memory: bf16 pairs in q[0..3], or fp32 bit
// patterns in q[0..7].  Kept raw so that a prefetch does not wait for its data.
struct Raw8 {
  uint32_t q[8];
};

__device__ __forceinline__ void raw_zero(Raw8 &r) {
#pragma unroll
  for (int e = 0; e < 8; ++e) r.q[e] = 0u;
}

// Row i, columns j..j+7 of a row-major bf16 or fp32 matrix (zero outside m x n).
__device__ __forceinline__ void raw_load8(const void *base, int64_t ld, int i, int j, int m, int n, bool f32,
                                          bool vec, Raw8 &r) {
  if (i >= m || j >= n) {
    raw_zero(r);
    return;
  }
  if (f32) {
    const float *row = static_cast<const float *>(base) + (int64_t)i * ld + j;
    if (vec && j + 7 < n) {
      const uint4 a = *reinterpret_cast<const uint4 *>(row);
      const uint4 b = *reinterpret_cast<const uint4 *>(row + 4);
      r.q[0] = a.x; r.q[1] = a.y; r.q[2] = a.z; r.q[3] = a.w;
      r.q[4] = b.x; r.q[5] = b.y; r.q[6] = b.z; r.q[7] = b.w;
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) r.q[e] = (j + e < n) ? __float_as_uint(row[e]) : 0u;
    }
  } else {
    const unsigned short *row = static_cast<const unsigned short *>(base) + (int64_t)i * ld + j;
    if (vec && j + 7 < n) {
      const uint4 a = *reinterpret_cast<const uint4 *>(row);
      r.q[0] = a.x; r.q[1] = a.y; r.q[2] = a.z; r.q[3] = a.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t lo = (j + 2 * e < n) ? row[2 * e] : 0u;
        const uint32_t hi = (j + 2 * e + 1 < n) ? row[2 * e + 1] : 0u;
        r.q[e] = lo | (hi << 16);
      }
    }
  }
}

__device__ __forceinline__ void raw_cvt8(const Raw8 &r, bool f32, float (&v)[8]) {
  if (f32) {
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(r.q[e]);
  } else {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[2 * e] = bf16lo(r.q[e]);
      v[2 * e + 1] = bf16hi(r.q[e]);
    }
  }
}

// Row i, columns j..j+7 of a row-major bf16 or fp32 matrix (bounds-checked).
__device__ __forceinline__ void store8(void *base, int64_t ld, int i, int j, int m, int n, bool f32, bool vec,
                                       const float (&v)[8]) {
  if (i >= m || j >= n) return;
  if (f32) {
    float *row = static_cast<float *>(base) + (int64_t)i * ld + j;
    if (vec && j + 7 < n) {
      *reinterpret_cast<float4 *>(row) = make_float4(v[0], v[1], v[2], v[3]);
      *reinterpret_cast<float4 *>(row + 4) = make_float4(v[4], v[5], v[6], v[7]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (j + e < n) row[e] = v[e];
    }
  } else {
    __nv_bfloat16 *row = static_cast<__nv_bfloat16 *>(base) + (int64_t)i * ld + j;
    if (vec && j + 7 < n) {
      uint4 t;
      t.x = pack_bf16(v[0], v[1]);
      t.y = pack_bf16(v[2], v[3]);
      t.z = pack_bf16(v[4], v[5]);
      t.w = pack_bf16(v[6], v[7]);
      *reinterpret_cast<uint4 *>(row) = t;
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (j + e < n) row[e] = __float2bfloat16_rn(v[e]);
    }
  }
}

// Byte offset (from xbase) of the 16-byte chunk holding X row xr, columns xc..xc+7 of a
// bf16 X (panel layout, or a grid of T x T panel tiles when tiled: tile (tr, tc), a T x T
// panel matrix, is tile tr * tiles_c + tc).  T (= ph) is 128, 256 or 512, so the tile and
// the position in it come from shifts and masks rather than divisions.
__device__ __forceinline__ const char *x_chunk(const char *xbase, const MatDesc &d, int xr, int xc) {
  if (d.flags & kTiled) {
    const int lg = __ffs(d.ph) - 1, mask = d.ph - 1;
    const int64_t tl = (int64_t)(xr >> lg) * d.tiles_c + (xc >> lg);
    return xbase + (tl << (2 * lg + 1)) + panel_chunk_off(xr & mask, xc & mask, d.ph);
  }
  return xbase + panel_chunk_off(xr, xc, d.ph);
}

// fp32 X (kNsF32): unpadded r x s, row stride ph.
__device__ __forceinline__ void xf32_dims(const MatDesc &d, int &rr, int &ss) {
  const bool tall = d.flags & kTall;
  rr = tall ? d.n : d.m;
  ss = tall ? d.m : d.n;
}

// Writes X row xr, columns xc..xc+7 into the NS operand storage.
__device__ __forceinline__ void x_store8(char *xbase, const MatDesc &d, int xr, int xc, const float (&v)[8],
                                         bool allow_f32) {
  if (allow_f32 && (d.flags & kNsF32)) {
    int rr, ss;
    xf32_dims(d, rr, ss);
    if (xr >= rr) return;
    float *row = reinterpret_cast<float *>(xbase) + (int64_t)xr * d.ph;
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (xc + e < ss) row[xc + e] = v[e];
    return;
  }
  uint4 t;
  t.x = pack_bf16(v[0], v[1]);
  t.y = pack_bf16(v[2], v[3]);
  t.z = pack_bf16(v[4], v[5]);
  t.w = pack_bf16(v[6], v[7]);
  *reinterpret_cast<uint4 *>(const_cast<char *>(x_chunk(xbase, d, xr, xc))) = t;
}

// Reads X row xr, columns xc..xc+7 raw (bf16 chunk, or fp32 values zero outside X).
__device__ __forceinline__ void x_load8(const char *xbase, const MatDesc &d, int xr, int xc, Raw8 &r,
                                        bool allow_f32) {
  if (allow_f32 && (d.flags & kNsF32)) {
    int rr, ss;
    xf32_dims(d, rr, ss);
    const float *row = reinterpret_cast<const float *>(xbase) + (int64_t)xr * d.ph;
#pragma unroll
    for (int e = 0; e < 8; ++e) r.q[e] = (xr < rr && xc + e < ss) ? __float_as_uint(row[xc + e]) : 0u;
    return;
  }
  const uint4 a = *reinterpret_cast<const uint4 *>(x_chunk(xbase, d, xr, xc));
  r.q[0] = a.x; r.q[1] = a.y; r.q[2] = a.z; r.q[3] = a.w;
}

// Fixed-order sum over the CTA of NV per-thread fp32 partials; thread 0 gets the totals
// in fp64.  Lanes combine in fp32 (five tree levels on top of each thread's own partial,
// which already sums 16 terms in fp32), warps in fp64.  `red` holds two buffers used
// alternately (`parity`), so that back-to-back calls need one barrier each: a buffer is
// rewritten only after the barrier of the call in between.
template <int NV>
__device__ __forceinline__ void cta_sum(const float (&v)[NV], double (&out)[NV], double (*red)[kWarps * NV],
                                        int parity) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float w[NV];
#pragma unroll
  for (int k = 0; k < NV; ++k) w[k] = warp_sum(v[k]);
  if (lane == 0) {
#pragma unroll
    for (int k = 0; k < NV; ++k) red[parity][warp * NV + k] = (double)w[k];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      double t = 0.0;
#pragma unroll
      for (int q = 0; q < kWarps; ++q) t += red[parity][q * NV + k];
      out[k] = t;
    }
  }
}

// True when the 64x64 block at (r0, c0) lies inside the m x n matrix.
__device__ __forceinline__ bool full_block(const MatDesc &d, int r0, int c0) {
  return r0 + kBlk <= d.m && c0 + kBlk <= d.n;
}

// ------------------------------------------------------------------------- momentum
// Inputs of one block as loaded: G (or the given U) and M for the thread's two rows.
struct MomIn {
  Raw8 g[2], m[2];
};

template <bool F32>
__device__ __forceinline__ void momentum_load(const MomentumParams &p, const MatDesc &d, int r0, int c0,
                                              MomIn &in) {
  const int rq = threadIdx.x >> 3, cq = (threadIdx.x & 7) * 8;
  const bool vec = d.flags & kVec;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int i = r0 + rq + 32 * h, j = c0 + cq;
    if (F32 && (d.flags & kFromP)) {
      // U is given (the Newton-Muon preconditioned update), fp32 row-major m x n.
      raw_load8(p.ws + d.u_off, d.n, i, j, d.m, d.n, true, (d.n % 4) == 0, in.g[h]);
      raw_zero(in.m[h]);
    } else {
      raw_load8(d.G, d.ld, i, j, d.m, d.n, F32 && (d.flags & kWF32), vec, in.g[h]);
      raw_load8(d.M, d.ld, i, j, d.m, d.n, true, vec, in.m[h]);
    }
  }
}

// One 64x64 block: momentum update, U into the NS operand storage, ||U||^2 partial.
template <bool F32>
__device__ __forceinline__ void momentum_block(const MomentumParams &p, const MatDesc &d, int cblk, int cr0,
                                               int cc0, const MomIn &in, float (&sT)[2][kBlk][kBlk + 1]) {
  const int rq = threadIdx.x >> 3, cq = (threadIdx.x & 7) * 8;
  const bool f32 = F32 && (d.flags & kWF32), vec = d.flags & kVec;
  const bool from_p = F32 && (d.flags & kFromP);
  const bool urow = F32 && (d.flags & kURow);
  const bool round_bf16 = !F32 || !(d.flags & (kNsF32 | kURow));
  const bool lo_part = round_bf16 && d.xlo_off >= 0;
  const bool tr = F32 && (d.flags & kTall) && (d.flags & kNsF32);   // the fp32 chain takes U^T
  char *xbase = p.ws + d.x_off;
  char *lbase = lo_part ? p.ws + d.xlo_off : nullptr;
  const float beta = p.beta, omb = 1.0f - p.beta;
  const bool full = full_block(d, cr0, cc0);
  float acc = 0.f;
  // Every thread has finished reading the previous block's transpose staging (tr is the
  // same for the whole CTA, so the barrier is uniform).
  if (tr && !urow) __syncthreads();
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int i = cr0 + rq + 32 * h, j = cc0 + cq;
    float g[8], mm[8], u[8], ul[8];
    raw_cvt8(in.g[h], f32 || from_p, g);
    raw_cvt8(in.m[h], true, mm);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float uf;
      if (from_p) {
        uf = g[e];
      } else {
        const float mnew = fmaf(beta, mm[e], omb * g[e]);
        mm[e] = mnew;
        uf = p.nesterov ? fmaf(omb, g[e], beta * mnew) : mnew;
      }
      if (!full && !(i < d.m && j + e < d.n)) uf = 0.f;
      const float uh = round_bf16 ? bf16_round(uf) : uf;
      u[e] = uh;
      ul[e] = uf - uh;                       // exact in fp32; stored as bf16 when kept
      const float un = lo_part ? uf : uh;    // the norm of what the first iteration reads
      acc = fmaf(un, un, acc);
    }
    if (!from_p) store8(d.M, d.ld, i, j, d.m, d.n, true, vec, mm);
    if (urow) {
      // Newton-Muon: U goes to an fp32 row-major buffer for the triangular solves.
      store8(p.ws + d.u_off, d.n, i, j, d.m, d.n, true, (d.n % 4) == 0, u);
    } else if (tr) {
      // X = U^T: stage hi and lo parts; the previous readers of sT finished before the
      // last cta_sum barrier.
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        sT[0][rq + 32 * h][cq + e] = u[e];
        if (lo_part) sT[1][rq + 32 * h][cq + e] = ul[e];
      }
    } else if (!(d.flags & kNoX)) {
      x_store8(xbase, d, i, j, u, F32);
      if (lo_part) x_store8(lbase, d, i, j, ul, F32);
    }
  }
  if (!urow) {
    if (tr) {
      __syncthreads();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = sT[0][cq + e][rq + 32 * h];
        x_store8(xbase, d, cc0 + rq + 32 * h, cr0 + cq, v, F32);
        if (lo_part) {
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] = sT[1][cq + e][rq + 32 * h];
          x_store8(lbase, d, cc0 + rq + 32 * h, cr0 + cq, v, F32);
        }
      }
    }
    // one partial per warp (fixed order within the warp), no block-wide barrier
    const float w = warp_sum(acc);
    if ((threadIdx.x & 31) == 0) p.partials[(int64_t)kWarps * cblk + (threadIdx.x >> 5)] = (double)w;
  }
}

// The inputs of the next two blocks (bf16 instance; one for fp32) are prefetched into
// registers while the current one is processed, so loads stay in flight through the block's
// arithmetic and stores even when a power-capped SM clock stretches them (two CTAs per SM;
// 12 % faster than one block ahead with three CTAs, and 8 % under the 1 kW cap).
template <bool F32>
__global__ void __launch_bounds__(kThreads, 2) momentum_kernel(const __grid_constant__ MomentumParams p) {
  constexpr bool kTwoAhead = !F32;          // the fp32 instance has no registers for a second block
  pdl_trigger();
  pdl_wait();
  __shared__ float sT[2][kBlk][kBlk + 1];   // transpose staging (tall matrices): hi, lo
  int blk = blockIdx.x;
  if (blk >= p.total_blocks) return;
  int mi = find_mat(p, blk);
  int r0, c0;
  block_origin(p.mats[mi], blk - p.mats[mi].blk_begin, r0, c0);
  MomIn n1, n2;
  momentum_load<F32>(p, p.mats[mi], r0, c0, n1);
  const int ahead = kTwoAhead ? 2 : 1;
  int blk2 = blk + gridDim.x, mi2 = mi, r2 = 0, c2 = 0;
  if (kTwoAhead && blk2 < p.total_blocks) {
    mi2 = advance_mat(p, mi, blk2);
    block_origin(p.mats[mi2], blk2 - p.mats[mi2].blk_begin, r2, c2);
    momentum_load<F32>(p, p.mats[mi2], r2, c2, n2);
  }
  for (;;) {
    const MomIn in = n1;
    const int cblk = blk, cr0 = r0, cc0 = c0;
    const MatDesc &d = p.mats[mi];
    if (kTwoAhead) {
      n1 = n2;
      blk = blk2; mi = mi2; r0 = r2; c0 = c2;
    } else {
      blk += gridDim.x;
      if (blk < p.total_blocks) {
        mi = advance_mat(p, mi, blk);
        block_origin(p.mats[mi], blk - p.mats[mi].blk_begin, r0, c0);
        momentum_load<F32>(p, p.mats[mi], r0, c0, n1);
      }
    }
    blk2 = blk + (ahead - 1) * gridDim.x;
    if (kTwoAhead && blk2 < p.total_blocks) {
      mi2 = advance_mat(p, mi, blk2);
      block_origin(p.mats[mi2], blk2 - p.mats[mi2].blk_begin, r2, c2);
      momentum_load<F32>(p, p.mats[mi2], r2, c2, n2);
    }
    momentum_block<F32>(p, d, cblk, cr0, cc0, in, sT);
    if (blk >= p.total_blocks) break;
  }
}

// ---------------------------------------------------------------- norm finalize
__global__ void norm_finalize_kernel(const __grid_constant__ NormFinParams p, int nseg_total) {
  pdl_trigger();
  pdl_wait();
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

// ------------------------------------------------------------ (W, O) streaming input
// W and O of one block as loaded.  O is read in X coordinates: for a matrix whose NS ran
// on the transpose, the thread loads X rows c0 + t/8 (+32) = W columns and turns the
// block around in shared memory when it processes it.
struct WoIn {
  Raw8 w[2], o[2];
};

// Only the fp32 chain runs on the transpose of a tall matrix; the bf16 chain keeps U's orientation.
__device__ __forceinline__ bool o_transposed(const MatDesc &d) { return (d.flags & kTall) && (d.flags & kNsF32); }

template <bool F32>
__device__ __forceinline__ void wo_load(const ApplyParams &p, const MatDesc &d, int r0, int c0, bool want_o,
                                        WoIn &in) {
  const int rq = threadIdx.x >> 3, cq = (threadIdx.x & 7) * 8;
  const bool tr = F32 && o_transposed(d);
  const char *xbase = p.ws + d.o_off;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    raw_load8(d.W, d.ld, r0 + rq + 32 * h, c0 + cq, d.m, d.n, F32 && (d.flags & kWF32), d.flags & kVec, in.w[h]);
    if (want_o) {
      if (tr) x_load8(xbase, d, c0 + rq + 32 * h, r0 + cq, in.o[h], F32);
      else x_load8(xbase, d, r0 + rq + 32 * h, c0 + cq, in.o[h], F32);
    }
  }
}

// The thread's O values in W coordinates (rows r0 + t/8 (+32), columns c0 + 8 (t%8) ..),
// zero outside W.  Transposed blocks go through sO and end with a barrier, after which
// sO may be rewritten.
template <bool F32>
__device__ __forceinline__ void wo_values(const MatDesc &d, int r0, int c0, const WoIn &in,
                                          float (&sO)[kBlk][kBlk + 1], float (&w)[2][8], float (&o)[2][8]) {
  const int rq = threadIdx.x >> 3, cq = (threadIdx.x & 7) * 8;
  const bool of32 = F32 && (d.flags & kNsF32);
#pragma unroll
  for (int h = 0; h < 2; ++h) raw_cvt8(in.w[h], F32 && (d.flags & kWF32), w[h]);
  if (F32 && o_transposed(d)) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float v[8];
      raw_cvt8(in.o[h], of32, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) sO[cq + e][rq + 32 * h] = v[e];
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int e = 0; e < 8; ++e) o[h][e] = sO[rq + 32 * h][cq + e];
    __syncthreads();
  } else {
#pragma unroll
    for (int h = 0; h < 2; ++h) raw_cvt8(in.o[h], of32, o[h]);
  }
  if (!full_block(d, r0, c0)) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = r0 + rq + 32 * h, j = c0 + cq;
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (!(i < d.m && j + e < d.n)) o[h][e] = 0.f;
    }
  }
}

// ------------------------------------------------------------ (W, O) reductions
template <bool F32>
__device__ __forceinline__ void reduce_block(const ApplyParams &p, const MatDesc &d, int cblk, int cr0, int cc0,
                                             const WoIn &in, float (&sO)[kBlk][kBlk + 1], double (*red)[3 * kWarps],
                                             int &nred) {
  float w[2][8], o[2][8];
  float om = 0.f, de = 0.f, pi = 0.f;
  if (p.op != kOpNorms) {
    wo_values<F32>(d, cr0, cc0, in, sO, w, o);
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        om = fmaf(o[h][e], o[h][e], om);
        de = fmaf(w[h][e], o[h][e], de);
      }
  } else {
#pragma unroll
    for (int h = 0; h < 2; ++h) raw_cvt8(in.w[h], F32 && (d.flags & kWF32), w[h]);
  }
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int e = 0; e < 8; ++e) pi = fmaf(w[h][e], w[h][e], pi);
  const float a3[3] = {om, de, pi};
  double s[3];
  cta_sum<3>(a3, s, red, nred & 1);
  ++nred;
  if (threadIdx.x == 0) {
    const int64_t rec = (int64_t)d.rec_begin + (cblk - d.blk_begin);   // the matrix's own records
    p.partials[3 * rec + 0] = s[0];
    p.partials[3 * rec + 1] = s[1];
    p.partials[3 * rec + 2] = s[2];
  }
}

// Register prefetch of the next block (F32 as for momentum_kernel).
template <bool F32>
__global__ void __launch_bounds__(kThreads, F32 ? 2 : 3) reduce_kernel(const __grid_constant__ ApplyParams p) {
  pdl_trigger();
  pdl_wait();
  __shared__ float sO[kBlk][kBlk + 1];
  __shared__ double red[2][3 * kWarps];
  const bool want_o = p.op != kOpNorms;
  int blk = blockIdx.x;
  if (blk >= p.total_blocks) return;
  int mi = find_mat(p, blk);
  int r0, c0;
  block_origin(p.mats[mi], blk - p.mats[mi].blk_begin, r0, c0);
  WoIn nxt;
  wo_load<F32>(p, p.mats[mi], r0, c0, want_o, nxt);
  int nred = 0;
  for (;;) {
    const WoIn in = nxt;
    const int cblk = blk, cr0 = r0, cc0 = c0;
    const MatDesc &d = p.mats[mi];
    blk += gridDim.x;
    const bool more = blk < p.total_blocks;
    if (more) {
      const int nmi = advance_mat(p, mi, blk);
      block_origin(p.mats[nmi], blk - p.mats[nmi].blk_begin, r0, c0);
      wo_load<F32>(p, p.mats[nmi], r0, c0, want_o, nxt);
      mi = nmi;
    }
    reduce_block<F32>(p, d, cblk, cr0, cc0, in, sO, red, nred);
    if (!more) break;
  }
}

// ||W - t O||^2 for matrices flagged need_exact; a persistent grid walks their blocks.
__global__ void __launch_bounds__(kThreads) exact_norm_kernel(const __grid_constant__ ApplyParams p) {
  pdl_trigger();
  pdl_wait();
  __shared__ float sO[kBlk][kBlk + 1];
  __shared__ double red[2][kWarps];
  if (*(volatile uint32_t *)(p.status + 1) == 0) return;  // no matrix of this call needs it
  int nred = 0;
  for (int mi = 0; mi < p.nmat; ++mi) {
    const MatDesc &d = p.mats[mi];
    const MatScalars &sc = p.scal[d.mat];
    if (!sc.need_exact) continue;
    const int nb = (mi + 1 < p.nmat ? p.mats[mi + 1].blk_begin : p.total_blocks) - d.blk_begin;
    const float tt = (float)sc.t;
    for (int lb = blockIdx.x; lb < nb; lb += gridDim.x) {
      int r0, c0;
      block_origin(d, lb, r0, c0);
      WoIn in;
      wo_load<true>(p, d, r0, c0, true, in);
      float w[2][8], o[2][8];
      wo_values<true>(d, r0, c0, in, sO, w, o);
      float acc = 0.f;
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float v = fmaf(-tt, o[h][e], w[h][e]);
          acc = fmaf(v, v, acc);
        }
      const float a1[1] = {acc};
      double s[1];
      cta_sum<1>(a1, s, red, nred & 1);
      ++nred;
      if (threadIdx.x == 0) p.partials[d.blk_begin + lb] = s[0];
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
  pdl_trigger();
  pdl_wait();
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
    // (||O||^2, <W,O>, ||W||^2) records of this matrix: one per block of the reduce pass,
    // or one per epilogue warp and tile of the last Newton-Schulz update
    for (int b = p.rec_begin[k] + lane; b < p.rec_begin[k + 1]; b += 32) {
      om += p.partials[3 * (int64_t)b];
      de += p.partials[3 * (int64_t)b + 1];
      pi += p.partials[3 * (int64_t)b + 2];
    }
    om = warp_sum(om);
    de = warp_sum(de);
    pi = warp_sum(pi);
  } else if (s.need_exact) {
    for (int b = p.blk_begin[k] + lane; b < p.blk_begin[k + 1]; b += 32) ex += p.xpartials[b];
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
    if (p.op == kOpRelative) {
      // RelativeUpdate: the update is rescaled to ||W||, so the step is lr ||W|| O / ||O||.
      s.alpha = (float)(1.0 - (double)p.lr * (double)p.weight_decay);
      s.beta = (float)(-(double)p.lr * sqrt(pi) / fmax(sqrt(om), (double)p.hb_eps));
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
template <bool F32>
__device__ __forceinline__ void apply_block(const MatDesc &d, int cr0, int cc0, const WoIn &in, float a, float b,
                                            float (&sO)[kBlk][kBlk + 1]) {
  const int rq = threadIdx.x >> 3, cq = (threadIdx.x & 7) * 8;
  const bool f32 = F32 && (d.flags & kWF32), vec = d.flags & kVec;
  float w[2][8], o[2][8];
  wo_values<F32>(d, cr0, cc0, in, sO, w, o);
  if (d.O_out) {
    const bool vo = ((uintptr_t)d.O_out % 16 == 0) && (d.n % (f32 ? 4 : 8) == 0);
#pragma unroll
    for (int h = 0; h < 2; ++h) store8(d.O_out, d.n, cr0 + rq + 32 * h, cc0 + cq, d.m, d.n, f32, vo, o[h]);
  }
  if (!(a == 1.f && b == 0.f)) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int e = 0; e < 8; ++e) w[h][e] = fmaf(a, w[h][e], b * o[h][e]);
      store8(d.W, d.ld, cr0 + rq + 32 * h, cc0 + cq, d.m, d.n, f32, vec, w[h]);
    }
  }
}

// Register prefetch of the next block (F32 as for momentum_kernel).
template <bool F32>
__global__ void __launch_bounds__(kThreads, F32 ? 2 : 4) apply_kernel(const __grid_constant__ ApplyParams p) {
  pdl_trigger();
  pdl_wait();
  __shared__ float sO[kBlk][kBlk + 1];
  int blk = blockIdx.x;
  if (blk >= p.total_blocks) return;
  int mi = find_mat(p, blk);
  int r0, c0;
  block_origin(p.mats[mi], blk - p.mats[mi].blk_begin, r0, c0);
  WoIn nxt;
  wo_load<F32>(p, p.mats[mi], r0, c0, true, nxt);
  float na = p.scal[p.mats[mi].mat].alpha, nb = p.scal[p.mats[mi].mat].beta;
  for (;;) {
    const WoIn in = nxt;
    const int cr0 = r0, cc0 = c0;
    const float a = na, b = nb;
    const MatDesc &d = p.mats[mi];
    blk += gridDim.x;
    const bool more = blk < p.total_blocks;
    if (more) {
      const int nmi = advance_mat(p, mi, blk);
      const MatDesc &dn = p.mats[nmi];
      block_origin(dn, blk - dn.blk_begin, r0, c0);
      wo_load<F32>(p, dn, r0, c0, true, nxt);
      if (nmi != mi) {
        na = p.scal[dn.mat].alpha;
        nb = p.scal[dn.mat].beta;
      }
      mi = nmi;
    }
    apply_block<F32>(d, cr0, cc0, in, a, b, sO);
    if (!more) break;
  }
}

// ------------------------------------------------------------------------- AdamH
// Inputs of one block: G, M, V and W for the thread's two rows.
struct AdamIn {
  Raw8 g[2], m[2], v[2], w[2];
};

template <bool F32>
__device__ __forceinline__ void adam_block(const AdamParams &p, const MatDesc &d, const float *V, int blk, int r0,
                                           int c0, double (*red)[3 * kWarps], int &nred) {
  const int rq = threadIdx.x >> 3, cq = (threadIdx.x & 7) * 8;
  const bool f32 = F32 && (d.flags & kWF32), vec = d.flags & kVec;
  AdamIn in;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int i = r0 + rq + 32 * h, j = c0 + cq;
    raw_load8(d.G, d.ld, i, j, d.m, d.n, f32, vec, in.g[h]);
    raw_load8(d.M, d.ld, i, j, d.m, d.n, true, vec, in.m[h]);
    raw_load8(V, d.ld, i, j, d.m, d.n, true, vec, in.v[h]);
    raw_load8(d.W, d.ld, i, j, d.m, d.n, f32, vec, in.w[h]);
  }
  const float b1 = p.beta1, b2 = p.beta2, omb1 = 1.0f - p.beta1, omb2 = 1.0f - p.beta2;
  float om = 0.f, de = 0.f, pi = 0.f;
  char *ubase = p.ws + d.o_off;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int i = r0 + rq + 32 * h, j = c0 + cq;
    float g[8], mm[8], vv[8], w[8], u[8];
    raw_cvt8(in.g[h], f32, g);
    raw_cvt8(in.m[h], true, mm);
    raw_cvt8(in.v[h], true, vv);
    raw_cvt8(in.w[h], f32, w);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      // Outside the matrix g = m = v = 0, so u = 0 there without masking.
      mm[e] = fmaf(b1, mm[e], omb1 * g[e]);
      vv[e] = fmaf(b2, vv[e], omb2 * g[e] * g[e]);
      const float uf = (mm[e] * p.bc1) / (sqrtf(vv[e] * p.bc2) + p.eps);
      u[e] = uf;
      const float us = f32 ? uf : bf16_round(uf);   // what the apply kernels will read
      om = fmaf(us, us, om);
      de = fmaf(w[e], us, de);
      pi = fmaf(w[e], w[e], pi);
    }
    store8(d.M, d.ld, i, j, d.m, d.n, true, vec, mm);
    store8(const_cast<float *>(V), d.ld, i, j, d.m, d.n, true, vec, vv);
    x_store8(ubase, d, i, j, u, F32);
  }
  const float a3[3] = {om, de, pi};
  double s[3];
  cta_sum<3>(a3, s, red, nred & 1);
  ++nred;
  if (threadIdx.x == 0) {
    p.partials[3 * (int64_t)blk + 0] = s[0];
    p.partials[3 * (int64_t)blk + 1] = s[1];
    p.partials[3 * (int64_t)blk + 2] = s[2];
  }
}

template <bool F32>
__global__ void __launch_bounds__(kThreads, F32 ? 2 : 3) adam_kernel(const __grid_constant__ AdamParams p) {
  pdl_trigger();
  pdl_wait();
  __shared__ double red[2][3 * kWarps];
  int blk = blockIdx.x;
  if (blk >= p.total_blocks) return;
  int mi = find_mat(p, blk);
  int nred = 0;
  for (; blk < p.total_blocks; blk += gridDim.x) {
    mi = advance_mat(p, mi, blk);
    const MatDesc &d = p.mats[mi];
    int r0, c0;
    block_origin(d, blk - d.blk_begin, r0, c0);
    adam_block<F32>(p, d, p.V[mi], blk, r0, c0, red, nred);
  }
}

// Persistent grid: the SM count times the CTAs of `kernel` that fit on one SM with
// `dyn_smem` bytes of dynamic shared memory, capped by the work.  Queried once per
// kernel and device.
template <typename K>
int stream_grid(K kernel, int slot, int dyn_smem, int total_blocks) {
  static PerDevice cached[8];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  int g = cached[slot].get(dev);
  if (g == 0) {
    int sms = 0, per = 0;
    if (dyn_smem > 0) cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_smem);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, kernel, kThreads, dyn_smem);
    g = (sms > 0 ? sms : 148) * (per > 0 ? per : 1);
    cached[slot].set(dev, g);
  }
  return total_blocks < g ? total_blocks : g;
}

}  // namespace

// The bf16 instances need every matrix of the launch in bf16 (W, G and X); anything
// else (fp32 W or X, the Newton-Muon U/P buffers) takes the F32 instances.
template <typename P>
bool needs_f32(const P &p) {
  for (int i = 0; i < p.nmat; ++i)
    if (p.mats[i].flags & (kWF32 | kNsF32 | kFromP | kURow)) return true;
  return false;
}

cudaError_t launch_momentum(const MomentumParams &p, cudaStream_t s) {
  if (p.total_blocks > 0) {
    if (needs_f32(p))
      return launch_pdl(momentum_kernel<true>, stream_grid(momentum_kernel<true>, 0, 0, p.total_blocks), kThreads, 0, s, p);
    else
      return launch_pdl(momentum_kernel<false>, stream_grid(momentum_kernel<false>, 1, 0, p.total_blocks), kThreads, 0, s,
                        p);
  }
  return cudaGetLastError();
}
cudaError_t launch_norm_finalize(const NormFinParams &p, int nseg_total, cudaStream_t s) {
  if (nseg_total > 0) return launch_pdl(norm_finalize_kernel, (nseg_total + 7) / 8, 256, 0, s, p, nseg_total);
  return cudaGetLastError();
}
cudaError_t launch_reduce(const ApplyParams &p, cudaStream_t s) {
  if (p.total_blocks > 0) {
    if (needs_f32(p))
      return launch_pdl(reduce_kernel<true>, stream_grid(reduce_kernel<true>, 2, 0, p.total_blocks), kThreads, 0, s, p);
    else
      return launch_pdl(reduce_kernel<false>, stream_grid(reduce_kernel<false>, 3, 0, p.total_blocks), kThreads, 0, s, p);
  }
  return cudaGetLastError();
}
cudaError_t launch_exact_norm(const ApplyParams &p, cudaStream_t s) {
  if (p.total_blocks > 0) return launch_pdl(exact_norm_kernel, 296, kThreads, 0, s, p);
  return cudaGetLastError();
}
cudaError_t launch_apply_finalize(const ApplyFinParams &p, cudaStream_t s) {
  if (p.nmat > 0) return launch_pdl(apply_finalize_kernel, (p.nmat + 3) / 4, 128, 0, s, p);
  return cudaGetLastError();
}
cudaError_t launch_adam(const AdamParams &p, cudaStream_t s) {
  if (p.total_blocks > 0) {
    if (needs_f32(p))
      return launch_pdl(adam_kernel<true>, stream_grid(adam_kernel<true>, 6, 0, p.total_blocks), kThreads, 0, s, p);
    else
      return launch_pdl(adam_kernel<false>, stream_grid(adam_kernel<false>, 7, 0, p.total_blocks), kThreads, 0, s, p);
  }
  return cudaGetLastError();
}
cudaError_t launch_apply(const ApplyParams &p, cudaStream_t s) {
  if (p.total_blocks > 0) {
    if (needs_f32(p))
      return launch_pdl(apply_kernel<true>, stream_grid(apply_kernel<true>, 4, 0, p.total_blocks), kThreads, 0, s, p);
    else
      return launch_pdl(apply_kernel<false>, stream_grid(apply_kernel<false>, 5, 0, p.total_blocks), kThreads, 0, s, p);
  }
  return cudaGetLastError();
}

}  // namespace nshb
