// Newton-Muon preconditioner pieces ("The Newton-Muon Optimizer", abstract: the update
// msgn(G (Z Z^T)^-1), here with a ridge lambda = ridge_rel tr(Z Z^T) / d_in).
//
//   ridge         lambda = ridge_rel tr(S) / d, S += lambda I (one CTA per Z, fixed order);
//   split         fp32 regions -> bf16 hi / lo panels, the operands of the split products;
//   potrf_diag    Cholesky factor of a 256 x 256 diagonal block and its inverse, which
//                 turns every panel and block solve into a product.
// S = Z Z^T itself runs on the grouped pair GEMM (ns_tc2.cu), reading each Z where the
// caller keeps it.  The column updates, the panels and the triangular solves for
// P = U S^-1 (a left-looking blocked Cholesky) run on the split-precision tensor-core GEMM
// (newton_tc.cu); the host sequences them.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "nshb_device.cuh"
#include "nshb_internal.h"

namespace nshb {
namespace {

// lambda = ridge_rel tr(S) / d added to the diagonal.  The padded rows and columns of S
// (d .. ld-1, zero from the Gram) get a unit diagonal, so the padded matrix factors as
// [L 0; 0 I] and the padded columns of every solve stay zero.
__global__ void __launch_bounds__(256) ridge_kernel(const __grid_constant__ CholParams p) {
  __shared__ double red[8];
  const int z = blockIdx.x;
  float *S = reinterpret_cast<float *>(p.ws + p.s_off[z]);
  const int ld = p.ld[z], d = p.d[z];
  double v[1] = {0.0};
  for (int i = threadIdx.x; i < d; i += blockDim.x) v[0] += (double)S[(int64_t)i * ld + i];
  block_sum<1>(v, red);
  const float lam = (float)((double)p.ridge_rel * v[0] / (double)d);
  for (int i = threadIdx.x; i < d; i += blockDim.x) S[(int64_t)i * ld + i] += lam;
  for (int i = d + threadIdx.x; i < ld; i += blockDim.x) S[(int64_t)i * ld + i] = 1.f;
}

// fp32 regions -> bf16 hi/lo panels (X_hi = bf16(X), X_lo = bf16(X - X_hi)), one 64 x 64
// block per CTA; thread t handles 8 columns 8 (t % 8) .. +7 of rows t / 8 and 32 + t / 8 (two
// 16-byte loads each where the row is whole and 16-byte aligned).
__global__ void __launch_bounds__(256) split_kernel(const __grid_constant__ SplitParams p) {
  pdl_trigger();
  pdl_wait();
  const int blk = blockIdx.x;
  if (blk >= p.total_blocks) return;
  int lo = 0, hi = p.n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.item[mid].blk_begin <= blk) lo = mid; else hi = mid - 1;
  }
  const SplitItem &it = p.item[lo];
  const int lb = blk - it.blk_begin, bc = it.pcol / 64;
  const int r0 = (lb / bc) * 64, c0 = (lb % bc) * 64;
  const float *src = reinterpret_cast<const float *>(p.ws + it.src32);
  float *dst = it.dst32 >= 0 ? reinterpret_cast<float *>(p.ws + it.dst32) : nullptr;
  const bool vsrc = (it.src_ld & 3) == 0 && (reinterpret_cast<uintptr_t>(src) & 15) == 0;
  const bool vdst = dst && (it.dst_ld & 3) == 0 && (reinterpret_cast<uintptr_t>(dst) & 15) == 0;
  float v[2][8];
#pragma unroll
  for (int u = 0; u < 2; ++u) {                     // both loads in flight before any store
    const int q = threadIdx.x + 256 * u;
    const int r = r0 + (q >> 3), c = c0 + 8 * (q & 7);
    const float *s = src + (int64_t)r * it.src_ld + c;
    if (vsrc && r < it.rows && c + 8 <= it.cols) {
      const float4 a = *reinterpret_cast<const float4 *>(s), b = *reinterpret_cast<const float4 *>(s + 4);
      v[u][0] = a.x; v[u][1] = a.y; v[u][2] = a.z; v[u][3] = a.w;
      v[u][4] = b.x; v[u][5] = b.y; v[u][6] = b.z; v[u][7] = b.w;
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) v[u][e] = (r < it.rows && c + e < it.cols) ? s[e] : 0.f;
    }
  }
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int q = threadIdx.x + 256 * u;
    const int r = r0 + (q >> 3), c = c0 + 8 * (q & 7);
    if (dst) {
      float *d = dst + (int64_t)r * it.dst_ld + c;
      if (vdst) {
        *reinterpret_cast<float4 *>(d) = make_float4(v[u][0], v[u][1], v[u][2], v[u][3]);
        *reinterpret_cast<float4 *>(d + 4) = make_float4(v[u][4], v[u][5], v[u][6], v[u][7]);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) d[e] = v[u][e];
      }
    }
    uint4 h, l;
    uint32_t *hp = &h.x, *lp = &l.x;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      hp[e] = pack_bf16(v[u][2 * e], v[u][2 * e + 1]);
      lp[e] = pack_bf16(v[u][2 * e] - bf16lo(hp[e]), v[u][2 * e + 1] - bf16hi(hp[e]));
    }
    const size_t off = panel_chunk_off(it.d_r0 + r, it.d_c0 + c, it.d_ph);
    *reinterpret_cast<uint4 *>(p.ws + it.dhi + off) = h;
    *reinterpret_cast<uint4 *>(p.ws + it.dlo + off) = l;
  }
}

// ------------------------------------------------ diagonal block of the factorisation
// One 256 x 256 diagonal block A of S per layer input (one CTA each), factored A = L L^T and
// inverted, D = L^-1, in one left-to-right sweep over eight 32-wide block columns.  The lower
// triangle lives in shared memory as 36 blocks of 32 x 32 (block (i, k), i >= k); every
// block is overwritten in turn by L and then by D.  Step j:
//   A  one warp factors the diagonal block, A_jj = L_jj L_jj^T, and inverts it, D_jj =
//      L_jj^-1 (L_jj itself is needed by nothing else);
//   B  panel L_ij = A_ij D_jj^T (i > j), and X_jm = D_jj L_jm (m < j: block row j of L is
//      no longer read by the factorisation);
//   C  trailing update A_ik -= L_ij L_kj^T (j < k <= i), and block row j of D,
//      D_jk = -sum_{k <= m < j} X_jm D_mk  (from D L = I).
// Step j + 1's A runs inside step j's C: the warp that updates block (j + 1, j + 1) factors
// it right away while the other warps finish the rest of C.  The result goes out as bf16
// hi / lo panels into the stack of 512-wide inverses (rows 256 k, columns 256 (k % 2)), with
// zeros above the diagonal.  A pivot that
// is not positive in fp32 is flagged (NSHB_DEV_NOT_SPD) and replaced by 1e-30.
constexpr int kNB = 8;                    // block columns
constexpr int kBS = 36;                   // row stride of a block (floats): conflict-free float4 rows
constexpr int kBlk = 32 * kBS + 4;        // block stride (floats): consecutive blocks start 4 banks apart
constexpr int kNBlk = kNB * (kNB + 1) / 2;
constexpr int kDiagThreads = 512, kDiagWarps = kDiagThreads / 32;
constexpr int kLtStride = 64;             // L^T scratch of the diagonal factor: 32 shifted rows
constexpr int kPartSlots = 10;            // partial sums of the split block-row products (at most 10)
constexpr int kDiagSmem = (kNBlk * kBlk + 32 * kLtStride + 128 + kPartSlots * 1024) * 4;
static_assert(kDiagSmem <= 227 * 1024, "diagonal block does not fit in shared memory");

__device__ __forceinline__ float *blk(float *sm, int i, int k) { return sm + (i * (i + 1) / 2 + k) * kBlk; }

// Block products on one warp: a 32 x 32 output, four rows (g + 8x, g = lane / 4) and eight
// columns per lane.  Reads are 16-byte rows of distinct banks, or broadcasts.
// acc[x][e] += sum_q A[g + 8x][q] B[h + 4e][q]   (A B^T;  h = lane % 4)
__device__ __forceinline__ void nt_acc(const float *A, const float *B, float (&acc)[4][8]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, h = lane & 3;
#pragma unroll 2
  for (int q = 0; q < 32; q += 4) {
    float4 a[4], b[8];
#pragma unroll
    for (int x = 0; x < 4; ++x) a[x] = *reinterpret_cast<const float4 *>(A + (g + 8 * x) * kBS + q);
#pragma unroll
    for (int e = 0; e < 8; ++e) b[e] = *reinterpret_cast<const float4 *>(B + (h + 4 * e) * kBS + q);
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float t = acc[x][e];
        t = fmaf(a[x].x, b[e].x, t);
        t = fmaf(a[x].y, b[e].y, t);
        t = fmaf(a[x].z, b[e].z, t);
        acc[x][e] = fmaf(a[x].w, b[e].w, t);
      }
  }
}

// acc[x][e] += sum_q A[g + 8x][q] B[q][8h + e]   (A B)
__device__ __forceinline__ void nn_acc(const float *A, const float *B, float (&acc)[4][8]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, h = lane & 3;
#pragma unroll 2
  for (int q = 0; q < 32; q += 4) {
    float4 a[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) a[x] = *reinterpret_cast<const float4 *>(A + (g + 8 * x) * kBS + q);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float4 b0 = *reinterpret_cast<const float4 *>(B + (q + t) * kBS + 8 * h);
      const float4 b1 = *reinterpret_cast<const float4 *>(B + (q + t) * kBS + 8 * h + 4);
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const float av = t == 0 ? a[x].x : t == 1 ? a[x].y : t == 2 ? a[x].z : a[x].w;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[x][e] = fmaf(av, b[e], acc[x][e]);
      }
    }
  }
}

__device__ __forceinline__ void zero_acc(float (&acc)[4][8]) {
#pragma unroll
  for (int x = 0; x < 4; ++x)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[x][e] = 0.f;
}

// Stores sgn * acc into a block, in the element order of nt_acc (nt) or nn_acc.
__device__ __forceinline__ void put_acc(float *C, const float (&acc)[4][8], float sgn, bool nt) {
  const int lane = threadIdx.x & 31, g = lane >> 2, h = lane & 3;
#pragma unroll
  for (int x = 0; x < 4; ++x)
#pragma unroll
    for (int e = 0; e < 8; ++e) C[(g + 8 * x) * kBS + (nt ? h + 4 * e : 8 * h + e)] = sgn * acc[x][e];
}

// One warp: block B (32 x 32, lower triangle read) is replaced by D = L^-1, where B = L L^T.
// Right-looking Cholesky with row r in lane r's registers, shifted by one column per step so
// that the current column is always a[0] and the loop body is the same for every step.  The
// column of L that every lane needs is exchanged through shared memory (each lane stores its
// entry already shifted, so the reads are eight aligned 16-byte broadcasts) instead of 31
// dependent shuffles; the lane that holds the next pivot computes it from its own L entry as
// soon as it has one (the same fma as its update below), so only one shuffle per step sits on
// the chain of pivots.  Row j of L^T is kept shifted the same way in LT (LT[j][k] = L[j + k][j],
// LT[j][0] = 1 / L[j][j], which is the pivot's rsqrt; entries past row 31 are never used), and
// lane c then solves column c
// of D by forward substitution, D[q][c] = (e_c - sum_{p < q} L[q][p] D[p][c]) / L[q][q].
__device__ void chol_inv_block(float *B, float *LT, float *xv, uint32_t *status) {
  const int lane = threadIdx.x & 31;
  float a[32];
#pragma unroll
  for (int c = 0; c < 32; c += 4) {
    const float4 v = *reinterpret_cast<const float4 *>(B + lane * kBS + c);
    a[c] = v.x; a[c + 1] = v.y; a[c + 2] = v.z; a[c + 3] = v.w;
  }
  bool bad = false;
  float pn = a[0];                                      // lane j's pivot at step j
#pragma unroll 1
  for (int j = 0; j < 32; ++j) {                       // a[k] = current A[lane][j + k]
    float piv = __shfl_sync(0xffffffffu, pn, j);
    bad |= !(piv > 0.f);
    piv = piv > 0.f ? piv : 1e-30f;
    const float rs = rsqrtf(piv);
    const float l = lane > j ? a[0] * rs : lane == j ? piv * rs : 0.f;   // L[lane][j]
    pn = fmaf(-l, l, a[1]);       // this lane's a[0] after the update below: lane j + 1's next pivot
    float *v = xv + 64 * (j & 1);                       // two buffers: step j + 1 writes the other
    v[(lane - j - 1) & 63] = l;                         // v[c - 1] = L[j + c][j]
    LT[j * kLtStride + ((lane - j) & 63)] = lane == j ? rs : l;   // 1 / L[j][j] = rsqrt(pivot)
    __syncwarp();
#pragma unroll
    for (int c4 = 0; c4 < 32; c4 += 4) {
      const float4 w = *reinterpret_cast<const float4 *>(v + c4);
      const float wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (c4 + u < 31) a[c4 + u] = fmaf(-l, wv[u], a[c4 + u + 1]);
    }
    a[31] = 0.f;
  }
  if (bad && lane == 0) set_status(status, 0x10u);
  __syncwarp();
  float d[32];                                          // d[k] = pending D[q + k][lane]
#pragma unroll
  for (int i = 0; i < 32; ++i) d[i] = i == lane ? 1.f : 0.f;
#pragma unroll 1
  for (int q = 0; q < 32; ++q) {
    const float *lt = LT + q * kLtStride;
    float w[32];
#pragma unroll
    for (int k4 = 0; k4 < 32; k4 += 4) {
      const float4 t = *reinterpret_cast<const float4 *>(lt + k4);
      w[k4] = t.x; w[k4 + 1] = t.y; w[k4 + 2] = t.z; w[k4 + 3] = t.w;
    }
    const float dq = d[0] * w[0];
    B[q * kBS + lane] = dq;
#pragma unroll
    for (int k = 1; k < 32; ++k) d[k - 1] = fmaf(-w[k], dq, d[k]);
    d[31] = 0.f;
  }
  __syncwarp();
}

// Block row J of D over `nw` warps (this one is number w of them): D_Jk = -sum_{k <= m < J} X_Jm D_mk,
// each sum cut into pieces of the fewest products that give every piece a warp (k-major, one
// piece per warp; at most 10 partial slots for J <= 7 and nw >= 12).  The pieces after the first
// of a sum leave their partial in a scratch slot; after every participating warp has read its
// operands (named barrier 1 over the nw warps), the first piece adds them in order and writes
// the block in place of X_Jk.
__device__ void drow(float *sm, float *part, int J, int w, int nw) {
  const int lane = threadIdx.x & 31;
  int sz = 1;                                           // smallest piece size whose pieces fit the warps
  for (;; ++sz) {
    int cnt = 0;
    for (int kk = 0; kk < J; ++kk) cnt += (J - kk + sz - 1) / sz;
    if (cnt <= nw) break;
  }
  int k = 0, p = 0, first = 0, np = 0;                  // this warp's piece: sum k, piece p of np
  bool mine = false;
  for (int kk = 0, idx = 0; kk < J; ++kk) {
    const int n = (J - kk + sz - 1) / sz;
    if (w >= idx && w < idx + n) {
      k = kk; p = w - idx; first = idx; np = n; mine = true;
    }
    idx += n;
  }
  float acc[4][8];
  zero_acc(acc);
  if (mine)
    for (int m = k + sz * p; m < min(J, k + sz * p + sz); ++m) nn_acc(blk(sm, J, m), blk(sm, m, k), acc);
  if (mine && p > 0) {
    float *slot = part + (first + p - (k + 1)) * 1024;
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int e = 0; e < 8; ++e) slot[(8 * x + e) * 32 + lane] = acc[x][e];
  }
  asm volatile("bar.sync 1, %0;" ::"r"(nw * 32) : "memory");
  if (mine && p == 0) {
    for (int q = 1; q < np; ++q) {
      const float *slot = part + (first + q - (k + 1)) * 1024;
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[x][e] += slot[(8 * x + e) * 32 + lane];
    }
    put_acc(blk(sm, J, k), acc, -1.f, false);
  }
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

__global__ void __launch_bounds__(kDiagThreads, 1) potrf_diag_kernel(const __grid_constant__ DiagParams p) {
  extern __shared__ __align__(16) float sm[];
  // Wait first, then let the next kernel start: it may run beside this one (the update of U by
  // the previous step does not touch S), and everything before this kernel is complete.
  pdl_wait();
  pdl_trigger();
  const int z = blockIdx.x;
  if (z >= p.n) return;
  const int ld = p.ld[z], k0 = 256 * p.k;
  if (k0 >= ld) return;
  const float *S = reinterpret_cast<const float *>(p.ws + p.s32[z]);
  char *hi = p.ws + p.dhi[z], *lo = p.ws + p.dlo[z];
  const int warp = threadIdx.x >> 5;
  float *LT = sm + kNBlk * kBlk, *xv = LT + 32 * kLtStride, *part = xv + 128;
  // the 36 lower blocks, 32 rows of eight 16-byte pieces each: block column 0 first (all that
  // step 0's factor and panel read), the other 28 blocks as a second group that lands while
  // the first diagonal block is factored
  auto load_blk = [&](int i, int k, int r, int c4) {
    cp_async16(blk(sm, i, k) + r * kBS + 4 * c4, S + (int64_t)(k0 + 32 * i + r) * ld + k0 + 32 * k + 4 * c4);
  };
  for (int q = threadIdx.x; q < kNB * 256; q += kDiagThreads) load_blk(q >> 8, 0, (q >> 3) & 31, q & 7);
  asm volatile("cp.async.commit_group;" ::: "memory");
  for (int q = threadIdx.x; q < (kNBlk - kNB) * 256; q += kDiagThreads) {
    int i = 0, k = q >> 8;
    while (k > i) k -= ++i;
    load_blk(i + 1, k + 1, (q >> 3) & 31, q & 7);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  asm volatile("cp.async.wait_group 1;" ::: "memory");
  __syncthreads();
  if (warp == 0) chol_inv_block(blk(sm, 0, 0), LT, xv, p.status);
  __syncthreads();
  // A_ik -= L_ij L_kj^T for one block
  auto trail = [&](int j, int i, int k) {
    float acc[4][8];
    zero_acc(acc);
    nt_acc(blk(sm, i, j), blk(sm, k, j), acc);
    float *C = blk(sm, i, k);
    const int lane = threadIdx.x & 31, g = lane >> 2, h = lane & 3;
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int e = 0; e < 8; ++e) C[(g + 8 * x) * kBS + h + 4 * e] -= acc[x][e];
  };
  for (int j = 0; j < kNB; ++j) {
    // B: the panel below (7 - j blocks) and block row j of X (j blocks), one block per warp
    if (warp < kNB - 1) {
      float acc[4][8];
      zero_acc(acc);
      float *C;
      const bool panel = warp < kNB - 1 - j;
      if (panel) {
        C = blk(sm, j + 1 + warp, j);
        nt_acc(C, blk(sm, j, j), acc);                  // L_ij = A_ij D_jj^T
      } else {
        C = blk(sm, j, warp - (kNB - 1 - j));
        nn_acc(blk(sm, j, j), C, acc);                  // X_jm = D_jj L_jm
      }
      __syncwarp();
      put_acc(C, acc, 1.f, panel);
    }
    if (j == 0) asm volatile("cp.async.wait_group 0;" ::: "memory");   // the trailing blocks
    __syncthreads();
    // C: the trailing update.  Warp 0 updates the next diagonal block first and factors and
    // inverts it at once (look-ahead: the next step needs nothing else from this one to start
    // its factor); warps 1..15 update the other blocks and then finish block row j of D.
    // The other warps of warp 0's sub-partition (4, 8, 12) stay idle, so that its chain of
    // dependent steps gets every issue slot there.
    const int n = kNB - 1 - j;
    constexpr int kHelpers = kDiagWarps - kDiagWarps / 4;    // warps 1-3, 5-7, 9-11, 13-15
    if (warp == 0) {
      if (n > 0) {
        trail(j, j + 1, j + 1);
        __syncwarp();
        chol_inv_block(blk(sm, j + 1, j + 1), LT, xv, p.status);
      }
    } else if (warp & 3) {
      const int w = warp - warp / 4 - 1;                     // 0 .. kHelpers - 1
      for (int t = 1 + w; t < n * (n + 1) / 2; t += kHelpers) {   // task 0 is warp 0's block
        int ii = 0, kk = t;
        while (kk > ii) kk -= ++ii;
        trail(j, j + 1 + ii, j + 1 + kk);
      }
      if (j >= 1) drow(sm, part, j, w, kHelpers);
    }
    __syncthreads();
  }
  // out: rows k0 .. k0+255, columns 0 .. 255 of the stack, eight columns per 16-byte piece
  const int cofs = (p.k & 1) * 256;
  for (int q = threadIdx.x; q < 256 * 32; q += kDiagThreads) {
    const int r = q >> 5, c = 8 * (q & 31), i = r >> 5, k = c >> 5;
    uint4 h = make_uint4(0, 0, 0, 0), l = h;
    if (k <= i) {
      const float *src = blk(sm, i, k) + (r & 31) * kBS + (c & 31);
      const float4 v0 = *reinterpret_cast<const float4 *>(src), v1 = *reinterpret_cast<const float4 *>(src + 4);
      const float v[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
      uint32_t *hp = &h.x, *lp = &l.x;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        hp[e] = pack_bf16(v[2 * e], v[2 * e + 1]);
        lp[e] = pack_bf16(v[2 * e] - bf16lo(hp[e]), v[2 * e + 1] - bf16hi(hp[e]));
      }
    }
    // block k's inverse goes to columns 256 (k % 2) .. +255 of the 512-wide stack; an even
    // block also zeroes columns 256 .. 511 of its rows, the upper-right block of the inverse
    // of the 512 x 512 diagonal block it forms with block k + 1
    const size_t off = panel_chunk_off(k0 + r, cofs + c, ld);
    *reinterpret_cast<uint4 *>(hi + off) = h;
    *reinterpret_cast<uint4 *>(lo + off) = l;
    if (cofs == 0) {
      const size_t zo = panel_chunk_off(k0 + r, 256 + c, ld);
      *reinterpret_cast<uint4 *>(hi + zo) = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4 *>(lo + zo) = make_uint4(0, 0, 0, 0);
    }
  }
}

}  // namespace

cudaError_t launch_ridge(const CholParams &p, cudaStream_t s) {
  if (p.n > 0) ridge_kernel<<<p.n, 256, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_split(const SplitParams &p, cudaStream_t s) {
  if (p.total_blocks > 0) return launch_pdl(split_kernel, p.total_blocks, 256, 0, s, p);
  return cudaGetLastError();
}
cudaError_t launch_potrf_diag(const DiagParams &p, cudaStream_t s) {
  static PerDevice attr_set;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr_set.get(dev)) {
    cudaError_t e = cudaFuncSetAttribute(potrf_diag_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDiagSmem);
    if (e != cudaSuccess) return e;
    attr_set.set(dev, 1);
  }
  if (p.n > 0) return launch_pdl(potrf_diag_kernel, p.n, kDiagThreads, kDiagSmem, s, p);
  return cudaGetLastError();
}

}  // namespace nshb
