// Newton-Muon preconditioner pieces ("The Newton-Muon Optimizer", abstract: the update
// msgn(G (Z Z^T)^-1), here with a ridge lambda = ridge_rel tr(Z Z^T) / d_in).
//
//   pack_panels   layer input Z (bf16 row-major d x n) -> the tensor-core panel layout,
//                 so that S = Z Z^T runs on the grouped tcgen05 GEMM (fp32 output);
//   ridge         lambda = ridge_rel tr(S) / d, S += lambda I (one CTA per Z, fixed order);
//   split         fp32 regions -> bf16 hi / lo panels, the operands of the split products;
//   potrf_diag    Cholesky factor of a 256 x 256 diagonal block and its inverse, which
//                 turns every panel and block solve into a product.
// The panel products, the trailing updates and the triangular solves for P = U S^-1 run
// on the split-precision tensor-core GEMM (newton_tc.cu); the host sequences them.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "nshb_device.cuh"
#include "nshb_internal.h"

namespace nshb {
namespace {

__global__ void __launch_bounds__(256) pack_panels_kernel(const __grid_constant__ PackParams p) {
  const int blk = blockIdx.x;
  int lo = 0, hi = p.n - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (p.blk_begin[mid] <= blk) lo = mid; else hi = mid - 1;
  }
  const int lb = blk - p.blk_begin[lo];
  const int rows = p.rows[lo], cols = p.cols[lo], ph = p.ph[lo];
  const int bc = cols / 64;
  const int r0 = (lb / bc) * 64, c0 = (lb % bc) * 64;
  const __nv_bfloat16 *src = static_cast<const __nv_bfloat16 *>(p.src[lo]);
  char *dst = p.ws + p.dst_off[lo];
  // 64 x 64 block = 512 chunks of 16 bytes; two per thread.
  for (int c = threadIdx.x; c < 512; c += 256) {
    const int rr = c >> 3, q = c & 7;
    const int r = r0 + rr, col = c0 + 8 * q;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < rows) v = *reinterpret_cast<const uint4 *>(src + (int64_t)r * p.ld[lo] + col);
    *reinterpret_cast<uint4 *>(dst + panel_chunk_off(r, col, ph)) = v;
  }
}

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
// block per CTA; thread t handles row t/4 (+ 64 (t/256)) ... columns 16 (t % 4) .. +15.
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
  for (int q = threadIdx.x; q < 64 * 8; q += blockDim.x) {
    const int r = r0 + (q >> 3), c = c0 + 8 * (q & 7);
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = (r < it.rows && c + e < it.cols) ? src[(int64_t)r * it.src_ld + c + e] : 0.f;
    if (dst) {
#pragma unroll
      for (int e = 0; e < 8; ++e) dst[(int64_t)r * it.dst_ld + c + e] = v[e];
    }
    uint4 h, l;
    uint32_t *hp = &h.x, *lp = &l.x;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      hp[e] = pack_bf16(v[2 * e], v[2 * e + 1]);
      lp[e] = pack_bf16(v[2 * e] - bf16lo(hp[e]), v[2 * e + 1] - bf16hi(hp[e]));
    }
    const size_t off = panel_chunk_off(it.d_r0 + r, it.d_c0 + c, it.d_ph);
    *reinterpret_cast<uint4 *>(p.ws + it.dhi + off) = h;
    *reinterpret_cast<uint4 *>(p.ws + it.dlo + off) = l;
  }
}

// ------------------------------------------------ diagonal block of the factorisation
// One 256 x 256 diagonal block of S per layer input, factored as two 128-column halves in
// shared memory (three 128 x 128 fp32 tiles), then inverted:
//   L11 = chol(A11);  D11 = L11^-1;  L21^T = D11 A12 (A12 = A21^T: the trailing update
//   keeps the whole diagonal block current);  L22 = chol(A22 - L21 L21^T);
//   D22 = L22^-1;  D21 = -D22 (L21 D11);
// the inverse D = [D11 0; D21 D22] goes out as bf16 hi/lo panels (block k of the stack).
constexpr int kT = 128, kTP = 132;       // tile size, row stride (floats; rows 16-byte aligned)
constexpr int kDiagThreads = 512;
constexpr int kDiagSmem = 3 * kT * kTP * 4;

// In-place lower Cholesky factor of a 128 x 128 tile (only its lower triangle is read).
// Column j: every thread takes the pivot a = T[j][j], updates its share of the trailing
// lower part with T[i][c] -= T[i][j] T[c][j] / a (four threads per row i, interleaved
// columns), and scales column j - 1 by 1 / sqrt of that column's pivot.  A pivot that is
// not positive is flagged (NSHB_DEV_NOT_SPD) and replaced by 1e-30.
__device__ __forceinline__ float pivot(float a) { return a > 0.f ? a : 1e-30f; }

__device__ void chol_tile(float *T, uint32_t *status) {
  const int tid = threadIdx.x, rr = tid >> 2, cpart = tid & 3;
  for (int j = 0; j < kT; ++j) {
    const float a0 = T[j * kTP + j];
    if (!(a0 > 0.f) && tid == 0) set_status(status, 0x10u);   // not positive definite in fp32
    const float a = pivot(a0);
    if (j > 0) {                                  // finish column j - 1
      const float rs = rsqrtf(pivot(T[(j - 1) * kTP + (j - 1)]));
      for (int i = j + tid; i < kT; i += kDiagThreads) T[i * kTP + (j - 1)] *= rs;
    }
    __syncthreads();
    if (tid == 0 && j > 0) T[(j - 1) * kTP + (j - 1)] = sqrtf(pivot(T[(j - 1) * kTP + (j - 1)]));
    const int i = j + 1 + rr;                     // one row per group of four threads
    if (i < kT) {
      const float li = T[i * kTP + j] / a;
      for (int c = j + 1 + cpart; c <= i; c += 4) T[i * kTP + c] = fmaf(-li, T[c * kTP + j], T[i * kTP + c]);
    }
    __syncthreads();
  }
  if (tid == 0) T[(kT - 1) * kTP + (kT - 1)] = sqrtf(pivot(T[(kT - 1) * kTP + (kT - 1)]));
  __syncthreads();
}

// D = L^-1 of a lower-triangular tile (D lower).  Warp w solves columns 8w .. 8w+7, four
// lanes per column: D[i][c] = (delta_ic - sum_{c <= q < i} L[i][q] D[q][c]) / L[i][i].
__device__ void inv_tile(const float *L, float *D) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = 8 * warp + (lane >> 2), part = lane & 3;
  for (int i = 0; i < kT; ++i) {
    float acc = 0.f;
    if (i > c)
      for (int q = c + part; q < i; q += 4) acc = fmaf(L[i * kTP + q], D[q * kTP + c], acc);
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    if (part == 0) D[i * kTP + c] = i < c ? 0.f : ((i == c ? 1.f : 0.f) - acc) / L[i * kTP + i];
    __syncwarp();
  }
  __syncthreads();
}

// acc[i][e] = sum_q A'[r0 + i][q] Y[q][c0 + e] over a 4 x 8 block per thread (r0 = 4 (t / 16),
// c0 = 8 (t % 16)), with A' = A, or A^T when atrans.  Four k steps at a time: A' as four
// float4 reads (rows of A, or rows of A^T = four consecutive rows of A' at one k), Y as
// eight; a warp's reads hit distinct banks or broadcast.
__device__ __forceinline__ void tile_products(const float *A, const float *Y, bool atrans, float (&acc)[4][8]) {
  const int tid = threadIdx.x, r0 = 4 * (tid >> 4), c0 = 8 * (tid & 15);
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[i][e] = 0.f;
  for (int q = 0; q < kT; q += 4) {
    float a[4][4];   // a[i][j] = A'[r0 + i][q + j]
    if (!atrans) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 v = *reinterpret_cast<const float4 *>(A + (r0 + i) * kTP + q);
        a[i][0] = v.x; a[i][1] = v.y; a[i][2] = v.z; a[i][3] = v.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 v = *reinterpret_cast<const float4 *>(A + (q + j) * kTP + r0);
        a[0][j] = v.x; a[1][j] = v.y; a[2][j] = v.z; a[3][j] = v.w;
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 y0 = *reinterpret_cast<const float4 *>(Y + (q + j) * kTP + c0);
      const float4 y1 = *reinterpret_cast<const float4 *>(Y + (q + j) * kTP + c0 + 4);
      const float y[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[i][e] = fmaf(a[i][j], y[e], acc[i][e]);
    }
  }
}

// Out = sgn * A' Y (128 x 128 tiles); Out may be A or Y (every read happens first).
__device__ void mul_tile(const float *A, const float *Y, float *Out, float sgn, bool atrans) {
  const int tid = threadIdx.x, r0 = 4 * (tid >> 4), c0 = 8 * (tid & 15);
  float acc[4][8];
  tile_products(A, Y, atrans, acc);
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    *reinterpret_cast<float4 *>(Out + (r0 + i) * kTP + c0) =
        make_float4(sgn * acc[i][0], sgn * acc[i][1], sgn * acc[i][2], sgn * acc[i][3]);
    *reinterpret_cast<float4 *>(Out + (r0 + i) * kTP + c0 + 4) =
        make_float4(sgn * acc[i][4], sgn * acc[i][5], sgn * acc[i][6], sgn * acc[i][7]);
  }
  __syncthreads();
}

// Writes a 128 x 128 tile into the hi / lo panels of the inverse stack at (r0, c0).
__device__ void store_tile_panels(const float *T, char *hi, char *lo, int ph, int r0, int c0) {
  for (int q = threadIdx.x; q < kT * kT / 8; q += kDiagThreads) {
    const int r = q >> 4, c = 8 * (q & 15);
    uint4 h, l;
    uint32_t *hp = &h.x, *lp = &l.x;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float v0 = T[r * kTP + c + 2 * e], v1 = T[r * kTP + c + 2 * e + 1];
      hp[e] = pack_bf16(v0, v1);
      lp[e] = pack_bf16(v0 - bf16lo(hp[e]), v1 - bf16hi(hp[e]));
    }
    const size_t off = panel_chunk_off(r0 + r, c0 + c, ph);
    *reinterpret_cast<uint4 *>(hi + off) = h;
    *reinterpret_cast<uint4 *>(lo + off) = l;
  }
}

__device__ void load_tile(const float *S, int ld, int r0, int c0, float *T) {
  for (int q = threadIdx.x; q < kT * kT / 4; q += kDiagThreads) {
    const int r = q >> 5, c = 4 * (q & 31);
    *reinterpret_cast<float4 *>(T + r * kTP + c) = *reinterpret_cast<const float4 *>(S + (int64_t)(r0 + r) * ld + c0 + c);
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kDiagThreads, 1) potrf_diag_kernel(const __grid_constant__ DiagParams p) {
  extern __shared__ __align__(16) float tsm[];
  float *T0 = tsm, *T1 = tsm + kT * kTP, *T2 = tsm + 2 * kT * kTP;
  pdl_trigger();
  pdl_wait();
  const int z = blockIdx.x;
  if (z >= p.n) return;
  const int ld = p.ld[z], k0 = 256 * p.k;
  if (k0 >= ld) return;
  const float *S = reinterpret_cast<const float *>(p.ws + p.s32[z]);
  char *hi = p.ws + p.dhi[z], *lo = p.ws + p.dlo[z];
  load_tile(S, ld, k0, k0, T0);                 // A11
  chol_tile(T0, p.status);                       // L11
  inv_tile(T0, T2);                              // D11
  load_tile(S, ld, k0, k0 + kT, T1);             // A12 = A21^T
  mul_tile(T2, T1, T1, 1.f, false);              // L21^T = D11 A12
  load_tile(S, ld, k0 + kT, k0 + kT, T0);        // A22
  {
    // A22 -= L21 L21^T: [r][c] -= sum_q L21^T[q][r] L21^T[q][c] (the upper part is never read)
    const int tid = threadIdx.x, r0 = 4 * (tid >> 4), c0 = 8 * (tid & 15);
    float acc[4][8];
    tile_products(T1, T1, true, acc);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int e = 0; e < 8; ++e) T0[(r0 + i) * kTP + c0 + e] -= acc[i][e];
    __syncthreads();
  }
  chol_tile(T0, p.status);                       // L22
  store_tile_panels(T2, hi, lo, ld, k0, 0);      // D11
  mul_tile(T1, T2, T1, 1.f, true);               // X = L21 D11
  inv_tile(T0, T2);                              // D22
  mul_tile(T2, T1, T0, -1.f, false);             // D21 = -D22 X
  store_tile_panels(T0, hi, lo, ld, k0 + kT, 0);
  store_tile_panels(T2, hi, lo, ld, k0 + kT, kT);
  // the upper-right 128 x 128 of the block inverse is zero
  for (int q = threadIdx.x; q < kT * kT / 8; q += kDiagThreads) {
    const int r = q >> 4, c = 8 * (q & 15);
    const size_t off = panel_chunk_off(k0 + r, kT + c, ld);
    *reinterpret_cast<uint4 *>(hi + off) = make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4 *>(lo + off) = make_uint4(0, 0, 0, 0);
  }
}

}  // namespace

cudaError_t launch_pack_panels(const PackParams &p, cudaStream_t s) {
  if (p.n > 0 && p.blk_begin[p.n] > 0) pack_panels_kernel<<<p.blk_begin[p.n], 256, 0, s>>>(p);
  return cudaGetLastError();
}
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
