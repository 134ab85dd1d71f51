// Newton-Muon preconditioner pieces ("The Newton-Muon Optimizer", abstract: the update
// msgn(G (Z Z^T)^-1), here with a ridge lambda = ridge_rel tr(Z Z^T) / d_in).
//
//   pack_panels   layer input Z (bf16 row-major d x n) -> the tensor-core panel layout,
//                 so that S = Z Z^T runs on the grouped tcgen05 GEMM (fp32 output);
//   ridge         lambda = ridge_rel tr(S) / d, S += lambda I (one CTA per Z, fixed order);
//   potrf_block   Cholesky of the 64 x 64 diagonal block at column k (lower factor, in
//                 place) and the inverse of that factor, which turns each panel and
//                 block solve into a small GEMM.
// The panel solves, the trailing updates and the triangular solves for P = U S^-1 run on
// the fp32 GEMM kernel; the host sequences them.
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
}

// Right-looking unblocked Cholesky of the 64 x 64 diagonal block in shared memory, then
// the inverse of the lower factor by forward substitution (one column per thread).
__global__ void __launch_bounds__(256) potrf_block_kernel(const __grid_constant__ CholParams p) {
  __shared__ float A[64][65];
  __shared__ float Li[64][65];
  const int z = blockIdx.x;
  if (p.k >= p.d[z]) return;
  float *S = reinterpret_cast<float *>(p.ws + p.s_off[z]);
  float *inv = reinterpret_cast<float *>(p.ws + p.inv_off[z]) + (int64_t)(p.k / 64) * 64 * 64;
  const int ld = p.ld[z], k = p.k;
  for (int e = threadIdx.x; e < 64 * 64; e += 256) {
    const int r = e >> 6, c = e & 63;
    A[r][c] = S[(int64_t)(k + r) * ld + k + c];
  }
  __syncthreads();
  for (int j = 0; j < 64; ++j) {
    if (threadIdx.x == 0) {
      float a = A[j][j];
      if (!(a > 0.f)) {           // not positive definite in fp32: flag it, keep going
        set_status(p.status, 0x10u);
        a = 1e-30f;
      }
      A[j][j] = sqrtf(a);
    }
    __syncthreads();
    const float djj = A[j][j];
    for (int i = j + 1 + threadIdx.x; i < 64; i += 256) A[i][j] /= djj;
    __syncthreads();
    const int rem = 63 - j;
    for (int e = threadIdx.x; e < rem * rem; e += 256) {
      const int i = j + 1 + e / rem, c = j + 1 + e % rem;
      if (c <= i) A[i][c] = fmaf(-A[i][j], A[c][j], A[i][c]);
    }
    __syncthreads();
  }
  // Inverse of the lower-triangular factor: L X = I, column c per thread.
  if (threadIdx.x < 64) {
    const int c = threadIdx.x;
    for (int i = 0; i < 64; ++i) {
      float acc = (i == c) ? 1.f : 0.f;
      for (int q = c; q < i; ++q) acc = fmaf(-A[i][q], Li[q][c], acc);
      Li[i][c] = (i >= c) ? acc / A[i][i] : 0.f;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < 64 * 64; e += 256) {
    const int r = e >> 6, c = e & 63;
    S[(int64_t)(k + r) * ld + k + c] = (c <= r) ? A[r][c] : 0.f;
    inv[e] = Li[r][c];
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
cudaError_t launch_potrf_block(const CholParams &p, cudaStream_t s) {
  if (p.n > 0) potrf_block_kernel<<<p.n, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace nshb
