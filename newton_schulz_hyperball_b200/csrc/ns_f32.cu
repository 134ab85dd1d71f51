// fp32 Newton-Schulz GEMMs on the CUDA cores (the fp32 path: NS in full single
// precision, used where the update must match an fp64 reference to ~1e-4, which rules
// out bf16 and TF32 tensor-core inputs).
//
// One launch runs one phase of one NS iteration for every matrix of the call:
//   kGram    A  = s^2 X X^T            (X row-major r x s, wide side)
//   kPoly    B  = b A + c A A
//   kUpdate  X' = s (a X + B X)
// where s = 1 / (||U|| + eps) on the first iteration (the normalisation folded into the
// first Gram and update epilogues) and 1 afterwards ("Muon: the orthogonalized optimizer
// explained", Newton-Schulz section and newton_schulz5).  The same kernel also computes the
// plain product D = A B and the update D = C - A B of the Newton-Muon Cholesky
// factorisation and triangular solves.
//
// 64x64 output tiles, 16-deep k slices staged in shared memory, 256 threads with a 4x4
// register tile each.  Deterministic: every output is one fixed-order fp32 dot product.
#include <cuda_runtime.h>

#include "nshb_internal.h"

namespace nshb {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

__global__ void __launch_bounds__(256) gemm_f32_kernel(const __grid_constant__ F32Params p) {
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN + 4];
  int lo = 0, hi = p.nprob - 1;
  const int tile = blockIdx.x;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (p.prob[mid].tile_begin <= tile) lo = mid; else hi = mid - 1;
  }
  const F32Prob &q = p.prob[lo];
  const int lt = tile - q.tile_begin;
  const int m0 = (lt / q.tiles_n) * TM, n0 = (lt % q.tiles_n) * TN;
  const float *A = reinterpret_cast<const float *>(p.ws + q.a_off);
  const float *B = reinterpret_cast<const float *>(p.ws + q.b_off);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < q.K; k0 += TK) {
    for (int e = threadIdx.x; e < TM * TK; e += 256) {
      const int r = e / TK, k = e % TK;
      const int gi = m0 + r, gk = k0 + k;
      As[k][r] = (gi < q.M && gk < q.K) ? A[(int64_t)gi * q.lda + gk] : 0.f;
    }
    for (int e = threadIdx.x; e < TN * TK; e += 256) {
      int c, k;
      if (q.b_trans) { c = e / TK; k = e % TK; } else { k = e / TN; c = e % TN; }
      const int gj = n0 + c, gk = k0 + k;
      float v = 0.f;
      if (gj < q.N && gk < q.K) v = q.b_trans ? B[(int64_t)gj * q.ldb + gk] : B[(int64_t)gk * q.ldb + gj];
      Bs[k][c] = v;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < TK; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int x = 0; x < 4; ++x) a[x] = As[k][ty * 4 + x];
#pragma unroll
      for (int y = 0; y < 4; ++y) b[y] = Bs[k][tx * 4 + y];
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(a[x], b[y], acc[x][y]);
    }
    __syncthreads();
  }
  const float s = q.scale_idx >= 0 ? p.scales[q.scale_idx] : 1.f;
  const float *C = reinterpret_cast<const float *>(p.ws + q.c_off);
  float *D = reinterpret_cast<float *>(p.ws + q.d_off);
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    const int gi = m0 + ty * 4 + x;
    if (gi >= q.M) continue;
#pragma unroll
    for (int y = 0; y < 4; ++y) {
      const int gj = n0 + tx * 4 + y;
      if (gj >= q.N) continue;
      const int64_t o = (int64_t)gi * q.ldc + gj;
      float v;
      if (p.mode == kGram) v = (s * s) * acc[x][y];
      else if (p.mode == kPoly) v = fmaf(p.cb, C[o], p.cc * acc[x][y]);
      else if (p.mode == kUpdate) v = s * fmaf(p.ca, C[o], acc[x][y]);
      else if (p.mode == kSub) v = C[o] - acc[x][y];
      else v = acc[x][y];
      D[o] = v;
    }
  }
}

}  // namespace

cudaError_t launch_gemm_f32(const F32Params &p, cudaStream_t s) {
  if (p.total_tiles > 0) gemm_f32_kernel<<<p.total_tiles, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace nshb
