// fp32 GEMMs on the CUDA cores (the fp32 path: NS in full single precision, used where
// the update must match an fp64 reference to ~1e-4, which rules out bf16 and TF32
// tensor-core inputs).
//
// One launch runs one phase of one NS iteration for every matrix of the call:
//   kGram    A  = s^2 X X^T            (X row-major r x s, wide side)
//   kPoly    B  = b A + c A A
//   kUpdate  X' = s (a X + B X)
// where s = 1 / (||U|| + eps) on the first iteration (the normalisation folded into the
// first Gram and update epilogues) and 1 afterwards ("Muon: the orthogonalized optimizer
// explained", Newton-Schulz section and newton_schulz5).
//
// 128x128 output tiles, 8-deep k slices double-buffered in shared memory, 256 threads
// with an 8x8 register tile each (rows ty*4 + {0..3, 64..67}, columns tx*4 + {0..3,
// 64..67}, so that the shared-memory reads are conflict-free float4s).  Global loads are
// float4 where the rows are 16-byte aligned and the slice lies inside the matrix, scalar
// with zero fill elsewhere.  Deterministic: every output is one fixed-order fp32 dot
// product (k ascending).
#include <cuda_runtime.h>

#include "nshb_device.cuh"
#include "nshb_internal.h"

namespace nshb {
namespace {

constexpr int BM = kF32Tile, BN = kF32Tile, BK = 8;
constexpr int kThreads = 256;

struct Slice {
  float a[4], b[4];   // the thread's share of one k slice of A and B
};

// Thread t loads A rows m0 + t/2, columns k0 + 4 (t % 2) .. +3 (A row-major M x K), and
// B either the same way (b_trans: B stored N x K) or B rows k0 + t/32, columns
// n0 + 4 (t % 32) .. +3 (B stored K x N).
__device__ __forceinline__ void load_slice(const F32Prob &q, const float *A, const float *B, int m0, int n0,
                                           int k0, bool vec_a, bool vec_b, Slice &s) {
  const int t = threadIdx.x;
  {
    const int gi = m0 + (t >> 1), gk = k0 + 4 * (t & 1);
    const float *src = A + (int64_t)gi * q.lda + gk;
    if (vec_a && gi < q.M && gk + 3 < q.K) {
      const float4 v = *reinterpret_cast<const float4 *>(src);
      s.a[0] = v.x; s.a[1] = v.y; s.a[2] = v.z; s.a[3] = v.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) s.a[e] = (gi < q.M && gk + e < q.K) ? src[e] : 0.f;
    }
  }
  if (q.b_trans) {
    const int gj = n0 + (t >> 1), gk = k0 + 4 * (t & 1);
    const float *src = B + (int64_t)gj * q.ldb + gk;
    if (vec_b && gj < q.N && gk + 3 < q.K) {
      const float4 v = *reinterpret_cast<const float4 *>(src);
      s.b[0] = v.x; s.b[1] = v.y; s.b[2] = v.z; s.b[3] = v.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) s.b[e] = (gj < q.N && gk + e < q.K) ? src[e] : 0.f;
    }
  } else {
    const int gk = k0 + (t >> 5), gj = n0 + 4 * (t & 31);
    const float *src = B + (int64_t)gk * q.ldb + gj;
    if (vec_b && gk < q.K && gj + 3 < q.N) {
      const float4 v = *reinterpret_cast<const float4 *>(src);
      s.b[0] = v.x; s.b[1] = v.y; s.b[2] = v.z; s.b[3] = v.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) s.b[e] = (gk < q.K && gj + e < q.N) ? src[e] : 0.f;
    }
  }
}

__device__ __forceinline__ void store_slice(const F32Prob &q, const Slice &s, float (*As)[BM + 4],
                                            float (*Bs)[BN + 4]) {
  const int t = threadIdx.x;
#pragma unroll
  for (int e = 0; e < 4; ++e) As[4 * (t & 1) + e][t >> 1] = s.a[e];
  if (q.b_trans) {
#pragma unroll
    for (int e = 0; e < 4; ++e) Bs[4 * (t & 1) + e][t >> 1] = s.b[e];
  } else {
    *reinterpret_cast<float4 *>(&Bs[t >> 5][4 * (t & 31)]) = make_float4(s.b[0], s.b[1], s.b[2], s.b[3]);
  }
}

// Tile (mi, ni) of local tile index lt, row by row.
__device__ __forceinline__ void decode_tile(const F32Prob &q, int lt, int &mi, int &ni) {
  mi = lt / q.tiles_n;
  ni = lt % q.tiles_n;
}

__global__ void __launch_bounds__(kThreads) gemm_f32_kernel(const __grid_constant__ F32Params p) {
  __shared__ __align__(16) float As[2][BK][BM + 4];
  __shared__ __align__(16) float Bs[2][BK][BN + 4];
  pdl_wait();
  int lo = 0, hi = p.nprob - 1;
  const int tile = blockIdx.x;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (p.prob[mid].tile_begin <= tile) lo = mid; else hi = mid - 1;
  }
  const F32Prob &q = p.prob[lo];
  int mi, ni;
  decode_tile(q, tile - q.tile_begin, mi, ni);
  const int m0 = mi * BM, n0 = ni * BN;
  const float *A = reinterpret_cast<const float *>(p.ws + q.a_off);
  const float *B = reinterpret_cast<const float *>(p.ws + q.b_off);
  const bool vec_a = (q.lda % 4 == 0) && ((reinterpret_cast<uintptr_t>(A) & 15) == 0);
  const bool vec_b = (q.ldb % 4 == 0) && ((reinterpret_cast<uintptr_t>(B) & 15) == 0);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[8][8] = {};
  Slice s;
  load_slice(q, A, B, m0, n0, 0, vec_a, vec_b, s);
  store_slice(q, s, As[0], Bs[0]);
  __syncthreads();
  int buf = 0;
  for (int k0 = 0; k0 < q.K; k0 += BK) {
    const bool more = k0 + BK < q.K;
    if (more) load_slice(q, A, B, m0, n0, k0 + BK, vec_a, vec_b, s);
#pragma unroll
    for (int k = 0; k < BK; ++k) {
      const float4 a0 = *reinterpret_cast<const float4 *>(&As[buf][k][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4 *>(&As[buf][k][ty * 4 + 64]);
      const float4 b0 = *reinterpret_cast<const float4 *>(&Bs[buf][k][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4 *>(&Bs[buf][k][tx * 4 + 64]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int x = 0; x < 8; ++x)
#pragma unroll
        for (int y = 0; y < 8; ++y) acc[x][y] = fmaf(a[x], b[y], acc[x][y]);
    }
    if (more) {
      store_slice(q, s, As[buf ^ 1], Bs[buf ^ 1]);
      __syncthreads();
      buf ^= 1;
    }
  }
  pdl_trigger();
  const float sc = q.scale_idx >= 0 ? p.scales[q.scale_idx] : 1.f;
  const float *C = reinterpret_cast<const float *>(p.ws + q.c_off);
  float *D = reinterpret_cast<float *>(p.ws + q.d_off);
  const bool vec_d = (q.ldc % 4 == 0) && ((reinterpret_cast<uintptr_t>(D) & 15) == 0) &&
                     ((reinterpret_cast<uintptr_t>(C) & 15) == 0);
#pragma unroll
  for (int x = 0; x < 8; ++x) {
    const int gi = m0 + ty * 4 + (x & 3) + (x >> 2) * 64;
    if (gi >= q.M) continue;
#pragma unroll
    for (int yh = 0; yh < 2; ++yh) {
      const int gj0 = n0 + tx * 4 + yh * 64;
      float v[4];
#pragma unroll
      for (int y = 0; y < 4; ++y) {
        const float a = acc[x][4 * yh + y];
        const int64_t o = (int64_t)gi * q.ldc + gj0 + y;
        if (gj0 + y >= q.N) { v[y] = 0.f; continue; }
        if (p.mode == kGram) v[y] = (sc * sc) * a;
        else if (p.mode == kPoly) v[y] = fmaf(p.cb, C[o], p.cc * a);
        else v[y] = sc * fmaf(p.ca, C[o], a);   // kUpdate
      }
      const int64_t o0 = (int64_t)gi * q.ldc + gj0;
      if (vec_d && gj0 + 3 < q.N) {
        *reinterpret_cast<float4 *>(D + o0) = make_float4(v[0], v[1], v[2], v[3]);
      } else {
#pragma unroll
        for (int y = 0; y < 4; ++y)
          if (gj0 + y < q.N) D[o0 + y] = v[y];
      }
    }
  }
}

}  // namespace

cudaError_t launch_gemm_f32(const F32Params &p, cudaStream_t s) {
  if (p.total_tiles > 0) return launch_pdl(gemm_f32_kernel, p.total_tiles, kThreads, 0, s, p);
  return cudaGetLastError();
}

}  // namespace nshb
