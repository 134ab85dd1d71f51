// Split-precision (bf16 x 3) GEMMs of the Newton-Muon preconditioner on CTA pairs
// ("The Newton-Muon Optimizer", abstract: the update msgn(G (Z Z^T)^-1), here
// P = U (Z Z^T + lambda I)^-1 through a blocked Cholesky factorisation and triangular
// solves whose updates are these products).
//
// Every operand X lives in the workspace as two bf16 panel matrices, X = X_hi + X_lo with
// X_hi = bf16(X) and X_lo = bf16(X - X_hi), so X carries about 16 significant bits.  A
// product accumulates A_hi B_hi + A_hi B_lo + A_lo B_hi in one fp32 TMEM accumulator (the
// A_lo B_lo term is below the fp32 rounding of the sum), three bf16 tensor-core passes
// instead of fp32 arithmetic on the CUDA cores.  With the conditioning of the layer-input
// Gram matrices (about 1e4) this keeps P within ~1e-5 of the fp64 solve, where one bf16
// pass would lose ~4e-3 (measured by emulation on the host).
//
// A problem computes one M x N region D = A B^T (B K-major) or D = A B (B MN-major), or
// D = C - A B^(T) with C an fp32 region, over 256 x 256 output tiles (all of them, or those
// on and below the diagonal).  D goes to an fp32 row-major region and/or back to bf16
// hi/lo panels, ready to be the operand of the next product.  The pipeline is the one of the
// Newton-Schulz pair GEMM: warp 0 of each CTA loads its halves with 2-SM TMA (no multicast)
// into a 3-stage ring, warp 1 of the leader issues tcgen05.mma.cta_group::2 and multicasts
// each commit, warps 2-9 of both CTAs drain double-buffered TMEM accumulators.  Every wait
// is bounded.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "nshb_device.cuh"
#include "nshb_internal.h"

namespace nshb {
namespace {

constexpr int BM = 256, BN = 256, STAGES = 3;
constexpr int SLICE_BYTES = 128 * 64 * 2;         // 16 KB: 128 rows x 64 bf16 (one k panel)
constexpr int HALF_BYTES = 2 * SLICE_BYTES;
constexpr int STAGE_BYTES = 2 * HALF_BYTES;       // A half + B half of one CTA, 128 deep in k
constexpr int TMEM_COLS = 2 * BN;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kTimeoutBit = 0x4u;
constexpr uint32_t kPeerMask = 0xFEFFFFFFu;       // clears the CTA-rank bit of a cluster address
constexpr int kTerms = 3;                          // hi*hi, hi*lo, lo*hi

struct NwTile {
  int prob, m0, n0;
};

__device__ __forceinline__ NwTile nw_decode(const NwParams &p, int tile) {
  int lo = 0, hi = p.nprob - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.prob[mid].tile_begin <= tile) lo = mid; else hi = mid - 1;
  }
  const NwProb &q = p.prob[lo];
  const int l = tile - q.tile_begin;
  NwTile t;
  t.prob = lo;
  t.m0 = (l / q.nt) * BM;
  t.n0 = (l % q.nt) * BN;
  return t;
}

__global__ void __launch_bounds__(kThreads, 1) newton_gemm_kernel(const __grid_constant__ NwParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 4);
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t bar_base = smem_u32(bars);
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (STAGES + s); };
  auto tfull_bar = [&](int b) { return bar_base + 8u * (2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return bar_base + 8u * (2 * STAGES + 2 + b); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cta_rank();
  const bool leader = rank == 0;
  const int cid = (int)cluster_id(), ncl = (int)num_clusters();
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 2 * kEpiWarps);
    }
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc2(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish2();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const long long limit = p.wait_limit;
  if (warp == 0 && lane == 0) prefetch_tmap(&p.tmap);
  pdl_trigger();
  if (!p.late_wait) pdl_wait();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      int last_parity[STAGES];
      for (int s = 0; s < STAGES; ++s) last_parity[s] = -1;
      bool ok = true;
      for (int tile = cid; ok && tile < p.total_tiles; tile += ncl) {
        const NwTile t = nw_decode(p, tile);
        const NwProb &q = p.prob[t.prob];
        const bool bmn = q.flags & kNwBMn;
        const int am = q.a_r0 + t.m0 + 128 * (int)rank;   // this CTA's A rows
        for (int term = 0; ok && term < kTerms; ++term) {
          const int64_t a_row = (term == 2 ? q.a_lo : q.a_hi) >> 7;   // 128-byte rows
          const int64_t b_row = (term == 1 ? q.b_lo : q.b_hi) >> 7;
          for (int kb = 0; kb < q.kt; kb += 2) {
            if (!mbar_wait(empty_bar(stage), phase ^ 1u, limit)) {
              set_status(p.status, kTimeoutBit);
              ok = false;
              break;
            }
            const uint32_t sA = smem_base + stage * STAGE_BYTES, sB = sA + HALF_BYTES;
            const uint32_t fb = full_bar(stage) & kPeerMask;
            if (leader) {
              mbar_arrive_expect_tx(full_bar(stage), 2 * STAGE_BYTES);
              last_parity[stage] = (int)phase;
            }
            const int64_t kp = (q.a_k0 >> 6) + kb;          // A's k panel
            const int64_t ya = a_row + kp * q.a_ph + am;
            tma_load_2sm(sA, &p.tmap, 0, (int)ya, fb);
            tma_load_2sm(sA + SLICE_BYTES, &p.tmap, 0, (int)(ya + q.a_ph), fb);
            if (!bmn) {
              // K-major B: rows (n) b_r0 + n0 + 128 rank of k panels b_k0/64 + kb, +1
              const int64_t yb = b_row + ((q.b_k0 >> 6) + kb) * q.b_ph + q.b_r0 + t.n0 + 128 * (int)rank;
              tma_load_2sm(sB, &p.tmap, 0, (int)yb, fb);
              tma_load_2sm(sB + SLICE_BYTES, &p.tmap, 0, (int)(yb + q.b_ph), fb);
            } else {
              // MN-major B: columns (n) b_r0 + n0 + 128 rank (two 64-column panels), k rows
              // b_k0 + 64 kb .. +127
              const int64_t y0 =
                  b_row + (int64_t)((q.b_r0 + t.n0 + 128 * (int)rank) >> 6) * q.b_ph + q.b_k0 + (int64_t)kb * 64;
              tma_load_2sm(sB, &p.tmap, 0, (int)y0, fb);
              tma_load_2sm(sB + SLICE_BYTES, &p.tmap, 0, (int)(y0 + q.b_ph), fb);
            }
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
      if (leader)
        for (int s = 0; s < STAGES; ++s)
          if (last_parity[s] >= 0 && !mbar_wait(full_bar(s), (uint32_t)last_parity[s], limit))
            set_status(p.status, kTimeoutBit);
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------------------ MMA issuer (leader)
      int stage = 0;
      uint32_t phase = 0;
      int tl = 0;
      bool ok = true;
      for (int tile = cid; ok && tile < p.total_tiles; tile += ncl, ++tl) {
        const NwTile t = nw_decode(p, tile);
        const NwProb &q = p.prob[t.prob];
        const bool bmn = q.flags & kNwBMn;
        const uint32_t idesc = idesc_bf16(BM, BN, 0, bmn ? 1 : 0);
        const int buf = tl & 1;
        const uint32_t tph = (uint32_t)(tl >> 1) & 1u;
        if (!mbar_wait(tempty_bar(buf), tph ^ 1u, limit)) {
          set_status(p.status, kTimeoutBit);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
        bool first = true;
        for (int term = 0; ok && term < kTerms; ++term) {
          for (int kb = 0; kb < q.kt; kb += 2) {
            if (!mbar_wait(full_bar(stage), phase, limit)) {
              set_status(p.status, kTimeoutBit);
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sA = smem_base + stage * STAGE_BYTES, sB = sA + HALF_BYTES;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint32_t kofs = (uint32_t)(k >> 2) * SLICE_BYTES + 32u * (k & 3);
              const uint64_t ad = smem_desc_sw128(sA + kofs, 16, 1024);
              const uint64_t bd = bmn ? smem_desc_sw128(sB + 2048u * k, SLICE_BYTES, 1024)
                                      : smem_desc_sw128(sB + kofs, 16, 1024);
              tc_mma2(d_tmem, ad, bd, idesc, first ? 0u : 1u);
              first = false;
            }
            tc_commit2_mc(empty_bar(stage), 0x3);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        if (ok) tc_commit2_mc(tfull_bar(buf), 0x3);
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue (both CTAs)
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = 128 * (int)rank + quarter * 32 + lane;
    int tl = 0;
    for (int tile = cid; tile < p.total_tiles; tile += ncl, ++tl) {
      const NwTile t = nw_decode(p, tile);
      const NwProb &q = p.prob[t.prob];
      const int buf = tl & 1;
      const uint32_t tph = (uint32_t)(tl >> 1) & 1u;
      const int64_t i = t.m0 + row;                        // row of the output region
      const bool sub = q.c32 >= 0, neg = q.flags & kNwNeg;
      const float *crow = sub ? reinterpret_cast<const float *>(p.ws + q.c32) + i * q.ld32 + t.n0 : nullptr;
      float *drow = q.d32 >= 0 ? reinterpret_cast<float *>(p.ws + q.d32) + i * q.ld32 + t.n0 : nullptr;
      const bool valid = i < q.m_valid;                   // rows past the valid region are not written
      // C of columns col0 .. col0+31 (issued a chunk ahead of its use).  A thread owns one row,
      // so a warp access touches 32 lines: 32-byte accesses move twice the bytes per L1
      // wavefront of 16-byte ones (rows and tiles are 32-byte aligned).
      auto load_c = [&](int col0, float (&c)[32]) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint32_t w[8];
          ld_global_256(crow + col0 + 8 * g, w);
#pragma unroll
          for (int e = 0; e < 8; ++e) c[8 * g + e] = __uint_as_float(w[e]);
        }
      };
      float c[32];
      if (sub) load_c(half * 128, c);                      // in flight while the MMAs finish
      if (!mbar_wait(tfull_bar(buf), tph, limit)) {
        set_status(p.status, kTimeoutBit);
        break;
      }
      tc_fence_after();
#pragma unroll 1
      for (int cc = half * 4; cc < half * 4 + 4; ++cc) {
        const int col0 = cc * 32;                           // column within the tile
        float cn[32];
        if (sub && cc + 1 < half * 4 + 4) load_c(col0 + 32, cn);
        uint32_t r[32];
        tmem_ld32(tmem_base + (uint32_t)(buf * BN + col0) + ((uint32_t)(quarter * 32) << 16), r);
        tmem_ld_wait();
        float v[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = sub ? c[e] - __uint_as_float(r[e]) : neg ? -__uint_as_float(r[e]) : __uint_as_float(r[e]);
        const int cvalid = q.n_valid - (t.n0 + col0);       // columns of this chunk that exist
        if (drow && valid && cvalid >= 32) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            uint32_t w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) w[e] = __float_as_uint(v[8 * g + e]);
            st_global_256(drow + col0 + 8 * g, w);
          }
        } else if (drow && valid) {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (e < cvalid) drow[col0 + e] = v[e];
        }
        if (q.dhi >= 0) {
          const int64_t pr = q.d_r0 + i;                    // row and column in D's panels
          const int64_t pc = q.d_c0 + t.n0 + col0;
          const bool odd = pr & 1;
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            uint32_t h[8], l[8], w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float x0 = v[16 * k + 2 * e], x1 = v[16 * k + 2 * e + 1];
              h[e] = pack_bf16(x0, x1);
              l[e] = pack_bf16(x0 - bf16lo(h[e]), x1 - bf16hi(h[e]));
            }
            const size_t off = panel_pair_off(pr, pc + 16 * k, q.d_ph);
            unswizzle_pair(h, odd, w);
            st_global_256(p.ws + q.dhi + off, w);
            unswizzle_pair(l, odd, w);
            st_global_256(p.ws + q.dlo + off, w);
          }
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) c[e] = cn[e];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) remote_arrive(mapa(tempty_bar(buf), 0));
    }
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem_base, TMEM_COLS);
  }
  // Ran beside the previous kernel: finish only after it, so that the next kernel's wait
  // covers both.
  if (p.late_wait) pdl_wait();
}

}  // namespace

cudaError_t launch_newton_gemm(const NwParams &p, int num_sms, cudaStream_t s, int reserve_pairs) {
  static PerDevice attr_set;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr_set.get(dev)) {
    cudaError_t e = cudaFuncSetAttribute(newton_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set.set(dev, 1);
  }
  if (p.total_tiles <= 0) return cudaSuccess;
  static PerDevice max_pairs;
  int mp = max_pairs.get(dev);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  if (!mp) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (num_sms / 2), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, newton_gemm_kernel, &cfg) != cudaSuccess || n <= 0) {
      (void)cudaGetLastError();
      n = num_sms / 2;
    }
    mp = n < num_sms / 2 ? n : num_sms / 2;
    max_pairs.set(dev, mp);
  }
  const int avail = mp - reserve_pairs > 1 ? mp - reserve_pairs : 1;
  const int clusters = p.total_tiles < avail ? p.total_tiles : avail;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, newton_gemm_kernel, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace nshb
