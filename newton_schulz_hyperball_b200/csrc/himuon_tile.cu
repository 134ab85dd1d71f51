// Hierarchical Muon with T = 256: the whole Newton-Schulz chain of one tile on one CTA
// pair, with the tile resident in shared and tensor memory.
// ("Hierarchical Muon: Tiled Newton-Schulz Updates", abstract: the same finite NS map
//  run independently on every T x T tile; "Muon: the orthogonalized optimizer
//  explained", Newton-Schulz section: A = X X^T, B = b A + c A^2, X <- a X + B X.)
//
// Why a separate kernel: with T = 256 one phase of one tile is about 1.5 us of
// tensor-core work, but as three grouped GEMM launches per iteration every phase
// reloads 128 KB of operands per CTA and writes its result back to memory, and a
// tile-phase takes 5.5-8 us.  Here a pair loads X once and runs, per iteration:
//   Gram    A = s^2 X X^T        -> TMEM columns [0, 256)   (operands: sXown, K-major)
//   epi 1   A -> bf16 sA                                  (A stays in TMEM in fp32)
//   poly    A^2 = A A            -> TMEM columns [256, 512) (operands: sA; A is symmetric)
//   epi 2   B = b A + c A^2 from the fp32 accumulators -> bf16 sA
//   update  B X                  -> TMEM columns [0, 256)   (sA K-major, sXcol MN-major)
//   epi 3   X' = s (a X + B X) -> own rows of sXown, the own column half of sXcol, and
//           the partner's column half of its sXcol (distributed shared memory).
// Only the first X, the low parts of the compensated iterations and the final O touch
// global memory.  The factor s (1 / (||tile|| + eps)) applies in the first iteration.
//
// Shared memory per CTA r (0 = leader): sXown 64 KB = X rows 128r .. 128r+127 (four
// 64-column panels of 128 rows, the tensor core's 128-byte swizzled image), sXcol 64 KB =
// X columns 128r .. 128r+127 over all 256 rows (two panels of 256 rows), sA 64 KB (this
// CTA's 128 rows of A, then of B).  A cta_group::2 MMA reads the same shared-memory
// offset in both CTAs, so each CTA keeps its own half at offset 0.
//
// Roles (320 threads per CTA): warp 0 loads X (TMA onto a local barrier, then tells the
// leader), warp 1 of the leader issues the MMAs and multicasts each commit, warps 2-9 of
// both CTAs run the epilogues on their 128 accumulator rows (lane quarter = warp % 4,
// column half = (warp - 2) / 4) and report to the leader.  Tiles are walked statically
// by the persistent grid.  Every wait is bounded; no load is multicast.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "nshb_device.cuh"
#include "nshb_internal.h"

namespace nshb {
namespace {

constexpr int T = 256;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kPanel128 = 128 * 128;            // 64 columns x 128 rows of bf16: 16 KB
constexpr int kPanel256 = 256 * 128;            // 64 columns x 256 rows: 32 KB
constexpr int kHalf = 4 * kPanel128;            // 64 KB
constexpr int SMEM_BYTES = 3 * kHalf + 1024 + 256;
constexpr uint32_t kTimeoutBit = 0x4u;

// 2-D TMA load into this CTA's shared memory, completing on this CTA's barrier.
__device__ __forceinline__ void tma_load_local(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}
// Generic-proxy shared-memory writes become visible to the tensor core (async proxy): this
// CTA's shared memory, or any shared memory of the cluster (writes into the partner's).
__device__ __forceinline__ void fence_proxy_async_cta() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_cluster() {
  asm volatile("fence.proxy.async.shared::cluster;" ::: "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, const uint32_t *w) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3])
               : "memory");
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, const uint32_t *w) {
  asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[0]), "r"(w[1]), "r"(w[2]),
               "r"(w[3])
               : "memory");
}
__device__ __forceinline__ void ld_shared_v4(uint32_t addr, uint32_t *w) {
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
               : "r"(addr)
               : "memory");
}

// Byte offset in a K-major half (sA, sXown: 128 rows, four 64-column panels) of the 16-byte
// chunk holding row rl, columns j .. j+7.
__device__ __forceinline__ uint32_t half_chunk(int rl, int j) {
  return (uint32_t)((j >> 6) * kPanel128 + rl * 128 + ((((j >> 3) & 7) ^ (rl & 7)) << 4));
}
// ... and in a column half (sXcol: 256 rows, two panels), row g, columns jj .. jj+7 (jj < 128).
__device__ __forceinline__ uint32_t col_chunk(int g, int jj) {
  return (uint32_t)((jj >> 6) * kPanel256 + g * 128 + ((((jj >> 3) & 7) ^ (g & 7)) << 4));
}

// The caller's bf16 W at row wr, columns wc .. wc+31 as 16 pairs in logical order (zero
// outside the matrix; fp32 weights take the reduce pass).  Loaded a chunk ahead of use.
__device__ __forceinline__ void w_load(const HmProb &q, int64_t wr, int64_t wc, uint32_t (&wv)[16]) {
  const bool rin = wr < q.w_m;
  const unsigned short *row = static_cast<const unsigned short *>(q.w) + wr * q.w_ld;
  if (rin && wc + 31 < q.w_n && (q.w_flags & kPwVec)) {
    const uint4 *src = reinterpret_cast<const uint4 *>(row + wc);
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const uint4 u = src[g];
      wv[4 * g] = u.x; wv[4 * g + 1] = u.y; wv[4 * g + 2] = u.z; wv[4 * g + 3] = u.w;
    }
  } else {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const uint32_t lo = (rin && wc + 2 * e < q.w_n) ? (uint32_t)row[wc + 2 * e] : 0u;
      const uint32_t hi = (rin && wc + 2 * e + 1 < q.w_n) ? (uint32_t)row[wc + 2 * e + 1] : 0u;
      wv[e] = lo | (hi << 16);
    }
  }
}

// Adds the (||O||^2, <W,O>, ||W||^2) terms of 32 elements of a tile row: O as stored (bf16
// pairs hw) and W (pairs wv, both in logical order).  fp32 terms over the 32 elements,
// added to the thread's fp64 sums.
__device__ __forceinline__ void w_partials(const uint32_t (&wv)[16], const uint32_t (&hw)[16], double &dom,
                                           double &dde, double &dpi) {
  float om = 0.f, de = 0.f, pi = 0.f;
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const float w0 = bf16lo(wv[e]), w1 = bf16hi(wv[e]);
    const float o0 = bf16lo(hw[e]), o1 = bf16hi(hw[e]);
    om = fmaf(o0, o0, fmaf(o1, o1, om));
    de = fmaf(w0, o0, fmaf(w1, o1, de));
    pi = fmaf(w0, w0, fmaf(w1, w1, pi));
  }
  dom += (double)om;
  dde += (double)de;
  dpi += (double)pi;
}

// Pulls the thread's W row segment (ncol elements from column wc) into L2 ahead of use.
__device__ __forceinline__ void w_prefetch(const HmProb &q, int64_t wr, int64_t wc, int ncol) {
  if (wr >= q.w_m || wc >= q.w_n) return;
  const char *base = static_cast<const char *>(q.w) + (wr * q.w_ld + wc) * 2;
  for (int b = 0; b < ncol * 2; b += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(base + b));
}

// One (||O||^2, <W,O>, ||W||^2) record per epilogue warp: the warp's fp64 sums in fixed order.
__device__ __forceinline__ void w_record(double *partials, int64_t rec, double dom, double dde, double dpi) {
  dom = warp_sum(dom);
  dde = warp_sum(dde);
  dpi = warp_sum(dpi);
  if ((threadIdx.x & 31) == 0) {
    partials[3 * rec] = dom;
    partials[3 * rec + 1] = dde;
    partials[3 * rec + 2] = dpi;
  }
}

__device__ __forceinline__ int find_prob(const HmParams &p, int tile) {
  int lo = 0, hi = p.nprob - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.prob[mid].tile_begin <= tile) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__global__ void __launch_bounds__(kThreads, 1) himuon_tile_kernel(const __grid_constant__ HmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sXown = smem_u32(smem), sXcol = sXown + kHalf, sA = sXcol + kHalf;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + 3 * kHalf);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 12);   // after the nine barriers
  const uint32_t bar_base = smem_u32(bars);
  const uint32_t xfull = bar_base, xfree = bar_base + 8, mmadone = bar_base + 16;
  const uint32_t xready = bar_base + 24;                          // used in the leader only
  const uint32_t stallbar = bar_base + 32;                        // test stall (leader only)
  // pready[p]: the epilogues have written 64-column panel p of the next phase's operand
  // (in the leader only; four warps of each CTA write a panel)
  auto pready = [&](int pnl) { return bar_base + 40 + 8u * pnl; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cta_rank();
  const bool leader = rank == 0;
  const int cid = (int)cluster_id(), ncl = (int)num_clusters();
  if (threadIdx.x == 0) {
    mbar_init(xfull, 1);
    mbar_init(xfree, 1);
    mbar_init(mmadone, 1);
    mbar_init(xready, 2);                 // both producers
    for (int pnl = 0; pnl < 4; ++pnl) mbar_init(pready(pnl), kEpiWarps);   // 4 warps x 2 CTAs
    mbar_init(stallbar, 1);
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc2(smem_u32(tmem_slot), 512);
    tmem_relinquish2();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const long long limit = p.wait_limit;
  if (warp == 0 && lane == 0) prefetch_tmap(&p.tmap);
  pdl_trigger();
  pdl_wait();                             // X0, its low part and the scales are written
  const int K = p.ns_steps;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer (both CTAs)
      uint32_t ph_f = 0, ph_x = 0;
      for (int tile = cid; tile < p.total_tiles; tile += ncl) {
        if (!mbar_wait(xfree, ph_f ^ 1u, limit)) {
          set_status(p.status, kTimeoutBit);
          break;
        }
        ph_f ^= 1u;
        const HmProb &q = p.prob[find_prob(p, tile)];
        const int64_t base = (q.x0 + (int64_t)(tile - q.tile_begin) * T * T * 2) >> 7;   // 128-byte rows
        mbar_arrive_expect_tx(xfull, 2 * kHalf);
#pragma unroll
        for (int pnl = 0; pnl < 4; ++pnl)   // own rows, all four panels
          tma_load_local(sXown + pnl * kPanel128, &p.tmap, 0, (int)(base + pnl * T + 128 * rank), xfull);
#pragma unroll
        for (int pp = 0; pp < 2; ++pp)      // own two panels, all rows
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
            tma_load_local(sXcol + pp * kPanel256 + hh * kPanel128, &p.tmap, 0,
                           (int)(base + (2 * rank + pp) * T + 128 * hh), xfull);
        if (!mbar_wait(xfull, ph_x, limit)) {
          set_status(p.status, kTimeoutBit);
          break;
        }
        ph_x ^= 1u;
        remote_arrive(mapa(xready, 0));
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------------------ MMA issuer (leader)
      const uint32_t idesc_k = idesc_bf16(2 * 128, T, 0, 0), idesc_mn = idesc_bf16(2 * 128, T, 0, 1);
      // A phase's MMAs go panel by panel (64 k columns: 4 MMAs) in the order the epilogue
      // warps finish them: warps of column half 0 write panels 0 then 1, those of half 1
      // panels 2 then 3.  Accumulators alternate between TMEM columns [0, 256) and
      // [256, 512) from phase to phase, so a phase never writes what the epilogue of the
      // previous phase is still reading.
      constexpr int kOrder[4] = {0, 2, 1, 3};
      uint32_t ph_r = 0, ph_p = 0;
      bool ok = true;
      auto wait_panel = [&](int pnl) {
        if (!mbar_wait(pready(pnl), ph_p, limit)) {
          set_status(p.status, kTimeoutBit);
          ok = false;
        }
        tc_fence_after();
      };
      auto wait_all_panels = [&]() {
        for (int pnl = 0; ok && pnl < 4; ++pnl) wait_panel(pnl);
        ph_p ^= 1u;
      };
      for (int tile = cid, tl = 0; ok && tile < p.total_tiles; tile += ncl, ++tl) {
        if (!mbar_wait(xready, ph_r, limit)) {
          set_status(p.status, kTimeoutBit);
          break;
        }
        ph_r ^= 1u;
        tc_fence_after();
        for (int it = 0; ok && it < K; ++it) {
          const uint32_t dg = tmem_base + (uint32_t)(((3 * it) & 1) * T);
          const uint32_t dq = tmem_base + (uint32_t)(((3 * it + 1) & 1) * T);
          const uint32_t du = tmem_base + (uint32_t)(((3 * it + 2) & 1) * T);
          // Gram: A = X X^T (X' of the previous epilogue 3, or X0 from the producer)
          for (int o = 0; ok && o < 4; ++o) {
            const int pnl = kOrder[o];
            if (it > 0) wait_panel(pnl);
            if (!ok) break;
#pragma unroll
            for (int k = 4 * pnl; k < 4 * pnl + 4; ++k) {
              const uint32_t kofs = (uint32_t)(k >> 2) * kPanel128 + 32u * (k & 3);
              const uint64_t d = smem_desc_sw128(sXown + kofs, 16, 1024);
              tc_mma2(dg, d, d, idesc_k, k != 0);
            }
          }
          if (it > 0) ph_p ^= 1u;
          if (!ok) break;
          if (p.test_stall && tl == 0 && it == 0) {
            // Test stall: the epilogues never hear of this accumulator, so their bounded
            // wait runs out.  The MMAs still complete (on a barrier of the leader only)
            // before this thread goes on, so none is in flight when the CTAs leave.
            tc_commit2_mc(stallbar, 0x1);
            if (!mbar_wait(stallbar, 0, limit)) set_status(p.status, kTimeoutBit);
          } else {
            tc_commit2_mc(mmadone, 0x3);
          }
          // A^2 = A A^T (A symmetric), panel by panel as epilogue 1 writes A to sA
          for (int o = 0; ok && o < 4; ++o) {
            const int pnl = kOrder[o];
            wait_panel(pnl);
            if (!ok) break;
#pragma unroll
            for (int k = 4 * pnl; k < 4 * pnl + 4; ++k) {
              const uint32_t kofs = (uint32_t)(k >> 2) * kPanel128 + 32u * (k & 3);
              const uint64_t d = smem_desc_sw128(sA + kofs, 16, 1024);
              tc_mma2(dq, d, d, idesc_k, k != 0);
            }
          }
          ph_p ^= 1u;
          if (!ok) break;
          tc_commit2_mc(mmadone, 0x3);
          // B X: B K-major (panels of sA as epilogue 2 writes them), X MN-major (16 rows of
          // sXcol per step)
          for (int o = 0; ok && o < 4; ++o) {
            const int pnl = kOrder[o];
            wait_panel(pnl);
            if (!ok) break;
#pragma unroll
            for (int k = 4 * pnl; k < 4 * pnl + 4; ++k) {
              const uint32_t kofs = (uint32_t)(k >> 2) * kPanel128 + 32u * (k & 3);
              const uint64_t ad = smem_desc_sw128(sA + kofs, 16, 1024);
              const uint64_t bd = smem_desc_sw128(sXcol + 2048u * k, kPanel256, 1024);
              tc_mma2(du, ad, bd, idesc_mn, k != 0);
            }
          }
          ph_p ^= 1u;
          if (!ok) break;
          tc_commit2_mc(mmadone, 0x3);
        }
        if (!ok) break;
        wait_all_panels();   // the tile's last epilogue is done with sXown and the TMEM
        if (!ok) break;
        remote_arrive(mapa(xfree, 0));
        remote_arrive(mapa(xfree, 1));
      }
    }
  } else {
    // -------------------------------------------------------------- epilogues (both CTAs)
    const int quarter = warp & 3;                      // TMEM lanes 32 quarter .. +31
    const int half = (warp - 2) >> 2;                  // columns 128 half .. +127
    const int rl = quarter * 32 + lane;                // row within this CTA's half
    const int g = 128 * (int)rank + rl;                // row within the tile
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const bool odd = g & 1;
    const bool own_cols = half == (int)rank;           // sXcol columns of this half live here
    uint32_t ph_x = 0, ph_m = 0;
    bool ok = true;
    auto wait_mma = [&]() {
      if (!mbar_wait(mmadone, ph_m, limit)) {
        if (lane == 0) set_status(p.status, kTimeoutBit);
        ok = false;
      }
      ph_m ^= 1u;
      tc_fence_after();
    };
    // This warp's rows of panel pnl are written (shared memory of this CTA, or also the
    // partner's): the MMA issuer may read the panel.
    auto report = [&](int pnl, bool partner_smem) {
      if (partner_smem) fence_proxy_async_cluster(); else fence_proxy_async_cta();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) remote_arrive(mapa(pready(pnl), 0));
    };
    for (int tile = cid; ok && tile < p.total_tiles; tile += ncl) {
      const HmProb &q = p.prob[find_prob(p, tile)];
      const int t = tile - q.tile_begin;
      const int64_t toff = (int64_t)t * T * T * 2;
      const float s = p.scales[q.seg_begin + t];
      // Hyperball partials: this thread's W row and the first column of its half
      const bool wp = p.partials != nullptr && q.w != nullptr;
      const int64_t wr = (int64_t)(t / q.w_tiles_c) * T + g;
      const int64_t wc = (int64_t)(t % q.w_tiles_c) * T + 128 * half;
      double dom = 0.0, dde = 0.0, dpi = 0.0;
      if (!mbar_wait(xfull, ph_x, limit)) {            // sXown holds X0 (read by epilogue 3)
        if (lane == 0) set_status(p.status, kTimeoutBit);
        break;
      }
      ph_x ^= 1u;
      for (int it = 0; ok && it < K; ++it) {
        const float ca = p.coef[it][0], cb = p.coef[it][1], cc = p.coef[it][2];
        const float s2 = it == 0 ? s * s : 1.0f, ks = it == 0 ? s : 1.0f;
        // TMEM columns of this iteration's three accumulators (they alternate by phase)
        const uint32_t rg = (uint32_t)(((3 * it) & 1) * T), rq0 = (uint32_t)(((3 * it + 1) & 1) * T);
        const uint32_t ru = (uint32_t)(((3 * it + 2) & 1) * T);
        if (wp && it + 1 == K) w_prefetch(q, wr, wc, 128);
        if (it < p.comp) {
          // epilogue 3 reads this thread's row of X's low part: pull it into L2 now
          const char *lo = p.ws + ((it % 2 == 0) ? q.xl0 : q.xl1) + toff;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(lo + panel_pair_off(g, 128 * half + 32 * k, T)));
        }
        // ---- epilogue 1: A -> sA (bf16)
        wait_mma();
        if (!ok) break;
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
          const int j0 = 128 * half + 32 * ch;
          uint32_t r[32];
          tmem_ld32(tmem_base + rg + (uint32_t)j0 + lane_off, r);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              w[e] = pack_bf16(s2 * __uint_as_float(r[8 * c + 2 * e]), s2 * __uint_as_float(r[8 * c + 2 * e + 1]));
            st_shared_v4(sA + half_chunk(rl, j0 + 8 * c), w);
          }
          if (ch & 1) report(2 * half + (ch >> 1), false);
        }
        // ---- epilogue 2: B = b A + c A^2 -> sA (bf16); A is the bf16 copy this thread wrote
        // to sA (the TMEM copy is being overwritten by the update), A^2 from TMEM in fp32
        wait_mma();
        if (!ok) break;
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
          const int j0 = 128 * half + 32 * ch;
          uint32_t rq[32], aw[16];
          tmem_ld32(tmem_base + rq0 + (uint32_t)j0 + lane_off, rq);
#pragma unroll
          for (int c = 0; c < 4; ++c) ld_shared_v4(sA + half_chunk(rl, j0 + 8 * c), aw + 4 * c);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i0 = 8 * c + 2 * e;
              w[e] = pack_bf16(fmaf(cb, bf16lo(aw[4 * c + e]), cc * __uint_as_float(rq[i0])),
                               fmaf(cb, bf16hi(aw[4 * c + e]), cc * __uint_as_float(rq[i0 + 1])));
            }
            st_shared_v4(sA + half_chunk(rl, j0 + 8 * c), w);
          }
          if (ch & 1) report(2 * half + (ch >> 1), false);
        }
        // ---- epilogue 3: X' = s (a X + B X)
        const bool last = it + 1 == K;
        const bool wlast = wp && last;
        uint32_t wv[16];
        if (wlast) w_load(q, wr, wc, wv);       // in flight while the update MMAs run
        wait_mma();
        if (!ok) break;
        const char *clo = it < p.comp ? p.ws + ((it % 2 == 0) ? q.xl0 : q.xl1) + toff : nullptr;
        char *dlo = (it + 1 < p.comp) ? p.ws + ((it % 2 == 0) ? q.xl1 : q.xl0) + toff : nullptr;
        char *dout = last ? p.ws + q.xo + toff : nullptr;
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
          const int j0 = 128 * half + 32 * ch;
          uint32_t wn[16];
          if (wlast && ch < 3) w_load(q, wr, wc + 32 * (ch + 1), wn);
          uint32_t r[32];
          tmem_ld32(tmem_base + ru + (uint32_t)j0 + lane_off, r);
          uint32_t xw[16], lw[16];
#pragma unroll
          for (int c = 0; c < 4; ++c) ld_shared_v4(sXown + half_chunk(rl, j0 + 8 * c), xw + 4 * c);
          if (clo) {
#pragma unroll
            for (int k = 0; k < 2; ++k) {
              uint32_t w8[8];
              ld_global_256(clo + panel_pair_off(g, j0 + 16 * k, T), w8);
              unswizzle_pair(w8, odd, lw + 8 * k);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) lw[e] = 0u;
          }
          tmem_ld_wait();
          uint32_t hw[16], low[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float x0 = bf16lo(xw[e]) + bf16lo(lw[e]), x1 = bf16hi(xw[e]) + bf16hi(lw[e]);
            const float v0 = ks * fmaf(ca, x0, __uint_as_float(r[2 * e]));
            const float v1 = ks * fmaf(ca, x1, __uint_as_float(r[2 * e + 1]));
            hw[e] = pack_bf16(v0, v1);
            low[e] = pack_bf16(v0 - bf16lo(hw[e]), v1 - bf16hi(hw[e]));
          }
          if (last) {
#pragma unroll
            for (int k = 0; k < 2; ++k) {
              uint32_t in8[8], w8[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) in8[e] = hw[8 * k + e];
              unswizzle_pair(in8, odd, w8);
              st_global_256(dout + panel_pair_off(g, j0 + 16 * k, T), w8);
            }
            if (wp) {
              w_partials(wv, hw, dom, dde, dpi);
#pragma unroll
              for (int e = 0; e < 16; ++e) wv[e] = wn[e];
            }
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              st_shared_v4(sXown + half_chunk(rl, j0 + 8 * c), hw + 4 * c);
              const uint32_t a = sXcol + col_chunk(g, j0 + 8 * c - 128 * half);
              if (own_cols) st_shared_v4(a, hw + 4 * c);
              else st_cluster_v4(mapa(a, rank ^ 1u), hw + 4 * c);
            }
            if (dlo) {
#pragma unroll
              for (int k = 0; k < 2; ++k) {
                uint32_t in8[8], w8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) in8[e] = low[8 * k + e];
                unswizzle_pair(in8, odd, w8);
                st_global_256(dlo + panel_pair_off(g, j0 + 16 * k, T), w8);
              }
            }
          }
          // sXown (own CTA) is what the next Gram reads; the partner's sXcol, written in every
          // chunk, is read by the next update, after this warp's second report: one
          // cluster-scope fence before that report covers it.
          if (ch & 1) report(2 * half + (ch >> 1), !last && ch == 3);
        }
      }
      if (ok && wp)
        w_record(p.partials, (int64_t)q.part_begin + (int64_t)t * (2 * kEpiWarps) + rank * kEpiWarps + (warp - 2),
                 dom, dde, dpi);
    }
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync();                         // no CTA leaves while its partner may still
                                          // read or write its shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem_base, 512);
  }
}

// ---------------------------------------------------------------------------- T = 128
// One CTA holds a whole 128 x 128 tile: sX (two 64-column panels of 128 rows, 32 KB)
// serves as the K-major Gram operand and as the MN-major update operand; sA (32 KB) holds
// A, then B; TMEM columns [0, 128) take A and then B X, [128, 256) take A^2, so B = b A +
// c A^2 is formed from the fp32 accumulators.  Two CTAs share an SM (64 KB of shared
// memory and 256 TMEM columns each), so one tile's epilogues overlap the other's MMAs
// (three per SM, with A taken from its bf16 copy, measured no faster).  192 threads:
// warp 0 loads X, warp 1 issues the MMAs, warps 2-5 run the epilogues (lane quarter =
// warp % 4, all 128 columns).
constexpr int T1 = 128;
constexpr int kThreads1 = 64 + 32 * 4;
constexpr int kTile1 = 2 * kPanel128;                 // 32 KB
// 64 KB of operands are used; asking for 100 KB keeps a third CTA off the SM, whose TMEM
// allocation would otherwise wait for a neighbour's whole tile loop.
constexpr int SMEM_BYTES1 = 100 * 1024;
constexpr int kCtasPerSm1 = 2;
static_assert(2 * kTile1 + 1024 + 256 <= SMEM_BYTES1, "shared memory of the T = 128 kernel");

__global__ void __launch_bounds__(kThreads1, kCtasPerSm1) himuon_tile128_kernel(const __grid_constant__ HmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sX = smem_u32(smem), sA = sX + kTile1;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + 2 * kTile1);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 8);
  const uint32_t bar_base = smem_u32(bars);
  const uint32_t xfull = bar_base, xfree = bar_base + 8, mmadone = bar_base + 16, opnd = bar_base + 24;
  const uint32_t stallbar = bar_base + 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(xfull, 1);
    mbar_init(xfree, 1);
    mbar_init(mmadone, 1);
    mbar_init(opnd, 4);                   // the four epilogue warps
    mbar_init(stallbar, 1);
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const long long limit = p.wait_limit;
  if (warp == 0 && lane == 0) prefetch_tmap(&p.tmap);
  pdl_trigger();
  pdl_wait();
  const int K = p.ns_steps;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t ph_f = 0;
      for (int tile = blockIdx.x; tile < p.total_tiles; tile += gridDim.x) {
        if (!mbar_wait(xfree, ph_f ^ 1u, limit)) {
          set_status(p.status, kTimeoutBit);
          break;
        }
        ph_f ^= 1u;
        const HmProb &q = p.prob[find_prob(p, tile)];
        const int64_t base = (q.x0 + (int64_t)(tile - q.tile_begin) * T1 * T1 * 2) >> 7;
        mbar_arrive_expect_tx(xfull, kTile1);
        tma_load_local(sX, &p.tmap, 0, (int)base, xfull);
        tma_load_local(sX + kPanel128, &p.tmap, 0, (int)(base + T1), xfull);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc_k = idesc_bf16(T1, T1, 0, 0), idesc_mn = idesc_bf16(T1, T1, 0, 1);
      uint32_t ph_x = 0, ph_o = 0;
      bool ok = true;
      auto wait_opnd = [&]() {
        if (!mbar_wait(opnd, ph_o, limit)) {
          set_status(p.status, kTimeoutBit);
          ok = false;
        }
        ph_o ^= 1u;
        tc_fence_after();
      };
      for (int tile = blockIdx.x, tl = 0; ok && tile < p.total_tiles; tile += gridDim.x, ++tl) {
        if (!mbar_wait(xfull, ph_x, limit)) {
          set_status(p.status, kTimeoutBit);
          break;
        }
        ph_x ^= 1u;
        tc_fence_after();
        for (int it = 0; ok && it < K; ++it) {
          if (it > 0) {
            wait_opnd();
            if (!ok) break;
          }
#pragma unroll
          for (int k = 0; k < T1 / 16; ++k) {
            const uint32_t kofs = (uint32_t)(k >> 2) * kPanel128 + 32u * (k & 3);
            const uint64_t d = smem_desc_sw128(sX + kofs, 16, 1024);
            tc_mma(tmem_base, d, d, idesc_k, k != 0);
          }
          if (p.test_stall && tl == 0 && it == 0) {
            // Test stall, as in the T = 256 kernel: the MMAs complete on a spare barrier.
            tc_commit(stallbar);
            if (!mbar_wait(stallbar, 0, limit)) set_status(p.status, kTimeoutBit);
          } else {
            tc_commit(mmadone);
          }
          wait_opnd();
          if (!ok) break;
#pragma unroll
          for (int k = 0; k < T1 / 16; ++k) {
            const uint32_t kofs = (uint32_t)(k >> 2) * kPanel128 + 32u * (k & 3);
            const uint64_t d = smem_desc_sw128(sA + kofs, 16, 1024);
            tc_mma(tmem_base + T1, d, d, idesc_k, k != 0);
          }
          tc_commit(mmadone);
          wait_opnd();
          if (!ok) break;
#pragma unroll
          for (int k = 0; k < T1 / 16; ++k) {
            const uint32_t kofs = (uint32_t)(k >> 2) * kPanel128 + 32u * (k & 3);
            const uint64_t ad = smem_desc_sw128(sA + kofs, 16, 1024);
            const uint64_t bd = smem_desc_sw128(sX + 2048u * k, kPanel128, 1024);
            tc_mma(tmem_base, ad, bd, idesc_mn, k != 0);
          }
          tc_commit(mmadone);
        }
        if (!ok) break;
        wait_opnd();
        if (!ok) break;
        mbar_arrive(xfree);
      }
    }
  } else {
    const int quarter = warp & 3;
    const int rl = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const bool odd = rl & 1;
    uint32_t ph_x = 0, ph_m = 0;
    bool ok = true;
    auto wait_mma = [&]() {
      if (!mbar_wait(mmadone, ph_m, limit)) {
        if (lane == 0) set_status(p.status, kTimeoutBit);
        ok = false;
      }
      ph_m ^= 1u;
      tc_fence_after();
    };
    auto report = [&]() {
      fence_proxy_async_cta();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(opnd);
    };
    for (int tile = blockIdx.x; ok && tile < p.total_tiles; tile += gridDim.x) {
      const HmProb &q = p.prob[find_prob(p, tile)];
      const int t = tile - q.tile_begin;
      const int64_t toff = (int64_t)t * T1 * T1 * 2;
      const float s = p.scales[q.seg_begin + t];
      const bool wp = p.partials != nullptr && q.w != nullptr;
      const int64_t wr = (int64_t)(t / q.w_tiles_c) * T1 + rl;
      const int64_t wc = (int64_t)(t % q.w_tiles_c) * T1;
      double dom = 0.0, dde = 0.0, dpi = 0.0;
      if (!mbar_wait(xfull, ph_x, limit)) {
        if (lane == 0) set_status(p.status, kTimeoutBit);
        break;
      }
      ph_x ^= 1u;
      for (int it = 0; ok && it < K; ++it) {
        const float ca = p.coef[it][0], cb = p.coef[it][1], cc = p.coef[it][2];
        const float s2 = it == 0 ? s * s : 1.0f, ks = it == 0 ? s : 1.0f;
        if (wp && it + 1 == K) w_prefetch(q, wr, wc, 128);
        if (it < p.comp) {
          // epilogue 3 reads this thread's row of X's low part: pull it into L2 now
          const char *lo = p.ws + ((it % 2 == 0) ? q.xl0 : q.xl1) + toff;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(lo + panel_pair_off(rl, 32 * k, T1)));
        }
        wait_mma();
        if (!ok) break;
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
          const int j0 = 32 * ch;
          uint32_t r[32];
          tmem_ld32(tmem_base + (uint32_t)j0 + lane_off, r);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              w[e] = pack_bf16(s2 * __uint_as_float(r[8 * c + 2 * e]), s2 * __uint_as_float(r[8 * c + 2 * e + 1]));
            st_shared_v4(sA + half_chunk(rl, j0 + 8 * c), w);
          }
        }
        report();
        wait_mma();
        if (!ok) break;
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
          const int j0 = 32 * ch;
          uint32_t ra[32], rq[32];
          tmem_ld32(tmem_base + (uint32_t)j0 + lane_off, ra);
          tmem_ld32(tmem_base + (uint32_t)(T1 + j0) + lane_off, rq);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i0 = 8 * c + 2 * e;
              w[e] = pack_bf16(fmaf(cb * s2, __uint_as_float(ra[i0]), cc * __uint_as_float(rq[i0])),
                               fmaf(cb * s2, __uint_as_float(ra[i0 + 1]), cc * __uint_as_float(rq[i0 + 1])));
            }
            st_shared_v4(sA + half_chunk(rl, j0 + 8 * c), w);
          }
        }
        report();
        const bool last = it + 1 == K;
        const bool wlast = wp && last;
        uint32_t wv[16];
        if (wlast) w_load(q, wr, wc, wv);       // in flight while the update MMAs run
        wait_mma();
        if (!ok) break;
        const char *clo = it < p.comp ? p.ws + ((it % 2 == 0) ? q.xl0 : q.xl1) + toff : nullptr;
        char *dlo = (it + 1 < p.comp) ? p.ws + ((it % 2 == 0) ? q.xl1 : q.xl0) + toff : nullptr;
        char *dout = last ? p.ws + q.xo + toff : nullptr;
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
          const int j0 = 32 * ch;
          uint32_t wn[16];
          if (wlast && ch < 3) w_load(q, wr, wc + 32 * (ch + 1), wn);
          uint32_t r[32];
          tmem_ld32(tmem_base + (uint32_t)j0 + lane_off, r);
          uint32_t xw[16], lw[16];
#pragma unroll
          for (int c = 0; c < 4; ++c) ld_shared_v4(sX + half_chunk(rl, j0 + 8 * c), xw + 4 * c);
          if (clo) {
#pragma unroll
            for (int k = 0; k < 2; ++k) {
              uint32_t w8[8];
              ld_global_256(clo + panel_pair_off(rl, j0 + 16 * k, T1), w8);
              unswizzle_pair(w8, odd, lw + 8 * k);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) lw[e] = 0u;
          }
          tmem_ld_wait();
          uint32_t hw[16], low[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float x0 = bf16lo(xw[e]) + bf16lo(lw[e]), x1 = bf16hi(xw[e]) + bf16hi(lw[e]);
            const float v0 = ks * fmaf(ca, x0, __uint_as_float(r[2 * e]));
            const float v1 = ks * fmaf(ca, x1, __uint_as_float(r[2 * e + 1]));
            hw[e] = pack_bf16(v0, v1);
            low[e] = pack_bf16(v0 - bf16lo(hw[e]), v1 - bf16hi(hw[e]));
          }
          if (last) {
#pragma unroll
            for (int k = 0; k < 2; ++k) {
              uint32_t in8[8], w8[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) in8[e] = hw[8 * k + e];
              unswizzle_pair(in8, odd, w8);
              st_global_256(dout + panel_pair_off(rl, j0 + 16 * k, T1), w8);
            }
            if (wp) {
              w_partials(wv, hw, dom, dde, dpi);
#pragma unroll
              for (int e = 0; e < 16; ++e) wv[e] = wn[e];
            }
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) st_shared_v4(sX + half_chunk(rl, j0 + 8 * c), hw + 4 * c);
            if (dlo) {
#pragma unroll
              for (int k = 0; k < 2; ++k) {
                uint32_t in8[8], w8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) in8[e] = low[8 * k + e];
                unswizzle_pair(in8, odd, w8);
                st_global_256(dlo + panel_pair_off(rl, j0 + 16 * k, T1), w8);
              }
            }
          }
        }
        report();
      }
      if (ok && wp) w_record(p.partials, (int64_t)q.part_begin + (int64_t)t * 4 + (warp - 2), dom, dde, dpi);
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 256);
  }
}

}  // namespace

cudaError_t launch_himuon_tile(const HmParams &p, int num_sms, cudaStream_t s) {
  static PerDevice attr_set;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr_set.get(dev)) {
    cudaError_t e = cudaFuncSetAttribute(himuon_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
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
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see pdl_wait
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  if (!mp) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (num_sms / 2), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, himuon_tile_kernel, &cfg) != cudaSuccess || n <= 0) {
      (void)cudaGetLastError();
      n = num_sms / 2;
    }
    mp = n < num_sms / 2 ? n : num_sms / 2;
    max_pairs.set(dev, mp);
  }
  const int clusters = p.total_tiles < mp ? p.total_tiles : mp;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, himuon_tile_kernel, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_himuon_tile128(const HmParams &p, int num_sms, cudaStream_t s) {
  static PerDevice max_ctas;   // set after the attribute, so nonzero means both are done
  int dev = 0;
  cudaGetDevice(&dev);
  int mc = max_ctas.get(dev);
  if (!mc) {
    cudaError_t e =
        cudaFuncSetAttribute(himuon_tile128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES1);
    if (e != cudaSuccess) return e;
    int per = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, himuon_tile128_kernel, kThreads1, SMEM_BYTES1) !=
            cudaSuccess ||
        per <= 0) {
      (void)cudaGetLastError();
      per = 1;
    }
    mc = num_sms * (per < kCtasPerSm1 ? per : kCtasPerSm1);   // TMEM: 256 columns per CTA
    max_ctas.set(dev, mc);
  }
  if (p.total_tiles <= 0) return cudaSuccess;
  const int grid = p.total_tiles < mc ? p.total_tiles : mc;
  return launch_pdl(himuon_tile128_kernel, grid, kThreads1, SMEM_BYTES1, s, p);
}

}  // namespace nshb
