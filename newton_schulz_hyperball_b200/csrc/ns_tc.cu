// Grouped bf16 Newton-Schulz GEMM on the 5th-generation tensor cores (tcgen05).
//
// One launch runs one phase of one NS iteration for every matrix (or every
// Hierarchical-Muon tile) of the call ("Muon: the orthogonalized optimizer explained",
// Newton-Schulz section and newton_schulz5; "Hierarchical Muon", abstract):
//   kGram    A  = s^2 X X^T          symmetric: lower-triangle tiles only, mirrored store
//   kPoly    B  = b A + c A A        symmetric: lower-triangle tiles only, mirrored store
//   kUpdate  X' = s (a X + B X)
// with s = 1 / (||U|| + eps) on the first iteration and 1 afterwards.  Operands are bf16,
// products accumulate in fp32 in tensor memory, the epilogue combines in fp32 and stores
// bf16 -- one rounding per phase.
//
// Design (sm_100a):
//  * persistent CTAs (one per SM) walk a static list of 128 x BN (BN = 256, or 128 for
//    small tiles) output tiles of all
//    problems, longest-K problems first;
//  * warp 0 streams 64-deep k slices of both operands into a 4- (6-) stage shared-memory ring
//    with bulk async copies -- the operands are stored in the workspace already in the
//    128-byte-swizzled panel image the tensor core reads, so every slice is one or four
//    contiguous copies and no tensor map is needed;
//  * warp 1 issues tcgen05.mma (M=128, N=BN, K=16) into one of two TMEM accumulators and
//    commits each stage back to the producer;
//  * warps 2-9 drain the other accumulator (tcgen05.ld), apply the phase epilogue and
//    store bf16, overlapping the next tile's main loop; the epilogue's C operand is
//    fetched a chunk ahead (the first chunk before the accumulator is ready).
// Every mbarrier wait is bounded; a wait that runs out sets NSHB_DEV_TIMEOUT and the role
// returns, after which the CTA drains its copies and frees its tensor memory.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "nshb_device.cuh"
#include "nshb_internal.h"

namespace nshb {
namespace {

constexpr int BM = 128, BK = 64;
constexpr int kEpiThreads = 256;              // eight epilogue warps
constexpr int kThreads = 64 + kEpiThreads;   // + producer warp + MMA warp
constexpr int A_BYTES = BM * BK * 2;  // 16 KB
template <int BN> struct Cfg {
  static constexpr int STAGES = BN == 256 ? 4 : 6;
  static constexpr int B_BYTES = BN * BK * 2;             // 32 KB / 16 KB
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;   // 48 KB / 32 KB
  static constexpr int TMEM_COLS = 2 * BN;                // two fp32 accumulators of 128 x BN
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
};
constexpr uint32_t kTimeoutBit = 0x4u;

struct Tile {
  int prob, batch, m0, n0;
};

// Number of BN-wide column tiles of 128-row block `mi` that touch the lower triangle.
template <int BN>
__device__ __forceinline__ int sym_cnt(int mi, int nt) {
  const int c = (BM * mi + BM - 1) / BN + 1;
  return c < nt ? c : nt;
}

template <int BN>
__device__ __forceinline__ Tile decode(const GemmParams &p, int tile) {
  int lo = 0, hi = p.nprob - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (p.prob[mid].tile_begin <= tile) lo = mid; else hi = mid - 1;
  }
  const GemmProb &q = p.prob[lo];
  const int lt = tile - q.tile_begin;
  Tile t;
  t.prob = lo;
  t.batch = lt / q.tiles_per_batch;
  int l = lt % q.tiles_per_batch;
  if (p.mode == kGram || p.mode == kPoly || p.mode == kGramF32) {
    int mi = 0;
    for (;; ++mi) {
      const int c = sym_cnt<BN>(mi, q.nt);
      if (l < c) break;
      l -= c;
    }
    t.m0 = mi * BM;
    t.n0 = l * BN;
  } else {
    t.m0 = (l / q.nt) * BM;
    t.n0 = (l % q.nt) * BN;
  }
  return t;
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ GemmParams p) {
  constexpr int STAGES = Cfg<BN>::STAGES, B_BYTES = Cfg<BN>::B_BYTES, STAGE_BYTES = Cfg<BN>::STAGE_BYTES;
  constexpr int TMEM_COLS = Cfg<BN>::TMEM_COLS;
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
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), kEpiThreads);
    }
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const long long limit = p.wait_limit;
  pdl_trigger();
  pdl_wait();                                      // the previous kernel's outputs are visible

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int stage = 0;
      uint32_t phase = 0;
      int last_parity[STAGES];
      for (int s = 0; s < STAGES; ++s) last_parity[s] = -1;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.total_tiles; tile += gridDim.x) {
        const Tile t = decode<BN>(p, tile);
        const GemmProb &q = p.prob[t.prob];
        const char *a_base = p.ws + q.a_off + (int64_t)t.batch * q.a_bs;
        const char *b_base = p.ws + q.b_off + (int64_t)t.batch * q.b_bs;
        for (int kb = 0; kb < q.kt; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, limit)) {
            set_status(p.status, kTimeoutBit);
            ok = false;
            break;
          }
          const uint32_t sA = smem_base + stage * STAGE_BYTES, sB = sA + A_BYTES;
          mbar_arrive_expect_tx(full_bar(stage), STAGE_BYTES);
          last_parity[stage] = (int)phase;
          bulk_g2s(sA, a_base + (((int64_t)kb * q.a_ph + t.m0) << 7), A_BYTES, full_bar(stage));
          if (p.mode != kUpdate) {
            bulk_g2s(sB, b_base + (((int64_t)kb * q.b_ph + t.n0) << 7), B_BYTES, full_bar(stage));
          } else {
#pragma unroll
            for (int c = 0; c < BN / 64; ++c)
              bulk_g2s(sB + c * (BK * 128),
                       b_base + ((((int64_t)(t.n0 >> 6) + c) * q.b_ph + (int64_t)kb * BK) << 7), BK * 128,
                       full_bar(stage));
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain: every copy this thread started must land before the CTA can exit.
      for (int s = 0; s < STAGES; ++s)
        if (last_parity[s] >= 0 && !mbar_wait(full_bar(s), (uint32_t)last_parity[s], limit))
          set_status(p.status, kTimeoutBit);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      const uint32_t idesc = idesc_bf16(BM, BN, p.mode == kUpdate ? 1 : 0);
      int stage = 0;
      uint32_t phase = 0;
      int tl = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.total_tiles; tile += gridDim.x, ++tl) {
        const Tile t = decode<BN>(p, tile);
        const GemmProb &q = p.prob[t.prob];
        const int buf = tl & 1;
        const uint32_t tph = (uint32_t)(tl >> 1) & 1u;
        if (!mbar_wait(tempty_bar(buf), tph ^ 1u, limit)) {
          set_status(p.status, kTimeoutBit);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
        for (int kb = 0; kb < q.kt; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, limit)) {
            set_status(p.status, kTimeoutBit);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = smem_base + stage * STAGE_BYTES, sB = sA + A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = smem_desc_sw128(sA + 32u * k, 16, 1024);
            const uint64_t bd = (p.mode == kUpdate) ? smem_desc_sw128(sB + 2048u * k, BK * 128, 1024)
                                                    : smem_desc_sw128(sB + 32u * k, 16, 1024);
            tc_mma(d_tmem, ad, bd, idesc, (kb | k) != 0);
          }
          tc_commit(empty_bar(stage));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok && !(p.test_stall && tl == 0)) tc_commit(tfull_bar(buf));
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    // Eight warps: warp w reads TMEM lane quarter (w % 4) -- the hardware restriction --
    // and one half of the tile's columns, so each quarter is drained by two warps.
    constexpr int NCH = BN / 64;                  // 32-column chunks per warp
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;          // row of the 128-row tile
    const bool sym = (p.mode == kGram || p.mode == kPoly || p.mode == kGramF32);
    const bool needc = (p.mode == kPoly || p.mode == kUpdate);
    int tl = 0;
    for (int tile = blockIdx.x; tile < p.total_tiles; tile += gridDim.x, ++tl) {
      const Tile t = decode<BN>(p, tile);
      const GemmProb &q = p.prob[t.prob];
      const int buf = tl & 1;
      const uint32_t tph = (uint32_t)(tl >> 1) & 1u;
      const float s = q.scale_idx >= 0 ? p.scales[q.scale_idx + t.batch] : 1.0f;
      const float s2 = s * s;
      const char *cbase = p.ws + q.c_off + (int64_t)t.batch * q.c_bs;
      char *dbase = p.ws + q.d_off + (int64_t)t.batch * q.d_bs;
      const char *clo = q.c_lo >= 0 ? p.ws + q.c_lo + (int64_t)t.batch * q.c_bs : nullptr;
      char *dlo = q.d_lo >= 0 ? p.ws + q.d_lo + (int64_t)t.batch * q.d_bs : nullptr;
      const int64_t i = t.m0 + row;
      const int ra = (int)(i >> 6);
      const int cc_end = (half + 1) * NCH;
      // chunk cc is processed unless it lies wholly above the diagonal (symmetric outputs)
      auto live = [&](int cc) { return cc < cc_end && !(sym && ((t.n0 + cc * 32) >> 6) > ra); };
      auto load_c = [&](int cc, uint4 (&h)[4], uint4 (&l)[4]) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const size_t off = panel_chunk_off(i, t.n0 + cc * 32 + 8 * g, q.d_ph);
          h[g] = *reinterpret_cast<const uint4 *>(cbase + off);
          l[g] = clo ? *reinterpret_cast<const uint4 *>(clo + off) : make_uint4(0, 0, 0, 0);
        }
      };
      int cc = half * NCH;
      uint4 ch[4], cl[4];
      // C does not depend on the accumulator: fetch the first chunk before waiting for it.
      if (needc && live(cc)) load_c(cc, ch, cl);
      if (!mbar_wait(tfull_bar(buf), tph, limit)) {
        set_status(p.status, kTimeoutBit);
        break;
      }
      tc_fence_after();
#pragma unroll 1
      for (; live(cc); ++cc) {
        const int col0 = t.n0 + cc * 32;
        const int ca = col0 >> 6;
        uint4 nh[4], nl[4];
        if (needc && live(cc + 1)) load_c(cc + 1, nh, nl);   // one chunk ahead
        uint32_t r[32];
        tmem_ld32(tmem_base + (uint32_t)(buf * BN + cc * 32) + ((uint32_t)(quarter * 32) << 16), r);
        tmem_ld_wait();
        float v[32];
        if (p.mode == kGramF32) {
          // fp32 row-major output (row stride d_ph) for the Newton-Muon Gram S = Z Z^T.
          float *drow = reinterpret_cast<float *>(dbase) + i * q.d_ph;
#pragma unroll
          for (int g = 0; g < 8; ++g)
            *reinterpret_cast<float4 *>(drow + col0 + 4 * g) =
                make_float4(__uint_as_float(r[4 * g]), __uint_as_float(r[4 * g + 1]), __uint_as_float(r[4 * g + 2]),
                            __uint_as_float(r[4 * g + 3]));
          if (ca < ra) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              reinterpret_cast<float *>(dbase)[(int64_t)(col0 + e) * q.d_ph + i] = __uint_as_float(r[e]);
          }
          continue;
        }
        if (p.mode == kGram) {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = s2 * __uint_as_float(r[e]);
        } else {
          const float kc = (p.mode == kPoly) ? p.cb : p.ca;
          const float ka = (p.mode == kPoly) ? p.cc : 1.0f;
          const float ks = (p.mode == kPoly) ? 1.0f : s;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const uint32_t hw[4] = {ch[g].x, ch[g].y, ch[g].z, ch[g].w};
            const uint32_t lw[4] = {cl[g].x, cl[g].y, cl[g].z, cl[g].w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              // C carried as a hi + lo pair (lo is zero when not kept)
              const float c0 = bf16lo(hw[h]) + bf16lo(lw[h]);
              const float c1 = bf16hi(hw[h]) + bf16hi(lw[h]);
              v[8 * g + 2 * h] = ks * fmaf(kc, c0, ka * __uint_as_float(r[8 * g + 2 * h]));
              v[8 * g + 2 * h + 1] = ks * fmaf(kc, c1, ka * __uint_as_float(r[8 * g + 2 * h + 1]));
            }
          }
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint4 o;
          o.x = pack_bf16(v[8 * g + 0], v[8 * g + 1]);
          o.y = pack_bf16(v[8 * g + 2], v[8 * g + 3]);
          o.z = pack_bf16(v[8 * g + 4], v[8 * g + 5]);
          o.w = pack_bf16(v[8 * g + 6], v[8 * g + 7]);
          const size_t off = panel_chunk_off(i, col0 + 8 * g, q.d_ph);
          *reinterpret_cast<uint4 *>(dbase + off) = o;
          if (dlo) {   // keep the rounding residual as a second bf16
            uint4 l;
            l.x = pack_bf16(v[8 * g + 0] - bf16lo(o.x), v[8 * g + 1] - bf16hi(o.x));
            l.y = pack_bf16(v[8 * g + 2] - bf16lo(o.y), v[8 * g + 3] - bf16hi(o.y));
            l.z = pack_bf16(v[8 * g + 4] - bf16lo(o.z), v[8 * g + 5] - bf16hi(o.z));
            l.w = pack_bf16(v[8 * g + 6] - bf16lo(o.w), v[8 * g + 7] - bf16hi(o.w));
            *reinterpret_cast<uint4 *>(dlo + off) = l;
          }
        }
        if (sym && ca < ra) {
          // Mirror: element (i, col0 + e) also lands at (col0 + e, i).
          const int64_t ib = i & ~7LL;
          const int ie = (int)(i & 7);
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            __nv_bfloat16 h = __float2bfloat16_rn(v[e]);
            *reinterpret_cast<__nv_bfloat16 *>(dbase + panel_chunk_off(col0 + e, ib, q.d_ph) + 2 * ie) = h;
          }
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          ch[g] = nh[g];
          cl[g] = nl[g];
        }
      }
      tc_fence_before();
      mbar_arrive(tempty_bar(buf));
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

template <int BN>
cudaError_t launch_bn(const GemmParams &p, int num_sms, cudaStream_t s) {
  static PerDevice attr_set;  // the attribute is set once per device
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr_set.get(dev)) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg<BN>::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set.set(dev, 1);
  }
  const int grid = p.total_tiles < num_sms ? p.total_tiles : num_sms;
  return launch_pdl(gemm_tc_kernel<BN>, grid, kThreads, Cfg<BN>::SMEM_BYTES, s, p);
}

}  // namespace

cudaError_t launch_gemm_tc(const GemmParams &p, int bn, int num_sms, cudaStream_t s) {
  if (p.total_tiles <= 0) return cudaSuccess;
  return bn == 256 ? launch_bn<256>(p, num_sms, s) : launch_bn<128>(p, num_sms, s);
}


}  // namespace nshb
