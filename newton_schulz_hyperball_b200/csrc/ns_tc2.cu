// Grouped bf16 Newton-Schulz GEMM on CTA pairs (tcgen05.mma.cta_group::2).
//
// Phases: Gram A = s^2 X X^T and polynomial B = b A + c A^2 (only the tiles on and below the diagonal are computed and
// stored; a reader takes a block above the diagonal as the transpose of its mirror), update
// X' = s (a X + B X) ("Muon: the orthogonalized optimizer explained", Newton-Schulz
// section), plus the fp32 Gram S = Z Z^T of the Newton-Muon layer inputs, whose operands are
// loaded straight from the caller's row-major Z through one swizzling tensor map per input.
//
// Why pairs: with single-CTA 128 x 256 tiles every SM must stream 96 bytes of operands
// per clock to keep its tensor core busy, more than the L2 delivers per SM.  A pair of
// CTAs on two SMs computes a 256 x 256 tile with one instruction stream: each CTA holds
// 128 rows of A and 128 columns of B, and the tensor cores read the partner's half
// directly, so each SM streams 64 bytes per clock for the same work.
//
// Stages are 128 deep in k (64 KB per CTA): the load path has a fixed cost of a few
// hundred ns per barrier round trip, so fewer, larger stages stream faster than many small
// ones (measured: 128 vs 74-89 GB/s per SM for 64 KB vs 32 KB stages).
//
// Roles per CTA (320 threads): warp 0 issues TMA loads of this CTA's halves into a
// 3-stage ring; in the leader CTA (rank 0) warp 1 issues the MMAs for the pair and
// multicasts each commit to both CTAs; warps 2-9 of both CTAs drain their own 128-row
// accumulator (two TMEM buffers, so the epilogue overlaps the next tile).  Loads of both
// CTAs complete on the leader's "full" barrier; the epilogues of both CTAs arrive on the
// leader's "tmem empty" barrier.  No load is multicast.  Every wait is bounded.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <mutex>
#include <type_traits>

#include "nshb_device.cuh"
#include "nshb_internal.h"

namespace nshb {
namespace {

constexpr int BM = 256, BN = 256, BK = 128, STAGES = 3;
constexpr int SLICE_BYTES = 128 * 64 * 2;         // 16 KB: 128 rows x 64 bf16 (one k panel)
constexpr int HALF_BYTES = 2 * SLICE_BYTES;       // one operand half: two 64-deep k panels
constexpr int STAGE_BYTES = 2 * HALF_BYTES;       // A half + B half of one CTA (64 KB)
constexpr int TMEM_COLS = 2 * BN;                 // two 128 x 256 fp32 accumulators
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
static_assert(2 * kEpiWarps == kPartsPerTile, "one partial record per epilogue warp of the pair");
constexpr uint32_t kTimeoutBit = 0x4u;
constexpr uint32_t kPeerMask = 0xFEFFFFFFu;       // clears the CTA-rank bit of a cluster address

struct Tile {
  int prob, batch, m0, n0;
};

__device__ __forceinline__ bool sym_mode(int mode) { return mode == kGram || mode == kPoly || mode == kGramF32; }

template <class P>
__device__ __forceinline__ Tile decode2(const P &p, int tile) {
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
  if (sym_mode(p.mode)) {
    // 256-row block mi needs the column tiles nj <= mi (lower triangle incl. diagonal)
    int mi = 0;
    for (;; ++mi) {
      const int c = (mi + 1 < q.nt) ? mi + 1 : q.nt;
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

// FUSE: the instance for the last update launch with Hyperball partials (W read in the
// epilogue); the other launches use the instance without that code, whose register budget
// it would otherwise raise.
// RAW (SyrkParams): A and B of problem i are rows of the caller's Z through p.zmap[i].
template <bool FUSE, class P>
__device__ __forceinline__ void gemm_tc2_body(const P &p) {
  constexpr bool RAW = std::is_same<P, SyrkParams>::value;
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
      mbar_init(tempty_bar(b), 2 * kEpiWarps);   // one arrive per epilogue warp of both CTAs
    }
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc2(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish2();
  }
  tc_fence_before();
  cluster_sync();                                  // barriers of both CTAs initialised
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const long long limit = p.wait_limit;
  if (warp == 0 && lane == 0) {
    if constexpr (RAW) {
      if (cid < p.total_tiles) prefetch_tmap(&p.zmap[decode2(p, cid).prob]);
    } else {
      prefetch_tmap(&p.tmap);
    }
  }
  pdl_trigger();
  pdl_wait();                                      // the previous kernel's outputs are visible

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      int last_parity[STAGES];
      for (int s = 0; s < STAGES; ++s) last_parity[s] = -1;
      bool ok = true;
      for (int tile = cid; ok && tile < p.total_tiles; tile += ncl) {
        const Tile t = decode2(p, tile);
        const GemmProb &q = p.prob[t.prob];
        const int64_t a_row = (q.a_off + (int64_t)t.batch * q.bs) >> 7;   // 128-byte rows
        const int64_t b_row = (q.b_off + (int64_t)t.batch * q.bs) >> 7;
        const int am = t.m0 + 128 * (int)rank;     // this CTA's A rows
        const int bn = t.n0 + 128 * (int)rank;     // this CTA's B columns
        for (int kb = 0; kb < q.kt; kb += 2) {      // q.kt counts 64-deep panels
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, limit)) {
            set_status(p.status, kTimeoutBit);
            ok = false;
            break;
          }
          const uint32_t sA = smem_base + stage * STAGE_BYTES, sB = sA + HALF_BYTES;
          const uint32_t fb = full_bar(stage) & kPeerMask;   // the leader's barrier
          if (leader) {
            mbar_arrive_expect_tx(full_bar(stage), 2 * STAGE_BYTES);
            last_parity[stage] = (int)phase;
          }
          // K-major: rows am .. am+127 of k panels kb and kb+1 (16 KB each); MN-major: the 128
          // rows (columns of the stored matrix) are two 64-column panels, k rows kb*64 .. +127.
          // A symmetric operand stored below the diagonal only reads a block above it (k tile
          // > the operand's row tile) MN-major from its mirror.
          const bool a_mn = (q.major & kAMn) || ((q.major & kASym) && (kb >> 2) > (t.m0 >> 8));
          const bool b_mn = (q.major & kBMn) || ((q.major & kBSym) && (kb >> 2) > (t.n0 >> 8));
          if constexpr (RAW) {
            // Columns kb*64 .. +127 of Z's rows am .. am+127 and bn .. bn+127; the tensor map
            // swizzles them into the same image as a stored panel, and reads zeros past the
            // last row or column.
            const CUtensorMap *zm = &p.zmap[t.prob];
            tma_load_2sm(sA, zm, kb * 64, am, fb);
            tma_load_2sm(sA + SLICE_BYTES, zm, kb * 64 + 64, am, fb);
            tma_load_2sm(sB, zm, kb * 64, bn, fb);
            tma_load_2sm(sB + SLICE_BYTES, zm, kb * 64 + 64, bn, fb);
          } else if (!a_mn) {
            const int64_t ya = a_row + (int64_t)kb * q.a_ph + am;
            tma_load_2sm(sA, &p.tmap, 0, (int)ya, fb);
            tma_load_2sm(sA + SLICE_BYTES, &p.tmap, 0, (int)(ya + q.a_ph), fb);
          } else {
            const int64_t y0 = a_row + (int64_t)(am >> 6) * q.a_ph + (int64_t)kb * 64;
            tma_load_2sm(sA, &p.tmap, 0, (int)y0, fb);
            tma_load_2sm(sA + SLICE_BYTES, &p.tmap, 0, (int)(y0 + q.a_ph), fb);
          }
          if (RAW) {
          } else if (!b_mn) {
            const int64_t yb = b_row + (int64_t)kb * q.b_ph + bn;
            tma_load_2sm(sB, &p.tmap, 0, (int)yb, fb);
            tma_load_2sm(sB + SLICE_BYTES, &p.tmap, 0, (int)(yb + q.b_ph), fb);
          } else {
            const int64_t y0 = b_row + (int64_t)(bn >> 6) * q.b_ph + (int64_t)kb * 64;
            tma_load_2sm(sB, &p.tmap, 0, (int)y0, fb);
            tma_load_2sm(sB + SLICE_BYTES, &p.tmap, 0, (int)(y0 + q.b_ph), fb);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain: every load of the pair that the leader armed must have landed.
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
        const Tile t = decode2(p, tile);
        const GemmProb &q = p.prob[t.prob];
        const int buf = tl & 1;
        const uint32_t tph = (uint32_t)(tl >> 1) & 1u;
        if (!mbar_wait(tempty_bar(buf), tph ^ 1u, limit)) {
          set_status(p.status, kTimeoutBit);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
        for (int kb = 0; kb < q.kt; kb += 2) {
          if (!mbar_wait(full_bar(stage), phase, limit)) {
            set_status(p.status, kTimeoutBit);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = smem_base + stage * STAGE_BYTES, sB = sA + HALF_BYTES;
          // the majorness the producer loaded this stage with
          const bool amn = (q.major & kAMn) || ((q.major & kASym) && (kb >> 2) > (t.m0 >> 8));
          const bool bmn = (q.major & kBMn) || ((q.major & kBSym) && (kb >> 2) > (t.n0 >> 8));
          const uint32_t idesc = idesc_bf16(BM, BN, amn ? 1 : 0, bmn ? 1 : 0);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            // K-major: panel k/4, 32-byte step k%4 inside the 128-byte swizzled rows.
            // MN-major: 16 k rows (2 KB) per step; the two 64-column chunks are 16 KB apart.
            const uint32_t kofs = (uint32_t)(k >> 2) * SLICE_BYTES + 32u * (k & 3);
            const uint64_t ad = amn ? smem_desc_sw128(sA + 2048u * k, SLICE_BYTES, 1024)
                                    : smem_desc_sw128(sA + kofs, 16, 1024);
            const uint64_t bd = bmn ? smem_desc_sw128(sB + 2048u * k, SLICE_BYTES, 1024)
                                    : smem_desc_sw128(sB + kofs, 16, 1024);
            tc_mma2(d_tmem, ad, bd, idesc, (kb | k) != 0);
          }
          tc_commit2_mc(empty_bar(stage), 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok && !(p.test_stall && tl == 0)) tc_commit2_mc(tfull_bar(buf), 0x3);
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue (both CTAs)
    constexpr int NCH = BN / 64;                  // 32-column chunks per warp (half the tile)
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = 128 * (int)rank + quarter * 32 + lane;   // row of the 256-row tile
    const bool needc = (p.mode == kPoly || p.mode == kUpdate);
    const bool fuse = FUSE && p.mode == kUpdate && p.partials != nullptr;
    int tl = 0;
    for (int tile = cid; tile < p.total_tiles; tile += ncl, ++tl) {
      const Tile t = decode2(p, tile);
      const GemmProb &q = p.prob[t.prob];
      const int buf = tl & 1;
      const uint32_t tph = (uint32_t)(tl >> 1) & 1u;
      const float s = q.scale_idx >= 0 ? p.scales[q.scale_idx + t.batch] : 1.0f;
      const float s2 = s * s;
      const char *cbase = p.ws + q.c_off + (int64_t)t.batch * q.bs;
      char *dbase = p.ws + q.d_off + (int64_t)t.batch * q.bs;
      const char *clo = q.c_lo >= 0 ? p.ws + q.c_lo + (int64_t)t.batch * q.bs : nullptr;
      char *dlo = q.d_lo >= 0 ? p.ws + q.d_lo + (int64_t)t.batch * q.bs : nullptr;
      const int64_t i = t.m0 + row;
      const int cc_end = (half + 1) * NCH;
      // Hyperball partials of this problem: the caller's W next to O (X coordinates (i, c)
      // are W's (i, c), offset by the tile origin for a Hierarchical-Muon tile).
      const bool wp = fuse && q.w != nullptr;
      int64_t wr0 = 0, wc0 = 0;
      if (wp && (q.w_flags & kPwTiled)) {
        wr0 = (int64_t)(t.batch / q.w_tiles_c) * q.d_ph;
        wc0 = (int64_t)(t.batch % q.w_tiles_c) * q.d_ph;
      }
      // bf16 W of columns t.n0 + 32 cc .. +31 as pairs in logical order, zero outside W (the
      // epilogue reads bf16 weights only; fp32 weights take the reduce pass).
      auto load_w = [&](int cc, uint32_t (&wv)[16]) {
        const int64_t xc0 = t.n0 + cc * 32;
        const unsigned short *w16 = static_cast<const unsigned short *>(q.w);
        {
          const int64_t wr = wr0 + i, wc = wc0 + xc0;
          if (wr < q.w_m && wc + 31 < q.w_n && (q.w_flags & kPwVec)) {
            const uint4 *src = reinterpret_cast<const uint4 *>(w16 + wr * q.w_ld + wc);
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const uint4 u = src[g];
              wv[4 * g] = u.x; wv[4 * g + 1] = u.y; wv[4 * g + 2] = u.z; wv[4 * g + 3] = u.w;
            }
          } else {
            const bool in = wr < q.w_m;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int64_t c = wc + 2 * e;
              const uint32_t lo = (in && c < q.w_n) ? (uint32_t)w16[wr * q.w_ld + c] : 0u;
              const uint32_t hi = (in && c + 1 < q.w_n) ? (uint32_t)w16[wr * q.w_ld + c + 1] : 0u;
              wv[e] = lo | (hi << 16);
            }
          }
        }
      };
      double dom = 0.0, dde = 0.0, dpi = 0.0;
      // Pulls this thread's W elements of the tile into L2 while the MMAs run, so that the
      // per-chunk loads below find them there.
      auto prefetch_w = [&]() {
        const int esz = 2;
        const char *wb = static_cast<const char *>(q.w);
        for (int c = half * NCH; c < cc_end; ++c) {
          const int64_t wr = wr0 + i, wc = wc0 + t.n0 + c * 32;
          if (wr < q.w_m && wc < q.w_n) asm volatile("prefetch.global.L2 [%0];" ::"l"(wb + (wr * q.w_ld + wc) * esz));
        }
      };
      // every chunk of the tile, the diagonal tiles of a symmetric result whole (its readers
      // take a block above the diagonal from the stored one below it)
      auto live = [&](int cc) { return cc < cc_end; };
      const bool odd = i & 1;
      // C words of columns col0 .. col0+31 in logical order (two 32-byte sector reads).
      // (The fused instance prefetches W instead of C's low part, which it reads in the chunk.)
      auto load_c = [&](int cc, uint32_t (&h)[16], uint32_t (&l)[16]) {
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const size_t off = panel_pair_off(i, t.n0 + cc * 32 + 16 * k, q.d_ph);
          uint32_t w[8];
          ld_global_256(cbase + off, w);
          unswizzle_pair(w, odd, h + 8 * k);
          if (!FUSE && clo) {
            ld_global_256(clo + off, w);
            unswizzle_pair(w, odd, l + 8 * k);
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) l[8 * k + e] = 0u;
          }
        }
      };
      int cc = half * NCH;
      uint32_t ch[16], cl[16], wcur[16];
      if (needc && live(cc)) load_c(cc, ch, cl);
      if (wp) {
        prefetch_w();
        load_w(cc, wcur);                    // in flight while the tile's MMAs finish
      }
      if (!mbar_wait(tfull_bar(buf), tph, limit)) {
        set_status(p.status, kTimeoutBit);
        break;
      }
      tc_fence_after();
#pragma unroll 1
      for (; live(cc); ++cc) {
        const int col0 = t.n0 + cc * 32;
        uint32_t nh[16], nl[16], wn[16];
        if (needc && live(cc + 1)) load_c(cc + 1, nh, nl);
        if (wp && live(cc + 1)) load_w(cc + 1, wn);
        if (FUSE && clo) {
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            uint32_t w[8];
            ld_global_256(clo + panel_pair_off(i, col0 + 16 * k, q.d_ph), w);
            unswizzle_pair(w, odd, cl + 8 * k);
          }
        }
        uint32_t r[32];
        tmem_ld32(tmem_base + (uint32_t)(buf * BN + cc * 32) + ((uint32_t)(quarter * 32) << 16), r);
        tmem_ld_wait();
        float v[32];
        if (p.mode == kGramF32) {
          float *drow = reinterpret_cast<float *>(dbase) + i * q.d_ph;
#pragma unroll
          for (int g = 0; g < 8; ++g)
            *reinterpret_cast<float4 *>(drow + col0 + 4 * g) =
                make_float4(__uint_as_float(r[4 * g]), __uint_as_float(r[4 * g + 1]), __uint_as_float(r[4 * g + 2]),
                            __uint_as_float(r[4 * g + 3]));
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
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const float c0 = bf16lo(ch[4 * g + h]) + bf16lo(cl[4 * g + h]);
              const float c1 = bf16hi(ch[4 * g + h]) + bf16hi(cl[4 * g + h]);
              v[8 * g + 2 * h] = ks * fmaf(kc, c0, ka * __uint_as_float(r[8 * g + 2 * h]));
              v[8 * g + 2 * h + 1] = ks * fmaf(kc, c1, ka * __uint_as_float(r[8 * g + 2 * h + 1]));
            }
          }
        }
        float pom = 0.f, pde = 0.f, ppi = 0.f;   // this chunk's partials (32 terms, fp32)
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          uint32_t o[8], w[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) o[e] = pack_bf16(v[16 * k + 2 * e], v[16 * k + 2 * e + 1]);
          if (wp) {
            // of O as stored (bf16), which is what the apply pass reads
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float o0 = bf16lo(o[e]), o1 = bf16hi(o[e]);
              const float w0 = bf16lo(wcur[8 * k + e]), w1 = bf16hi(wcur[8 * k + e]);
              pom = fmaf(o0, o0, fmaf(o1, o1, pom));
              pde = fmaf(w0, o0, fmaf(w1, o1, pde));
              ppi = fmaf(w0, w0, fmaf(w1, w1, ppi));
            }
          }
          const size_t off = panel_pair_off(i, col0 + 16 * k, q.d_ph);
          unswizzle_pair(o, odd, w);              // the same swap puts logical order back
          st_global_256(dbase + off, w);
          if (dlo) {
            uint32_t l[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              l[e] = pack_bf16(v[16 * k + 2 * e] - bf16lo(o[e]), v[16 * k + 2 * e + 1] - bf16hi(o[e]));
            unswizzle_pair(l, odd, w);
            st_global_256(dlo + off, w);
          }
        }
        if (wp) {
          dom += (double)pom;
          dde += (double)pde;
          dpi += (double)ppi;
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          ch[e] = nh[e];
          if (!FUSE) cl[e] = nl[e];
          if (FUSE) wcur[e] = wn[e];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) remote_arrive(mapa(tempty_bar(buf), 0));   // the leader's barrier
      if (wp) {
        // One record per epilogue warp and tile: fixed order, so the sums are deterministic.
        dom = warp_sum(dom);
        dde = warp_sum(dde);
        dpi = warp_sum(dpi);
        if (lane == 0) {
          const int64_t rec = (int64_t)q.part_begin + (int64_t)(tile - q.tile_begin) * kPartsPerTile +
                              (int64_t)rank * kEpiWarps + (warp - 2);
          p.partials[3 * rec] = dom;
          p.partials[3 * rec + 1] = dde;
          p.partials[3 * rec + 2] = dpi;
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync();                                  // no CTA leaves while its partner may still
                                                   // read its shared memory or signal it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem_base, TMEM_COLS);
  }
}

// 320 threads: three warps share one SM sub-partition's 16K registers, so 168 per thread is
// the most a CTA can be given.
__global__ void __launch_bounds__(kThreads, 1) gemm_tc2_kernel(const __grid_constant__ GemmParams p) {
  gemm_tc2_body<false>(p);
}
__global__ void __launch_bounds__(kThreads, 1) gemm_tc2_fused_kernel(const __grid_constant__ GemmParams p) {
  gemm_tc2_body<true>(p);
}
__global__ void __launch_bounds__(kThreads, 1) gemm_tc2_syrk_kernel(const __grid_constant__ SyrkParams p) {
  gemm_tc2_body<false>(p);
}

std::mutex g_tmap_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// The driver's tensor-map encoder, looked up once.
cudaError_t load_encoder() {
  std::lock_guard<std::mutex> g(g_tmap_mu);
  if (!g_encode) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) return e != cudaSuccess ? e : cudaErrorNotSupported;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t encode_ws_tensor_map(CUtensorMap *map, void *ws, size_t bytes) {
  cudaError_t e = load_encoder();
  if (e != cudaSuccess) return e;
  const cuuint64_t dims[2] = {64, (cuuint64_t)(bytes / 128)};
  const cuuint64_t strides[1] = {128};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t encode_z_tensor_map(CUtensorMap *map, const void *z, int64_t d, int64_t n) {
  cudaError_t e = load_encoder();
  if (e != cudaSuccess) return e;
  if (d <= 0 || n <= 0 || n % 64 != 0 || reinterpret_cast<uintptr_t>(z) % 16 != 0) return cudaErrorInvalidValue;
  const cuuint64_t dims[2] = {(cuuint64_t)n, (cuuint64_t)d};
  const cuuint64_t strides[1] = {(cuuint64_t)n * 2};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(z), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

namespace {

int set_up_device(int dev, int num_sms, cudaError_t *err) {
  static PerDevice attr_set;  // the attributes are set once per device
  if (!attr_set.get(dev)) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemm_tc2_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemm_tc2_syrk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) {
      *err = e;
      return 0;
    }
    attr_set.set(dev, 1);
  }
  // Pairs that can be resident at once (a GPC with an odd number of free SMs leaves one
  // idle), so that the persistent grid never spills into a second wave.  The three kernels
  // have the same shape.
  static PerDevice max_pairs;
  int mp = max_pairs.get(dev);
  if (!mp) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (num_sms / 2), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_tc2_kernel, &cfg) != cudaSuccess || n <= 0) {
      (void)cudaGetLastError();
      n = num_sms / 2;
    }
    mp = n < num_sms / 2 ? n : num_sms / 2;
    max_pairs.set(dev, mp);
  }
  return mp;
}

template <class P>
cudaError_t launch_pairs(void (*kernel)(P), const P &p, int num_sms, cudaStream_t s) {
  int dev = 0;
  cudaGetDevice(&dev);
  cudaError_t err = cudaSuccess;
  const int mp = set_up_device(dev, num_sms, &err);
  if (!mp) return err;
  if (p.total_tiles <= 0) return cudaSuccess;
  const int clusters = p.total_tiles < mp ? p.total_tiles : mp;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see pdl_wait
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_tc2(const GemmParams &p, int num_sms, cudaStream_t s) {
  const bool fused = p.mode == kUpdate && p.partials != nullptr;
  return launch_pairs(fused ? gemm_tc2_fused_kernel : gemm_tc2_kernel, p, num_sms, s);
}

cudaError_t launch_gemm_syrk(const SyrkParams &p, int num_sms, cudaStream_t s) {
  if (p.mode != kGramF32) return cudaErrorInvalidValue;
  return launch_pairs(gemm_tc2_syrk_kernel, p, num_sms, s);
}

}  // namespace nshb
