// FlashAttention forward on CTA pairs: the same online softmax and the same
// warp roles as fwd.cu, with every product issued once for two SMs (tcgen05
// with cta_group::2, M = 256).  Used for dense inputs without a mask, bias or
// dropout whose head dims take 128-column tiles (the long head-dim-128
// workloads, whose time is spent in the products and the exponentials).
//
// A pair works on 512 query rows of one (batch, head): CTA r holds query
// tiles [256 r, 256 r + 256) of them as two 128-row tiles, like one CTA of
// fwd.cu.  The B operands are split between the CTAs: CTA r loads keys
// [64 r, 64 r + 64) of each key tile (S = Q K^T, N = 128) and columns
// [64 r, 64 r + 64) of each value tile (O += P V, N = 128), and the pair's
// leader (cluster rank 0) issues both products for the pair's 256 rows per
// query tile; each CTA's TMEM receives its own rows.  Per SM and key tile
// that reads 160 KiB of shared memory against 256 KiB in fwd.cu (the B
// halves cross between the two SMs), for the same tensor work.
//
// Roles per CTA (384 threads): warps 0-7 softmax (two groups, one per query
// tile of this CTA); warp 8 TMA producer; warp 9 TMEM allocation and, in the
// leader, the MMA issuer; warps 10-11 idle.  Completion of the pair's
// products is signalled to both CTAs (multicast commit); both CTAs' loads
// complete on the leader's barriers, whose transaction counts the leader
// sets for both; the softmax warps of both CTAs report P ready to the
// leader's barriers.  Units (512 rows; a last round at most half full in
// 256-row halves, one query tile per CTA) are dealt to the pairs round
// robin; every barrier's phase follows a running count of key tiles.
#include <cuda_runtime.h>

#include "common.cuh"
#include "fwd.h"

namespace attn {
namespace {

struct PairCfg {
  static constexpr int kThreads = 384;
  static constexpr int kLaunchRegs = 168;
  static constexpr int kLowRegs = 104;
  static constexpr int kHighRegs = (kThreads * kLaunchRegs - 128 * kLowRegs) / 256 / 8 * 8;
  static constexpr int kQTile = 128 * 128 * 2;  // one query tile, two 64-column blocks
  static constexpr int kKHalf = 64 * 128 * 2;   // 64 keys x 128 columns, two blocks
  static constexpr int kVHalf = 128 * 64 * 2;   // 128 keys x 64 columns, one block
  static constexpr int kStages = 4;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + 2 * kQTile;
  static constexpr int kOffV = kOffK + kStages * kKHalf;
  static constexpr int kOffBar = kOffV + kStages * kVHalf;
  // q_full[2] q_empty k_full[S] k_empty[S] v_full[S] v_empty[S] s_full[2]
  // p_ready[2] o_done[2] mma_done
  static constexpr int kNumBars = 3 + 4 * kStages + 7;
  static constexpr int kOffMisc = kOffBar + 8 * kNumBars;
  static constexpr int kSmemBytes = kOffMisc + 16;
  static constexpr int kColO = 256;  // S of tile t at [128 t, +128), O at [256 + 128 t, +128)
};

__device__ __forceinline__ uint32_t cta_rank_in_cluster() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// The pair's leader (CTA 0) holds the barriers both CTAs' loads complete on
// and the softmax warps report to: the cluster address of the leader's copy
// of a local shared variable.
__device__ __forceinline__ uint32_t leader_addr(uint32_t local) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(a) : "r"(local));
  return a;
}
__device__ __forceinline__ void tma_load_4d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                 int x, int y, int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(leader_addr(bar))
      : "memory");
}
__device__ __forceinline__ void mma_ss_pair(uint32_t d, uint32_t a_lo, uint32_t a_hi, uint32_t b_lo,
                                            uint32_t b_hi, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
      "mov.b64 da, {%1, %2};\n\tmov.b64 db, {%3, %4};\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], da, db, %5, p;\n\t}" ::"r"(d),
      "r"(a_lo), "r"(a_hi), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void mma_ts_pair(uint32_t d, uint32_t a_tmem, uint32_t b_lo, uint32_t b_hi,
                                            uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], db, %4, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(acc)
      : "memory");
}
// Completion of the pair's products so far, on `bar` of both CTAs.
__device__ __forceinline__ void commit_pair(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"((uint16_t)3)
      : "memory");
}
// One arrival per warp on the leader's copy of `bar`, after the warp's TMEM
// stores have completed (tcgen05.wait::st) and been fenced by the caller.
// Default semantics: the cluster-scope release form costs the arriving warp
// about a thousand cycles, and what the MMA reads is this SM's own TMEM,
// written before the arrival is issued.
__device__ __forceinline__ void arrive_leader_warp(uint32_t bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0)
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(leader_addr(bar))
                 : "memory");
}

}  // namespace

template <bool BF16>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg::kThreads, 1)
    attn_fwd_pair_kernel(const __grid_constant__ FwdArgs args) {
  using C = PairCfg;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cta_rank_in_cluster();
  const bool leader = rank == 0;
  const int64_t pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int32_t n_mblocks = (args.Sq + 511) / 512;
  // Units: n_full of 512 rows (two query tiles per CTA), dealt round robin.
  // When the last round would be at most half full, its units are split in
  // two halves of 256 rows (one query tile per CTA), so that round takes
  // about the time of one query tile's chain instead of two tiles'.
  const int64_t n_full = (int64_t)n_mblocks * args.H * args.B;
  const int64_t rounds = n_full / n_pairs, left = n_full - rounds * n_pairs;
  const bool split = rounds >= 1 && left > 0 && 2 * left <= n_pairs;
  const int64_t split_from = split ? rounds * n_pairs : n_full;
  const int64_t n_units = split ? split_from + 2 * left : n_full;
  const int32_t n_tiles = (args.Sk + 127) / 128;
  if (sbase & 1023) {  // identical in both CTAs of the pair, so both return
    if (threadIdx.x == 0) atomicOr(args.status, 1u << kSiteTeardown);
    return;
  }
  // Unit u: (batch b, head h), this CTA's first row m0 and its nt query
  // tiles (rows m0 + 128 t); every role decodes the same units.
  auto unit_of = [&](int64_t u, int32_t& b, int32_t& h, int32_t& m0, int& nt) {
    int64_t fu = u;
    int32_t half = 0;
    nt = 2;
    if (u >= split_from) {
      fu = split_from + (u - split_from) / 2;
      half = (int32_t)((u - split_from) & 1);
      nt = 1;
    }
    const int64_t hb = fu / n_mblocks;
    m0 = (int32_t)(fu - hb * n_mblocks) * 512 +
         (nt == 2 ? 256 * (int32_t)rank : 256 * half + 128 * (int32_t)rank);
    h = (int32_t)(hb % args.H);
    b = (int32_t)(hb / args.H);
  };

  const uint32_t sQ = sbase + C::kOffQ, sK = sbase + C::kOffK, sV = sbase + C::kOffV;
  const uint32_t bar0 = sbase + C::kOffBar;
  auto q_full = [&](int t) { return bar0 + 8 * t; };
  const uint32_t q_empty = bar0 + 16;
  auto k_full = [&](int s) { return bar0 + 8 * (3 + s); };
  auto k_empty = [&](int s) { return bar0 + 8 * (3 + C::kStages + s); };
  auto v_full = [&](int s) { return bar0 + 8 * (3 + 2 * C::kStages + s); };
  auto v_empty = [&](int s) { return bar0 + 8 * (3 + 3 * C::kStages + s); };
  auto s_full = [&](int t) { return bar0 + 8 * (3 + 4 * C::kStages + t); };
  auto p_ready = [&](int t) { return bar0 + 8 * (5 + 4 * C::kStages + t); };
  auto o_done = [&](int t) { return bar0 + 8 * (7 + 4 * C::kStages + t); };
  const uint32_t mma_done = bar0 + 8 * (9 + 4 * C::kStages);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(q_full(t), 1);
      mbar_init(s_full(t), 1);
      mbar_init(p_ready(t), 8);  // one arrival per softmax warp of tile t in both CTAs
      mbar_init(o_done(t), 1);
    }
    mbar_init(q_empty, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs exist before any load or product
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto o_row_ptr = [&](int32_t b, int32_t h, int32_t i) -> uint8_t* {
    const int64_t off = (int64_t)b * args.o_stride[0] + (int64_t)h * args.o_stride[1] +
                        (int64_t)i * args.o_stride[2];
    return reinterpret_cast<uint8_t*>(args.o) + 2 * off;
  };
  auto lse_ptr = [&](int32_t b, int32_t h, int32_t i) -> float* {
    const int64_t idx = args.lse_th ? ((int64_t)b * args.Sq + i) * args.H + h
                                    : ((int64_t)b * args.H + h) * args.Sq + i;
    return args.lse + idx;
  };

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::kLowRegs));
    if (warp == 8 && lane == 0) {
      // ===================== TMA producer (both CTAs) =====================
      // This CTA's Q tiles, K rows [n0 + 64 rank, +64) and V columns
      // [64 rank, +64); completion counted on the leader's barriers, whose
      // transaction counts the leader sets for both CTAs.
      prefetch_tmap(&args.tq);
      prefetch_tmap(&args.tk2);
      prefetch_tmap(&args.tv);
      int64_t nk = 0, nv = 0, uc = 0;
      int64_t qn0 = 0, qn1 = 0;  // Q loads issued per tile
      bool stop = false;
      for (int64_t u = pair; u < n_units && !stop; u += n_pairs) {
        int32_t b, h, m0;
        int nt;
        unit_of(u, b, h, m0, nt);
        if (uc > 0 && !mbar_wait(q_empty, (uint32_t)((uc - 1) & 1), abort_flag, args.status, kSiteLoad))
          break;
        for (int t = 0; t < nt; ++t) {
          if (leader) mbar_expect_tx(q_full(t), 2 * C::kQTile);
          for (int blk = 0; blk < 2; ++blk)
            tma_load_4d_pair(sQ + t * C::kQTile + blk * 16384, &args.tq, q_full(t), 64 * blk,
                             m0 + 128 * t, h, b);
          ++(t == 0 ? qn0 : qn1);
        }
        ++uc;
        for (int it = 0; it < n_tiles; ++it) {
          const int n0 = it * 128;
          const int ks = (int)(nk % C::kStages);
          if (nk >= C::kStages &&
              !mbar_wait(k_empty(ks), (uint32_t)(((nk / C::kStages) - 1) & 1), abort_flag,
                         args.status, kSiteLoad)) {
            stop = true;
            break;
          }
          if (leader) mbar_expect_tx(k_full(ks), 2 * C::kKHalf);
          for (int blk = 0; blk < 2; ++blk)
            tma_load_4d_pair(sK + ks * C::kKHalf + blk * 8192, &args.tk2, k_full(ks), 64 * blk,
                             n0 + 64 * (int)rank, h, b);
          ++nk;
          const int vs = (int)(nv % C::kStages);
          if (nv >= C::kStages &&
              !mbar_wait(v_empty(vs), (uint32_t)(((nv / C::kStages) - 1) & 1), abort_flag,
                         args.status, kSiteLoad)) {
            stop = true;
            break;
          }
          if (leader) mbar_expect_tx(v_full(vs), 2 * C::kVHalf);
          tma_load_4d_pair(sV + vs * C::kVHalf, &args.tv, v_full(vs), 64 * (int)rank, n0, h, b);
          ++nv;
        }
      }
      if (*abort_flag && leader) {
        // the leader's barriers count both CTAs' copies: wait (bounded) for them
        for (int64_t i = nk > C::kStages ? nk - C::kStages : 0; i < nk; ++i)
          mbar_drain(k_full((int)(i % C::kStages)), (uint32_t)((i / C::kStages) & 1), args.status);
        for (int64_t i = nv > C::kStages ? nv - C::kStages : 0; i < nv; ++i)
          mbar_drain(v_full((int)(i % C::kStages)), (uint32_t)((i / C::kStages) & 1), args.status);
        if (qn0 > 0) mbar_drain(q_full(0), (uint32_t)((qn0 - 1) & 1), args.status);
        if (qn1 > 0) mbar_drain(q_full(1), (uint32_t)((qn1 - 1) & 1), args.status);
      }
    } else if (warp == 9 && lane == 0 && leader) {
      // ===================== MMA issuer (the leader) =====================
      const uint32_t idesc_s = make_idesc(BF16, 256, 128, false, false, args.negate != 0);
      const uint32_t idesc_o = make_idesc(BF16, 256, 128, false, true);
      const uint32_t kHiK = (uint32_t)(make_sdesc(0, 16, 1024) >> 32);
      const uint32_t kHiV = (uint32_t)(make_sdesc(0, 16384, 1024) >> 32);
      const uint32_t dQ = (uint32_t)make_sdesc(sQ, 16, 1024), dK = (uint32_t)make_sdesc(sK, 16, 1024);
      const uint32_t dV = (uint32_t)make_sdesc(sV, 16384, 1024);
      auto issue_s = [&](int t, int ks) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t oa = (uint32_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
          const uint32_t ob = (uint32_t)(((kk >> 2) * 8192 + (kk & 3) * 32) >> 4);
          mma_ss_pair(tmem + 128 * t, dQ + (uint32_t)(t * (C::kQTile >> 4)) + oa, kHiK,
                      dK + (uint32_t)(ks * (C::kKHalf >> 4)) + ob, kHiK, idesc_s, kk > 0 ? 1u : 0u);
        }
        commit_pair(s_full(t));
      };
      auto issue_pv = [&](int t, int vs, bool accumulate) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts_pair(tmem + C::kColO + 128 * t, tmem + 128 * t + 8 * kk,
                      dV + (uint32_t)(vs * (C::kVHalf >> 4)) + (uint32_t)((kk * 2048) >> 4), kHiV,
                      idesc_o, (accumulate || kk > 0) ? 1u : 0u);
        commit_pair(o_done(t));
      };
      // Phases: K / V rings follow the key tiles of all units (g); the S,
      // P and O barriers of query tile t the key tiles of the units that
      // include tile t (gt0, gt1); the Q barrier of tile t its loads (qn0,
      // qn1).  The unit body is instantiated for two tiles and for one (a
      // half unit), so its tile loops unroll and the counters stay in
      // registers.
      int64_t g = 0, gt0 = 0, gt1 = 0, qn0 = 0, qn1 = 0;
      auto run_unit = [&](auto tiles) -> bool {
        constexpr int NT = decltype(tiles)::value;
        bool ok = true;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          int64_t& qn = t == 0 ? qn0 : qn1;
          if (ok) ok = mbar_wait(q_full(t), (uint32_t)(qn & 1), abort_flag, args.status, kSiteMma);
          ++qn;
        }
        for (int it = 0; it < n_tiles && ok; ++it) {
          const int64_t gi = g + it;
          const int ks = (int)(gi % C::kStages);
          if (!(ok = mbar_wait(k_full(ks), (uint32_t)((gi / C::kStages) & 1), abort_flag,
                               args.status, kSiteMma)))
            break;
          const int vs = (int)((gi - 1) % C::kStages);
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            if (!ok) break;
            if (it > 0) {
              const int64_t gt = t == 0 ? gt0 : gt1;
              if (!(ok = mbar_wait(p_ready(t), (uint32_t)((gt + it - 1) & 1), abort_flag,
                                   args.status, kSiteMma)))
                break;
              if (t == 0 && !(ok = mbar_wait(v_full(vs), (uint32_t)(((gi - 1) / C::kStages) & 1),
                                             abort_flag, args.status, kSiteMma)))
                break;
              tc_fence_after();
              issue_pv(t, vs, it > 1);
              if (t == NT - 1) commit_pair(v_empty(vs));
            }
            tc_fence_after();
            issue_s(t, ks);
          }
          if (!ok) break;
          commit_pair(k_empty(ks));
          if (it == n_tiles - 1) commit_pair(q_empty);
        }
        if (ok) {
          const int64_t gl = g + n_tiles - 1;
          const int vs = (int)(gl % C::kStages);
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            if (!ok) break;
            const int64_t gt = t == 0 ? gt0 : gt1;
            if (!(ok = mbar_wait(p_ready(t), (uint32_t)((gt + n_tiles - 1) & 1), abort_flag,
                                 args.status, kSiteMma)))
              break;
            if (t == 0 && !(ok = mbar_wait(v_full(vs), (uint32_t)((gl / C::kStages) & 1), abort_flag,
                                           args.status, kSiteMma)))
              break;
            tc_fence_after();
            issue_pv(t, vs, n_tiles > 1);
            if (t == NT - 1) commit_pair(v_empty(vs));
          }
        }
        g += n_tiles;
        gt0 += n_tiles;
        if (NT == 2) gt1 += n_tiles;
        return ok;
      };
      bool ok = true;
      for (int64_t u = pair; u < n_units && ok; u += n_pairs) {
        int32_t b, h, m0;
        int nt;
        unit_of(u, b, h, m0, nt);
        ok = nt == 2 ? run_unit(std::integral_constant<int, 2>{})
                     : run_unit(std::integral_constant<int, 1>{});
      }
      // every product issued has completed before TMEM is released
      commit_pair(mma_done);
      mbar_drain(mma_done, 0, args.status);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::kHighRegs));
    // ===================== softmax / correction / epilogue =====================
    const int t = warp / 4;
    const int quad = warp % 4;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off + 128 * t;
    const uint32_t tO = tmem + lane_off + C::kColO + 128 * t;
    const float sl2 = args.scale_log2;
    int64_t g = 0;  // key tiles of the units that include this query tile
    bool ok = true;
    for (int64_t u = pair; u < n_units && ok; u += n_pairs) {
      int32_t b, h, m0;
      int nt;
      unit_of(u, b, h, m0, nt);
      if (t >= nt) continue;  // a half unit: tile 0 only
      const int32_t i = m0 + 128 * t + r;
      const bool valid = i < args.Sq;
      float m_used = -INFINITY, l = 0.f;
      for (int it = 0; it < n_tiles; ++it) {
        const int64_t gi = g + it;
        const int32_t n0 = it * 128;
        ok = mbar_wait(s_full(t), (uint32_t)(gi & 1), abort_flag, args.status, kSiteSoftmax);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        float s[128];
        {
          uint32_t raw[128];
          tmem_ld128(tS, raw);
#pragma unroll
          for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(raw[c]);
        }
        const bool full = n0 + 128 <= args.Sk;  // no mask: only keys past Sk are masked
        if (!full) {
          const int32_t z = args.Sk - 1 - n0;
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c > z) s[c] = -INFINITY;
        }
        float m8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) m8[k] = fmax3(s[k], s[8 + k], s[16 + k]);
#pragma unroll
        for (int c = 24; c < 120; c += 16)
#pragma unroll
          for (int k = 0; k < 8; ++k) m8[k] = fmax3(m8[k], s[c + k], s[c + 8 + k]);
#pragma unroll
        for (int k = 0; k < 8; ++k) m8[k] = fmaxf(m8[k], s[120 + k]);
        const float mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]),
                               fmaxf(m8[6], m8[7]));
        const float m_tile = (mx == -INFINITY) ? -INFINITY : mx * sl2;
        float alpha = 1.f;
        if (m_tile > m_used + 8.f || (m_used == -INFINITY && m_tile != -INFINITY)) {
          alpha = (m_used == -INFINITY) ? 0.f : ex2(m_used - m_tile);
          m_used = m_tile;
        }
        const float neg_m = (m_used == -INFINITY) ? 0.f : -m_used;
        uint64_t l4[4] = {0, 0, 0, 0};
        const uint64_t sl2x2 = f2_pack(sl2, sl2), negm2 = f2_pack(neg_m, neg_m);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t packed[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float x0 = s[32 * c + 2 * e], x1 = s[32 * c + 2 * e + 1];
            float y0, y1;
            f2_unpack(f2_fma(f2_pack(x0, x1), sl2x2, negm2), y0, y1);
            float p0 = ex2(y0), p1 = ex2(y1);
            if (!full) {
              p0 = (x0 == -INFINITY) ? 0.f : p0;
              p1 = (x1 == -INFINITY) ? 0.f : p1;
            }
            l4[e & 3] = f2_add(l4[e & 3], f2_pack(p0, p1));
            packed[e] = pack2<BF16>(p0, p1);
          }
          tmem_st16(tS + 16 * c, packed);
        }
        float la, lb, lc, ld;
        f2_unpack(f2_add(l4[0], l4[1]), la, lb);
        f2_unpack(f2_add(l4[2], l4[3]), lc, ld);
        l = alpha * l + ((la + lb) + (lc + ld));
        if (it > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
          ok = mbar_wait(o_done(t), (uint32_t)((gi - 1) & 1), abort_flag, args.status, kSiteSoftmax);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          tc_fence_after();
          for (int c = 0; c < 8; ++c) {
            uint32_t rr[16];
            tmem_ld16(tO + 16 * c, rr);
#pragma unroll
            for (int e = 0; e < 16; ++e) rr[e] = __float_as_uint(__uint_as_float(rr[e]) * alpha);
            tmem_st16(tO + 16 * c, rr);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        arrive_leader_warp(p_ready(t));
      }
      if (ok) {
        ok = mbar_wait(o_done(t), (uint32_t)((g + n_tiles - 1) & 1), abort_flag, args.status,
                       kSiteEpilogue);
        ok = __all_sync(0xffffffffu, ok);
      }
      if (ok) {
        tc_fence_after();
        const float inv = l > 0.f ? 1.f / l : 0.f;
        uint8_t* orow = valid ? o_row_ptr(b, h, i) : nullptr;
        // O / l to 16 bits, 16 columns at a time up to Dv (a multiple of 16;
        // the columns past it are TMA fill and not stored)
        for (int c = 0; c < 8; ++c) {
          uint32_t rr[16];
          tmem_ld16(tO + 16 * c, rr);
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            pk[e] = pack2<BF16>(__uint_as_float(rr[2 * e]) * inv, __uint_as_float(rr[2 * e + 1]) * inv);
          if (valid && 16 * c < args.Dv) {
            st_global_v4(orow + 32 * c, pk[0], pk[1], pk[2], pk[3]);
            st_global_v4(orow + 32 * c + 16, pk[4], pk[5], pk[6], pk[7]);
          }
        }
        if (valid && args.lse)
          *lse_ptr(b, h, i) = l > 0.f ? (m_used + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      }
      g += n_tiles;
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // neither CTA leaves while the pair's products may touch it
  if (warp == 9) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

template <bool BF16>
static cudaError_t launch_pair(const FwdArgs& args, cudaStream_t stream) {
  using C = PairCfg;
  static_assert(C::kSmemBytes <= 232448, "shared memory budget");
  static_assert(2 * 128 * C::kHighRegs + 128 * C::kLowRegs <= C::kThreads * C::kLaunchRegs,
                "register split exceeds the launch budget");
  auto kern = attn_fwd_pair_kernel<BF16>;
  static std::atomic<uint64_t> prepared{0};
  // Pairs that fit on the device at once (not every SM has a partner in its
  // cluster group), asked once per device: more would run as a second wave.
  static std::atomic<int> resident[64];
  const int64_t n_units = (int64_t)((args.Sq + 511) / 512) * args.H * args.B;
  if (n_units <= 0) return cudaSuccess;
  return prepared_launch(kern, prepared, args.dev, C::kSmemBytes, C::kLaunchRegs, [&] {
    const bool cache = args.dev >= 0 && args.dev < 64;
    int pairs = cache ? resident[args.dev].load(std::memory_order_relaxed) : 0;
    if (pairs <= 0) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * ((args.sms > 0 ? args.sms : 148) / 2));
      cfg.blockDim = dim3(C::kThreads);
      cfg.dynamicSmemBytes = C::kSmemBytes;
      cfg.stream = stream;
      if (cudaOccupancyMaxActiveClusters(&pairs, kern, &cfg) != cudaSuccess || pairs <= 0) {
        (void)cudaGetLastError();
        pairs = (args.sms > 0 ? args.sms : 148) / 2;
      } else if (cache) {
        resident[args.dev].store(pairs, std::memory_order_relaxed);
      }
    }
    const dim3 grid((unsigned)(2 * (n_units < pairs ? n_units : pairs)));
    kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(args);
  });
}

// Dense calls without a window, bias or dropout whose head dims take the
// 128-column tiles (the wider of D and Dv above 64; TMA fills the columns past
// a tensor's own head dim with zeros) and whose O rows end on a 16-column
// boundary (Dv a multiple of 16: O is stored in whole 16-column chunks).
bool fwd_pair_eligible(const FwdArgs& a) {
  return (a.D > 64 || a.Dv > 64) && a.D <= 128 && a.Dv <= 128 && a.Dv % 16 == 0 &&
         !a.q_packed && !a.k_packed &&
         !a.q_padded && !a.k_padded && a.wl == 2147483647 && a.wr == 2147483647 && !a.dropout &&
         !a.bias && a.Sq > 0 && a.Sk > 0;
}

cudaError_t launch_fwd_pair(const FwdArgs& args, cudaStream_t stream) {
  return args.bf16 ? launch_pair<true>(args, stream) : launch_pair<false>(args, stream);
}

}  // namespace attn
