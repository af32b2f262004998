// FlashAttention forward for sm_100a (the aotriton README, "Kernel Support":
// FlashAttention after Tri Dao): tiled online softmax, O and LSE out.
//
// A persistent kernel: one CTA per SM walks a list of work units.  A unit is
// NQ query tiles of 128 rows of one (sequence, head) (fewer where the
// sequence ends); its key tiles of 128 are those the Generalized Sliding
// Window lets any of its rows see (mask.cuh), and tiles with no masked pair
// skip the element test.  Without a mask units are numbered query block
// fastest, so the CTAs running at one time share a few heads' K and V in L2;
// under a window query block slowest, most expensive first (longest
// processing time first); they are dealt to the CTAs round robin, and a last
// round at most half full is split into single-tile units.  TMEM, the
// barriers and the K / V rings live for the whole kernel; every barrier
// phase follows one running count of key tiles, so the load of the next
// unit's tiles and its first S product overlap the current unit's last
// softmax and epilogue.
// Warp roles:
//   warps 0..4*NQ-1  softmax: one 4-warp group per query tile, one row per
//                    thread (TMEM lane = row); online exp2 softmax with lazy
//                    rescaling (an additive bias added from shared memory),
//                    P written into TMEM as 16-bit, O rescale and the
//                    epilogue (and the zero rows of fully masked units);
//   warp 4*NQ        TMA producer: Q once per unit (double-buffered at head
//                    dims up to 64), K and V through separate rings;
//   warp 4*NQ+1      MMA issuer (one thread): S = Q K^T (smem x smem) and
//                    O += P V (P from TMEM, V from smem), TMEM owner;
//   warp 4*NQ+2      with a bias: TMA producer of the bias tiles;
//   the rest         idle: they complete the producer / MMA warpgroup, whose
//                    registers go to the softmax groups through setmaxnreg.
// TMEM columns: S of tile t at [128 t, 128 t + 128); at head dim 128 P is
// written over S and O of tile t sits at [128 NQ + 128 t, ...); at head dims
// up to 64 P has columns of its own, [128 NQ + 64 t, ...), and O of tile t
// follows at [192 NQ + 64 t, ...), so the next S product can be issued as
// soon as the softmax has read S.
#include <cuda_runtime.h>

#include <type_traits>

#include "common.cuh"
#include "fwd.h"
#include "mask.cuh"

namespace attn {

template <int NQ, int DPAD, bool BIAS = false, bool DROPOUT = false>
struct FwdCfg {
  static constexpr int kSoftmaxWarps = 4 * NQ;
  static constexpr int kLoadWarp = kSoftmaxWarps;
  static constexpr int kMmaWarp = kSoftmaxWarps + 1;
  static constexpr int kBiasWarp = kSoftmaxWarps + 2;  // bias tile producer (with a bias)
  // One more full warpgroup after the softmax groups (TMA warp, MMA warp and
  // two spare warps), so registers can be moved between warpgroups.
  static constexpr int kThreads = 32 * (kSoftmaxWarps + 4);
  // Register split (setmaxnreg): the launch gives every thread kLaunchRegs;
  // the producer/MMA group drops to kLowRegs, the softmax groups rise to
  // kHighRegs.  NQ*128*kHighRegs + 128*kLowRegs <= kThreads*kLaunchRegs.  The
  // low shares are the smallest the producer / MMA code compiles into without
  // spilling, so the softmax (one 128-column score row per thread) gets the
  // most: 192 at head dim 128, 200 at 64 (with dropout at 128 its Philox
  // state needs the 136 / 184 split).
  static constexpr int kLaunchRegs = 168;  // 65536 / (4 sub-partitions x 3 warps x 32) rounded to 8
  static constexpr int kLowRegs = DPAD == 128 ? (DROPOUT ? 136 : 112) : 104;
  static constexpr int kHighRegs = (kThreads * kLaunchRegs - 128 * kLowRegs) / (128 * NQ) / 8 * 8;
  static constexpr int kBlocks = DPAD / 64;                // 128-byte swizzle blocks per row
  static constexpr int kTileBytes = 128 * DPAD * 2;        // one 128-row tile of Q, K or V
  // Sets of Q tiles: two at head dims up to 64 (the next unit's Q loads while
  // the current unit runs), one at 128 (shared memory holds no second set).
  // With a bias, one 128 x 128 bias tile per query tile takes the room of
  // K / V stages.
  static constexpr int kQBufs = DPAD == 128 ? 1 : 2;
  static constexpr int kKStages = BIAS ? 2 : (DPAD == 128 ? 3 : 4);
  static constexpr int kVStages = BIAS ? (DPAD == 128 ? 1 : 2) : (DPAD == 128 ? 2 : 4);
  static constexpr int kBiasTileBytes = BIAS ? 128 * 128 * 2 : 0;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBufs * NQ * kTileBytes;
  static constexpr int kOffV = kOffK + kKStages * kTileBytes;
  static constexpr int kOffB = kOffV + kVStages * kTileBytes;
  static constexpr int kOffBar = kOffB + NQ * kBiasTileBytes;
  // barriers: q_full[QB][NQ] q_empty[QB] k_full[KS] k_empty[KS] v_full[VS]
  //           v_empty[VS] s_full[NQ] p_ready[NQ] o_done[NQ] mma_done
  //           b_full[NQ] b_empty[NQ] s_free[NQ]
  static constexpr int kNumBars =
      kQBufs * (NQ + 1) + 2 * kKStages + 2 * kVStages + 3 * NQ + 1 + 3 * NQ;
  static constexpr int kOffMisc = kOffBar + 8 * kNumBars;
  static constexpr int kSmemBytes = kOffMisc + 16;
  // TMEM: S of tile t at [128 t, 128 t + 128).  At head dims up to 64, P of
  // tile t has columns of its own, [256 + 64 t, +64) as 16-bit pairs, so the
  // next S product can overwrite S as soon as the softmax has read it (it runs
  // while the softmax computes P); at 128 there is no room and P overwrites S.
  static constexpr bool kSplitP = DPAD == 64 && NQ == 2;
  static constexpr int kColP = kSplitP ? 128 * NQ : 0;
  static constexpr int kColO = kSplitP ? 128 * NQ + 64 * NQ : 128 * NQ;
  static constexpr int kTmemCols = (kColO + DPAD * NQ) <= 256 ? 256 : 512;
};

// O (+)= P V for one query tile: P from TMEM (8 columns per K step of 16
// keys), V MN-major in shared memory (next 16 keys = +2048 bytes).
__device__ __forceinline__ void fwd_issue_pv(uint32_t d, uint32_t a, uint32_t vd, uint32_t hi,
                                             uint32_t idesc, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    mma_ts2(d, a + 8 * kk, vd + (uint32_t)(kk * 2048 >> 4), hi, idesc,
            (accumulate || kk > 0) ? 1u : 0u);
}

// S = Q K^T for one query tile: both K-major; 16-column K steps are +32 bytes
// inside a 64-column block, blocks 16 KiB apart.  Padded head-dim columns
// are zero in both operands (TMA fill), so all KSTEPS steps are issued.
template <int KSTEPS>
__device__ __forceinline__ void fwd_issue_s(uint32_t d, uint32_t qd, uint32_t kd, uint32_t hi,
                                            uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < KSTEPS; ++kk) {
    const uint32_t o = (uint32_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
    mma_ss2(d, qd + o, hi, kd + o, hi, idesc, kk > 0 ? 1u : 0u);
  }
}

// One work unit: query rows [m0, m0 + 128 nt) of sequence b, head h, as nt
// query tiles (NQ; 1 for the halves of a split unit or where the sequence ends
// within the first tile of its last block).
struct FwdUnit {
  int32_t h, b, m0, nt, sq, sk, qrow0, krow0, bq, bk, nb, n_tiles;
  SeqWindow win;
};

// The unit list: n_full units of NQ tiles.  Without a mask every unit costs
// the same, and units are numbered query block fastest (last block first),
// then head, then sequence, so the CTAs that run at the same time work on the
// query blocks of a few heads and share those heads' K and V tiles in L2.
// Under a window the cost of a unit depends on its query block (a causal
// mask gives the last block of a head the most key tiles), and units are
// numbered query block slowest, last block first: dealt round robin, the
// most expensive units go out first and every CTA gets a mix (longest
// processing time first).  Dealt to G CTAs, the units fill n_full / G whole
// rounds and a last, partial one; when the units of that last round number
// at most G / 2, each is split into its NQ = 2 query tiles, units of one
// tile, so the last round takes about half as long.
struct FwdUnits {
  int64_t n_full, split_from, count;
};
template <int NQ>
__device__ __forceinline__ FwdUnits fwd_units(int32_t n_mblocks, int H, int B, int64_t G) {
  FwdUnits s;
  s.n_full = (int64_t)n_mblocks * H * B;
  const int64_t rounds = s.n_full / G, left = s.n_full - rounds * G;
  const bool split = NQ == 2 && rounds >= 1 && left > 0 && 2 * left <= G;
  s.split_from = split ? rounds * G : s.n_full;
  s.count = split ? s.split_from + 2 * left : s.n_full;
  return s;
}

// Unit u.  False if it holds no query row (a packed or padded sequence
// shorter than the largest one); n_tiles <= 0 marks a unit whose rows are all
// fully masked.  Every warp role decodes the same units the same way.
template <int NQ>
__device__ __forceinline__ bool fwd_unit(const FwdArgs& a, int32_t n_mblocks, const FwdUnits& us,
                                         int64_t u, FwdUnit& w) {
  int64_t fu = u;
  int32_t half = 0;
  w.nt = NQ;
  if (u >= us.split_from) {
    fu = us.split_from + (u - us.split_from) / 2;
    half = (int32_t)((u - us.split_from) & 1);
    w.nt = 1;
  }
  int64_t hb;
  int32_t mrev;
  if (a.units_by_cost) {
    const int64_t HB = (int64_t)a.H * a.B;
    mrev = (int32_t)(fu / HB);
    hb = fu - (int64_t)mrev * HB;
  } else {
    hb = fu / n_mblocks;
    mrev = (int32_t)(fu - hb * n_mblocks);
  }
  w.h = (int32_t)(hb % a.H);
  w.b = (int32_t)(hb / a.H);
  // Q and K sides are addressed independently: packed (rows from the
  // cumulative lengths, TMA batch coordinate 0), padded (dense rows, lengths
  // from the per-batch array) or dense.
  w.sq = a.Sq, w.sk = a.Sk, w.qrow0 = 0, w.krow0 = 0, w.bq = w.b, w.bk = w.b;
  if (a.q_packed) {
    stacked_bounds(a.cu_q, a.q_used ? a.used_q : nullptr, a.q_offsets != 0, w.b, a.total_q,
                   &w.qrow0, &w.sq);
    w.bq = 0;
  } else if (a.q_padded) {
    w.sq = min(max(a.cu_q[w.b], 0), a.Sq);
  }
  if (a.k_packed) {
    stacked_bounds(a.cu_k, a.k_used ? a.used_k : nullptr, a.k_offsets != 0, w.b, a.total_k,
                   &w.krow0, &w.sk);
    w.bk = 0;
  } else if (a.k_padded) {
    w.sk = min(max(a.cu_k[w.b], 0), a.Sk);
  }
  w.m0 = (n_mblocks - 1 - mrev) * 128 * NQ + 128 * half;
  if (w.m0 >= w.sq) return false;
  // a unit takes only the query tiles that hold rows of the sequence (the
  // last block of a sequence whose length is not a multiple of 128 NQ may
  // need fewer)
  w.nt = min(w.nt, (w.sq - w.m0 + 127) / 128);
  w.win = seq_window(a.wl, a.wr, a.bottom_right != 0, w.sq, w.sk);
  int32_t ne;
  fwd_tile_range(w.win, w.sq, w.sk, w.m0, 128 * w.nt, &w.nb, &ne);
  w.n_tiles = ne - w.nb;
  return true;
}

template <int NQ, int DPAD, bool BF16, bool DROPOUT, bool BIAS>
__global__ void __launch_bounds__(FwdCfg<NQ, DPAD, BIAS, DROPOUT>::kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ FwdArgs args) {
  using C = FwdCfg<NQ, DPAD, BIAS, DROPOUT>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int32_t n_mblocks = (args.Sq + 128 * NQ - 1) / (128 * NQ);
  const FwdUnits units = fwd_units<NQ>(n_mblocks, args.H, args.B, gridDim.x);
  const int64_t n_units = units.count;

  if (sbase & 1023) {  // the swizzled tiles need 1 KiB alignment
    if (threadIdx.x == 0) atomicOr(args.status, 1u << kSiteTeardown);
    return;
  }

  // Output addressing for row i (sequence-local) of a unit.
  auto o_row_ptr = [&](const FwdUnit& w, int32_t i) -> uint8_t* {
    int64_t off = args.q_packed ? (int64_t)(w.qrow0 + i) * args.o_stride[2]
                                : (int64_t)w.b * args.o_stride[0] + (int64_t)i * args.o_stride[2];
    off += (int64_t)w.h * args.o_stride[1];
    return reinterpret_cast<uint8_t*>(args.o) + 2 * off;
  };
  auto lse_ptr = [&](const FwdUnit& w, int32_t i) -> float* {
    int64_t idx;
    if (args.q_packed)
      idx = args.lse_th ? (int64_t)(w.qrow0 + i) * args.H + w.h
                        : (int64_t)w.h * args.total_q + w.qrow0 + i;
    else
      idx = args.lse_th ? ((int64_t)w.b * args.Sq + i) * args.H + w.h
                        : ((int64_t)w.b * args.H + w.h) * args.Sq + i;
    return args.lse + idx;
  };

  // ---- shared memory carve-up ----
  const uint32_t sQ = sbase + C::kOffQ, sK = sbase + C::kOffK, sV = sbase + C::kOffV;
  const uint32_t bar0 = sbase + C::kOffBar;
  auto q_full = [&](int qb, int t) { return bar0 + 8 * (qb * NQ + t); };
  const int bq0 = C::kQBufs * NQ;
  auto q_empty = [&](int qb) { return bar0 + 8 * (bq0 + qb); };
  const int bk0 = bq0 + C::kQBufs;
  auto k_full = [&](int s) { return bar0 + 8 * (bk0 + s); };
  auto k_empty = [&](int s) { return bar0 + 8 * (bk0 + C::kKStages + s); };
  auto v_full = [&](int s) { return bar0 + 8 * (bk0 + 2 * C::kKStages + s); };
  auto v_empty = [&](int s) { return bar0 + 8 * (bk0 + 2 * C::kKStages + C::kVStages + s); };
  const int bs = bk0 + 2 * C::kKStages + 2 * C::kVStages;
  auto s_full = [&](int t) { return bar0 + 8 * (bs + t); };
  auto p_ready = [&](int t) { return bar0 + 8 * (bs + NQ + t); };
  auto o_done = [&](int t) { return bar0 + 8 * (bs + 2 * NQ + t); };
  const uint32_t mma_done = bar0 + 8 * (bs + 3 * NQ);
  auto b_full = [&](int t) { return bar0 + 8 * (bs + 3 * NQ + 1 + t); };
  auto b_empty = [&](int t) { return bar0 + 8 * (bs + 4 * NQ + 1 + t); };
  // split P: the softmax group of tile t has read S(t), which the next S
  // product may overwrite
  auto s_free = [&](int t) { return bar0 + 8 * (bs + 5 * NQ + 1 + t); };
  const uint32_t sB = sbase + C::kOffB;  // bias tile of query tile t at sB + t * 32 KiB
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  if (threadIdx.x == 0) {
    for (int qb = 0; qb < C::kQBufs; ++qb) {
      for (int t = 0; t < NQ; ++t) mbar_init(q_full(qb, t), 1);
      mbar_init(q_empty(qb), 1);
    }
    for (int t = 0; t < NQ; ++t) {
      mbar_init(s_full(t), 1);
      mbar_init(p_ready(t), 4);  // one arrival per softmax warp
      mbar_init(o_done(t), 1);
    }
    for (int s = 0; s < C::kKStages; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
    }
    for (int s = 0; s < C::kVStages; ++s) {
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    mbar_init(mma_done, 1);
    for (int t = 0; t < NQ; ++t) {
      mbar_init(b_full(t), 1);
      mbar_init(b_empty(t), 4);  // one arrival per softmax warp of the tile
      mbar_init(s_free(t), 4);   // the same
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == C::kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Every barrier of the key-tile pipeline completes once per key tile, in
  // the order the units are taken, so its phase parity is that of a running
  // count of key tiles: g over all units for the K / V rings, gt[t] over the
  // units that include query tile t for that tile's barriers (a split unit
  // has tile 0 only).  The Q sets alternate per unit that has work (count
  // uc); each (set, tile) Q barrier counts its own loads.
  if (warp >= C::kSoftmaxWarps) {
  // The producer / MMA warpgroup gives registers back to the softmax groups.
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::kLowRegs));
  if (warp == C::kLoadWarp) {
    // ===================== TMA producer =====================
    if (lane == 0) {
      prefetch_tmap(&args.tq);
      prefetch_tmap(&args.tk);
      prefetch_tmap(&args.tv);
      int64_t nk = 0, nv = 0;  // K / V tiles issued (the running count g)
      int uc = 0;              // units with work whose Q tiles were issued
      int qn[C::kQBufs][NQ] = {};  // Q loads issued per (set, tile)
      bool stop = false;
      for (int64_t u = blockIdx.x; u < n_units && !stop; u += gridDim.x) {
        FwdUnit w;
        if (!fwd_unit<NQ>(args, n_mblocks, units, u, w) || w.n_tiles <= 0) continue;
        const int qb = uc % C::kQBufs, qr = uc / C::kQBufs;
        if (qr > 0 && !mbar_wait(q_empty(qb), (qr - 1) & 1, abort_flag, args.status, kSiteLoad))
          break;
        for (int t = 0; t < w.nt; ++t) {
          mbar_expect_tx(q_full(qb, t), C::kTileBytes);
          for (int blk = 0; blk < C::kBlocks; ++blk)
            tma_load_4d(sQ + (qb * NQ + t) * C::kTileBytes + blk * 16384, &args.tq, q_full(qb, t),
                        64 * blk, w.qrow0 + w.m0 + 128 * t, w.h, w.bq);
          ++qn[qb][t];
        }
        ++uc;
        for (int it = 0; it < w.n_tiles; ++it) {
          const int krow = w.krow0 + (w.nb + it) * 128;
          const int ks = (int)(nk % C::kKStages);
          const int64_t kr = nk / C::kKStages;
          if (kr > 0 && !mbar_wait(k_empty(ks), (uint32_t)((kr - 1) & 1), abort_flag, args.status,
                                   kSiteLoad)) {
            stop = true;
            break;
          }
          mbar_expect_tx(k_full(ks), C::kTileBytes);
          for (int blk = 0; blk < C::kBlocks; ++blk)
            tma_load_4d(sK + ks * C::kTileBytes + blk * 16384, &args.tk, k_full(ks), 64 * blk, krow,
                        w.h, w.bk);
          ++nk;
          const int vs = (int)(nv % C::kVStages);
          const int64_t vr = nv / C::kVStages;
          if (vr > 0 && !mbar_wait(v_empty(vs), (uint32_t)((vr - 1) & 1), abort_flag, args.status,
                                   kSiteLoad)) {
            stop = true;
            break;
          }
          mbar_expect_tx(v_full(vs), C::kTileBytes);
          for (int blk = 0; blk < C::kBlocks; ++blk)
            tma_load_4d(sV + vs * C::kTileBytes + blk * 16384, &args.tv, v_full(vs), 64 * blk, krow,
                        w.h, w.bk);
          ++nv;
        }
      }
      if (*abort_flag) {
        // Drain: wait (bounded) for every copy still in flight.
        for (int64_t i = nk > C::kKStages ? nk - C::kKStages : 0; i < nk; ++i)
          mbar_drain(k_full((int)(i % C::kKStages)), (uint32_t)((i / C::kKStages) & 1), args.status);
        for (int64_t i = nv > C::kVStages ? nv - C::kVStages : 0; i < nv; ++i)
          mbar_drain(v_full((int)(i % C::kVStages)), (uint32_t)((i / C::kVStages) & 1), args.status);
        for (int qb = 0; qb < C::kQBufs; ++qb)
          for (int t = 0; t < NQ; ++t)
            if (qn[qb][t] > 0)
              mbar_drain(q_full(qb, t), (uint32_t)((qn[qb][t] - 1) & 1), args.status);
      }
    }
  } else if (warp == C::kMmaWarp) {
    // ===================== MMA issuer =====================
    // Shared-memory descriptors are built once and advanced by adding (byte
    // offset >> 4) to their start-address field, so issuing an MMA costs a
    // 64-bit add, not a rebuilt descriptor.
    if (lane == 0) {
      const uint32_t idesc_s = make_idesc(BF16, 128, 128, false, false, args.negate != 0);
      const uint32_t idesc_o = make_idesc(BF16, 128, args.Dv16, false, true);
      // descriptor words: hi is fixed per layout, lo carries the start address
      const uint32_t kHiK = (uint32_t)(make_sdesc(0, 16, 1024) >> 32);
      const uint32_t kHiV = (uint32_t)(make_sdesc(0, 16384, 1024) >> 32);
      const uint32_t dQ = (uint32_t)make_sdesc(sQ, 16, 1024), dK = (uint32_t)make_sdesc(sK, 16, 1024);
      const uint32_t dV = (uint32_t)make_sdesc(sV, 16384, 1024);
      constexpr uint32_t kTile16 = C::kTileBytes >> 4;
      // The unit loop is instantiated twice, with the V padding clears (a K
      // side whose sequences leave rows unused: padded, or stacked with used
      // lengths) and without them, so other calls run code that carries no
      // trace of the clears.
      auto run = [&](auto padding) {
        int64_t g = 0;        // key tiles of the units done so far
        int64_t gt[NQ] = {};  // the same, per query tile
        int uc = 0;           // units with work so far
        int qw[C::kQBufs][NQ] = {};  // Q tiles consumed per (set, tile)
        bool ok = true;
        for (int64_t u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
          FwdUnit w;
          if (!fwd_unit<NQ>(args, n_mblocks, units, u, w) || w.n_tiles <= 0) continue;
          const int qb = uc % C::kQBufs;
          ++uc;
          // Rows of a V tile past seqlen_k may hold the caller's padding (a
          // padded batch, the unused rows of a slot or a gap between stacked
          // sequences), not TMA zero fill; P is 0 there, but 0 * NaN is not,
          // so the rows are zeroed before the tensor cores read the tile.
          auto clear_v_padding = [&](int it_v, int vs) {
            if constexpr (decltype(padding)::value) {
              const int r0 = w.sk - (w.nb + it_v) * 128;
              if (r0 < 128) {
                zero_tile_rows(sV + vs * C::kTileBytes, r0, C::kBlocks);
                fence_proxy_async_smem();
              }
            } else {
              (void)it_v, (void)vs;
            }
          };
          // O_t (+)= P_t V, then O_t's completion on o_done(t).
          auto issue_pv = [&](int t, int vs, bool accumulate) {
            fwd_issue_pv(tmem + C::kColO + DPAD * t, tmem + (C::kSplitP ? C::kColP + 64 * t : 128 * t),
                         dV + (uint32_t)vs * kTile16, kHiV, idesc_o, accumulate);
            tc_commit(o_done(t));
          };
          // S_t = Q_t K^T, then its completion on s_full(t).
          auto issue_s = [&](int t, int ks) {
            fwd_issue_s<DPAD / 16>(tmem + 128 * t, dQ + (uint32_t)(qb * NQ + t) * kTile16,
                                   dK + (uint32_t)ks * kTile16, kHiK, idesc_s);
            tc_commit(s_full(t));
          };
          for (int t = 0; t < w.nt && ok; ++t) {
            ok = mbar_wait(q_full(qb, t), (uint32_t)(qw[qb][t] & 1), abort_flag, args.status,
                           kSiteMma);
            ++qw[qb][t];
          }
          if constexpr (C::kSplitP) {
            // S(t, it + 1) goes out as soon as the softmax has read S(t, it),
            // before P V of tile it: the products of the next key tile run
            // while the softmax computes P.
            auto issue_s_tile = [&](int it) -> bool {  // S of key tile it, both query tiles
              const int64_t gi = g + it;
              const int ks = (int)(gi % C::kKStages);
              if (!mbar_wait(k_full(ks), (uint32_t)((gi / C::kKStages) & 1), abort_flag,
                             args.status, kSiteMma))
                return false;
              for (int t = 0; t < w.nt; ++t) {
                const int64_t prev = gt[t] + it - 1;  // the S(t) the softmax must have read
                if (prev >= 0 && !mbar_wait(s_free(t), (uint32_t)(prev & 1), abort_flag,
                                            args.status, kSiteMma))
                  return false;
                tc_fence_after();
                issue_s(t, ks);
              }
              tc_commit(k_empty(ks));
              if (it == w.n_tiles - 1) tc_commit(q_empty(qb));
              return true;
            };
            ok = issue_s_tile(0);
            for (int it = 0; it < w.n_tiles && ok; ++it) {
              if (it + 1 < w.n_tiles && !(ok = issue_s_tile(it + 1))) break;
              const int64_t gi = g + it;
              const int vs = (int)(gi % C::kVStages);
              for (int t = 0; t < w.nt && ok; ++t) {
                if (!(ok = mbar_wait(p_ready(t), (uint32_t)((gt[t] + it) & 1), abort_flag,
                                     args.status, kSiteMma)))
                  break;
                if (t == 0) {
                  if (!(ok = mbar_wait(v_full(vs), (uint32_t)((gi / C::kVStages) & 1), abort_flag,
                                       args.status, kSiteMma)))
                    break;
                  clear_v_padding(it, vs);
                }
                tc_fence_after();
                issue_pv(t, vs, it > 0);
                if (t == w.nt - 1) tc_commit(v_empty(vs));
              }
            }
          } else {
          for (int it = 0; it < w.n_tiles && ok; ++it) {
            const int64_t gi = g + it;
            const int ks = (int)(gi % C::kKStages);
            if (!(ok = mbar_wait(k_full(ks), (uint32_t)((gi / C::kKStages) & 1), abort_flag,
                                 args.status, kSiteMma)))
              break;
            const int vs = (int)((gi - 1) % C::kVStages);  // V of the previous key tile
            for (int t = 0; t < w.nt && ok; ++t) {
              if (it > 0) {
                if (!(ok = mbar_wait(p_ready(t), (uint32_t)((gt[t] + it - 1) & 1), abort_flag,
                                     args.status, kSiteMma)))
                  break;
                if (t == 0) {
                  if (!(ok = mbar_wait(v_full(vs), (uint32_t)(((gi - 1) / C::kVStages) & 1),
                                       abort_flag, args.status, kSiteMma)))
                    break;
                  clear_v_padding(it - 1, vs);
                }
                tc_fence_after();
                issue_pv(t, vs, it > 1);
                if (t == w.nt - 1) tc_commit(v_empty(vs));
              }
              issue_s(t, ks);
            }
            if (!ok) break;
            tc_commit(k_empty(ks));
            // the unit's Q set is free once its last S products are done
            if (it == w.n_tiles - 1) tc_commit(q_empty(qb));
          }
          if (ok) {
            const int64_t gl = g + w.n_tiles - 1;
            const int vs = (int)(gl % C::kVStages);
            for (int t = 0; t < w.nt && ok; ++t) {
              if (!(ok = mbar_wait(p_ready(t), (uint32_t)((gt[t] + w.n_tiles - 1) & 1), abort_flag,
                                   args.status, kSiteMma)))
                break;
              if (t == 0) {
                if (!(ok = mbar_wait(v_full(vs), (uint32_t)((gl / C::kVStages) & 1), abort_flag,
                                     args.status, kSiteMma)))
                  break;
                clear_v_padding(w.n_tiles - 1, vs);
              }
              tc_fence_after();
              issue_pv(t, vs, w.n_tiles > 1);
              if (t == w.nt - 1) tc_commit(v_empty(vs));
            }
          }
          }
          g += w.n_tiles;
          for (int t = 0; t < w.nt; ++t) gt[t] += w.n_tiles;
        }
      };
      if (args.k_padded || args.k_used)
        run(Flag<true>{});
      else
        run(Flag<false>{});
      // Everything issued has completed before TMEM is released.
      tc_commit(mma_done);
      mbar_drain(mma_done, 0, args.status);
    }
  } else if (BIAS && warp == C::kBiasWarp) {
    // ===================== bias tile producer =====================
    // The bias tile (query tile t, key tile) of every unit, in the order the
    // softmax groups take them: one buffer per query tile, refilled as soon
    // as the group has added the previous tile to its scores.  A thread of
    // its own, so no K / V wait delays a bias load.
    if (lane == 0) {
      prefetch_tmap(&args.tb);
      int64_t nbt[NQ] = {};  // bias tiles issued per query tile
      bool stop = false;
      for (int64_t u = blockIdx.x; u < n_units && !stop; u += gridDim.x) {
        FwdUnit w;
        if (!fwd_unit<NQ>(args, n_mblocks, units, u, w) || w.n_tiles <= 0) continue;
        const int cb = args.bias_b_bcast ? 0 : w.b, ch = args.bias_h_bcast ? 0 : w.h;
        for (int it = 0; it < w.n_tiles && !stop; ++it) {
          const int n0 = (w.nb + it) * 128;
          for (int t = 0; t < w.nt; ++t) {
            if (nbt[t] > 0 && !mbar_wait(b_empty(t), (uint32_t)((nbt[t] - 1) & 1), abort_flag,
                                         args.status, kSiteLoad)) {
              stop = true;
              break;
            }
            mbar_expect_tx(b_full(t), C::kBiasTileBytes);
            for (int blk = 0; blk < 2; ++blk)
              tma_load_4d(sB + t * C::kBiasTileBytes + blk * 16384, &args.tb, b_full(t),
                          n0 + 64 * blk, w.m0 + 128 * t, ch, cb);
            ++nbt[t];
          }
        }
      }
      if (*abort_flag) {
        for (int t = 0; t < NQ; ++t)
          if (nbt[t] > 0) mbar_drain(b_full(t), (uint32_t)((nbt[t] - 1) & 1), args.status);
      }
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::kHighRegs));
    // ===================== softmax / correction / epilogue =====================
    const int t = warp / 4;               // query tile of this warp group
    const int quad = warp % 4;            // TMEM lane quadrant
    const int r = quad * 32 + lane;       // row within the tile
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off + 128 * t;
    const uint32_t tO = tmem + lane_off + C::kColO + DPAD * t;
    const uint32_t tP = C::kSplitP ? tmem + lane_off + C::kColP + 64 * t : tS;  // where P goes
    const float sl2 = args.scale_log2;
    int64_t g = 0;  // key tiles of the units that include this query tile
    bool ok = true;
    for (int64_t u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      FwdUnit w;
      if (!fwd_unit<NQ>(args, n_mblocks, units, u, w) || t >= w.nt) continue;
      const int32_t i = w.m0 + 128 * t + r;  // sequence-local query row
      const bool valid = i < w.sq;
      if (w.n_tiles <= 0) {
        // Every row of the unit is fully masked: O = 0 (only the first D
        // columns are written) and LSE = -inf.
        if (valid) {
          zero_row16(o_row_ptr(w, i), args.Dv, 0, 1);
          if (args.lse) *lse_ptr(w, i) = -INFINITY;
        }
        continue;
      }
      const int32_t lo = row_lo(w.win, i), hi = row_hi(w.win, i, w.sk);
      const uint32_t bh = (uint32_t)(w.b * args.H + w.h);  // dropout counter word
      (void)bh;
      // With a bias the logits are formed in the log2 domain below
      // (c S log2(e) + B log2(e)), and the shift works at unit scale.
      const float sl2e = BIAS ? 1.f : sl2;
      // Row r of this tile's staged bias (128-byte swizzled 64-column blocks).
      const uint32_t brow_s = sB + t * C::kBiasTileBytes + r * 128;
      (void)brow_s;
      float m_used = -INFINITY, l = 0.f;
      for (int it = 0; it < w.n_tiles; ++it) {
        const int64_t gi = g + it;
        const int32_t n0 = (w.nb + it) * 128;
        ok = mbar_wait(s_full(t), (uint32_t)(gi & 1), abort_flag, args.status, kSiteSoftmax);
        if (BIAS && ok)
          ok = mbar_wait(b_full(t), (uint32_t)(gi & 1), abort_flag, args.status, kSiteSoftmax);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        float s[128];
        if constexpr (BIAS) {
          // Four TMEM loads of 32 columns, each folded with its 32 bias
          // columns (rows past the tensor read TMA's zero fill; rows past the
          // sequence are not stored).
#pragma unroll
          for (int part = 0; part < 4; ++part) {
            uint32_t raw[32];
            tmem_ld32(tS + 32 * part, raw);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int ch = 4 * part + q;  // 16-byte chunk of the row, 0..15
              uint32_t wv[4];
              asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                           : "=r"(wv[0]), "=r"(wv[1]), "=r"(wv[2]), "=r"(wv[3])
                           : "r"(brow_s + (ch >> 3) * 16384 + (((ch & 7) ^ (r & 7)) << 4)));
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const int c = 8 * ch + e;
                const float bias = h16_to_f32<BF16>((wv[e >> 1] >> (16 * (e & 1))) & 0xFFFFu);
                s[c] = fmaf(__uint_as_float(raw[8 * q + e]), sl2, bias * 1.4426950408889634f);
              }
            }
          }
          // the bias tile has been read: its buffer can take the next one
          mbar_arrive_warp(b_empty(t));
        } else {
          // The whole score row in one TMEM load.
          uint32_t raw[128];
          tmem_ld128(tS, raw);
#pragma unroll
          for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(raw[c]);
        }
        if constexpr (C::kSplitP) {
          // S has been read (the loads above waited for their data): the next
          // S product may overwrite it
          tc_fence_before();
          mbar_arrive_warp(s_free(t));
        }
        const bool full = tile_is_full(w.win, w.sq, w.sk, w.m0 + 128 * t, n0);
        if (!full) {
          const int32_t a = lo - n0, z = hi - n0;  // allowed columns [a, z]
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c < a || c > z) s[c] = -INFINITY;
        }
        // Row maximum over 8 independent chains of three-input maxima: chain k
        // takes columns k, k+8, ..., k+120 (0-23 to start, 24-119 in pairs,
        // 120-127 last).
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
        const float m_tile = (mx == -INFINITY) ? -INFINITY : mx * sl2e;
        // Lazy rescale: keep the running reference unless the new maximum
        // exceeds it by more than 2^8 (P stays below 256, exact in fp32 sums).
        float alpha = 1.f;
        if (m_tile > m_used + 8.f || (m_used == -INFINITY && m_tile != -INFINITY)) {
          alpha = (m_used == -INFINITY) ? 0.f : ex2(m_used - m_tile);
          m_used = m_tile;
        }
        const float neg_m = (m_used == -INFINITY) ? 0.f : -m_used;
        // Scale-and-shift and the row sum run on packed fp32 pairs.
        uint64_t l4[4] = {0, 0, 0, 0};
        const uint64_t sl2x2 = f2_pack(sl2e, sl2e), negm2 = f2_pack(neg_m, neg_m);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          // Dropout: bit k of `keep` says whether column 32 c + k survives.
          // Key j = n0 + 32 c + 4 g + word takes that word of Philox on the
          // counter (j div 4, i, b H + h, offset); the row sum (hence LSE)
          // keeps every element, P V only the kept ones.
          uint32_t keep = 0xFFFFFFFFu;
          if constexpr (DROPOUT) {
            keep = 0;
            const uint32_t g0 = (uint32_t)(n0 >> 2) + 8u * c;
#pragma unroll
            for (int gq = 0; gq < 8; ++gq) {
              const uint4 wd = philox4x32_10(make_uint4(g0 + gq, (uint32_t)i, bh, args.philox_offset),
                                             args.seed_lo, args.seed_hi);
              keep |= ((wd.x < args.keep_below ? 1u : 0u) | (wd.y < args.keep_below ? 2u : 0u) |
                       (wd.z < args.keep_below ? 4u : 0u) | (wd.w < args.keep_below ? 8u : 0u))
                      << (4 * gq);
            }
          }
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
            if constexpr (DROPOUT) {
              p0 = (keep >> (2 * e)) & 1u ? p0 : 0.f;
              p1 = (keep >> (2 * e + 1)) & 1u ? p1 : 0.f;
            }
            packed[e] = pack2<BF16>(p0, p1);
          }
          if (C::kSplitP && c == 0 && it > 0) {
            // P of the previous key tile must have been read by its P V
            // product before this tile's P overwrites it (waited for only now,
            // after the first 32 columns' exponentials)
            ok = mbar_wait(o_done(t), (uint32_t)((gi - 1) & 1), abort_flag, args.status,
                           kSiteSoftmax);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
          }
          tmem_st16(tP + 16 * c, packed);
        }
        if (!ok) break;
        float la, lb, lc, ld;
        f2_unpack(f2_add(l4[0], l4[1]), la, lb);
        f2_unpack(f2_add(l4[2], l4[3]), lc, ld);
        const float rowsum = (la + lb) + (lc + ld);
        l = alpha * l + rowsum;
        if (it > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
          // O_t must hold PV of the previous tile before it is rescaled.
          ok = mbar_wait(o_done(t), (uint32_t)((gi - 1) & 1), abort_flag, args.status,
                         kSiteSoftmax);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          tc_fence_after();
          for (int c = 0; c < args.Dv16 / 16; ++c) {
            uint32_t rr[16];
            tmem_ld16(tO + 16 * c, rr);
#pragma unroll
            for (int e = 0; e < 16; ++e) rr[e] = __float_as_uint(__uint_as_float(rr[e]) * alpha);
            tmem_st16(tO + 16 * c, rr);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive_warp(p_ready(t));
      }
      if (ok) {
        ok = mbar_wait(o_done(t), (uint32_t)((g + w.n_tiles - 1) & 1), abort_flag, args.status,
                       kSiteEpilogue);
        ok = __all_sync(0xffffffffu, ok);
      }
      if (ok) {
        tc_fence_after();
        // with dropout, the kept elements carry the factor 1 / (1 - p)
        const float inv = l > 0.f ? (DROPOUT ? args.drop_scale : 1.f) / l : 0.f;
        uint8_t* orow = valid ? o_row_ptr(w, i) : nullptr;
        for (int c = 0; c < args.Dv16 / 16; ++c) {
          uint32_t rr[16];
          tmem_ld16(tO + 16 * c, rr);
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            pk[e] = pack2<BF16>(__uint_as_float(rr[2 * e]) * inv, __uint_as_float(rr[2 * e + 1]) * inv);
          if (valid) st_row16(orow, c, pk, args.Dv);
        }
        if (valid && args.lse)
          *lse_ptr(w, i) = l > 0.f ? (m_used + __log2f(l)) * 0.69314718055994531f : -INFINITY;
        // The O columns are read: the next unit's first P V product, which
        // overwrites them, is issued only after this thread's next p_ready
        // arrival (whose fence orders these loads before it).
      }
      g += w.n_tiles;
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == C::kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int NQ, int DPAD, bool BF16, bool DROPOUT, bool BIAS>
static cudaError_t launch(const FwdArgs& args, int64_t n_units, cudaStream_t stream) {
  using C = FwdCfg<NQ, DPAD, BIAS, DROPOUT>;
  static_assert(C::kSmemBytes <= 232448, "shared memory budget");
  static_assert(NQ * 128 * C::kHighRegs + 128 * C::kLowRegs <= C::kThreads * C::kLaunchRegs,
                "register split exceeds the launch budget");
  auto kern = attn_fwd_kernel<NQ, DPAD, BF16, DROPOUT, BIAS>;
  static std::atomic<uint64_t> prepared{0};
  // One CTA per SM (the shared-memory footprint allows no second one).
  const int64_t sms = args.sms > 0 ? args.sms : 148;
  const dim3 grid((unsigned)(n_units < sms ? n_units : sms));
  return prepared_launch(kern, prepared, args.dev, C::kSmemBytes, C::kLaunchRegs, [&] {
    kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(args);
  });
}

cudaError_t launch_fwd(const FwdArgs& args, cudaStream_t stream) {
  if (fwd_pair_eligible(args)) return launch_fwd_pair(args, stream);
  constexpr int NQ = 2;
  const int rows = 128 * NQ;
  const int64_t n_units = (int64_t)((args.Sq + rows - 1) / rows) * args.H * args.B;
  if (n_units == 0) return cudaSuccess;
  const bool bf16 = args.bf16 != 0;
  // Q, K, V and O tiles all take the wider of the two head dims (TMA fills
  // the columns past a tensor's own head dim with zeros).
  const bool narrow = args.D <= 64 && args.Dv <= 64;
  // Runtime choices to template arguments: head-dim class, dtype, dropout,
  // bias.
  auto by_bias = [&](auto dpad, auto bf, auto drop) -> cudaError_t {
    constexpr int P = decltype(dpad)::value;
    constexpr bool F = decltype(bf)::value, DR = decltype(drop)::value;
    return args.bias ? launch<NQ, P, F, DR, true>(args, n_units, stream)
                     : launch<NQ, P, F, DR, false>(args, n_units, stream);
  };
  auto by_drop = [&](auto dpad, auto bf) -> cudaError_t {
    return args.dropout ? by_bias(dpad, bf, Flag<true>{}) : by_bias(dpad, bf, Flag<false>{});
  };
  auto by_dtype = [&](auto dpad) -> cudaError_t {
    return bf16 ? by_drop(dpad, Flag<true>{}) : by_drop(dpad, Flag<false>{});
  };
  return narrow ? by_dtype(std::integral_constant<int, 64>{})
                : by_dtype(std::integral_constant<int, 128>{});
}

}  // namespace attn
