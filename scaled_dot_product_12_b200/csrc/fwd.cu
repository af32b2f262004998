// FlashAttention forward for sm_100a (the aotriton README, "Kernel Support":
// FlashAttention after Tri Dao): tiled online softmax, O and LSE out.
//
// One CTA owns NQ query tiles of 128 rows of one (sequence, head) and walks
// the key tiles of 128 that the Generalized Sliding Window lets any of its
// rows see (mask.cuh), skipping the element test on tiles with no masked
// pair.  Warp roles:
//   warps 0..4*NQ-1  softmax: one 4-warp group per query tile, one row per
//                    thread (TMEM lane = row); online exp2 softmax with lazy
//                    rescaling, P written back into TMEM as 16-bit, O rescale
//                    and the epilogue;
//   warp 4*NQ        TMA producer: Q once, K and V through separate rings;
//   warp 4*NQ+1      MMA issuer (one thread): S = Q K^T (smem x smem) and
//                    O += P V (P from TMEM, V from smem), TMEM owner;
//   warps 4*NQ+2..   idle: they complete the producer / MMA warpgroup, whose
//                    registers go to the softmax groups through setmaxnreg.
// TMEM columns: S/P of tile t at [128 t, 128 t + 128), O of tile t at
// [128 NQ + DPAD t, ...).
#include <cuda_runtime.h>

#include "common.cuh"
#include "fwd.h"
#include "mask.cuh"

namespace attn {

template <int NQ, int DPAD>
struct FwdCfg {
  static constexpr int kSoftmaxWarps = 4 * NQ;
  static constexpr int kLoadWarp = kSoftmaxWarps;
  static constexpr int kMmaWarp = kSoftmaxWarps + 1;
  // One more full warpgroup after the softmax groups (TMA warp, MMA warp and
  // two spare warps), so registers can be moved between warpgroups.
  static constexpr int kThreads = 32 * (kSoftmaxWarps + 4);
  // Register split (setmaxnreg): the launch gives every thread kLaunchRegs;
  // the producer/MMA group drops to kLowRegs, the softmax groups rise to
  // kHighRegs.  NQ*128*kHighRegs + 128*kLowRegs == kThreads*kLaunchRegs.
  static constexpr int kLaunchRegs = 168;  // 65536 / (4 sub-partitions x 3 warps x 32) rounded to 8
  static constexpr int kLowRegs = 136;
  static constexpr int kHighRegs = (kThreads * kLaunchRegs - 128 * kLowRegs) / (128 * NQ) / 8 * 8;
  static constexpr int kBlocks = DPAD / 64;                // 128-byte swizzle blocks per row
  static constexpr int kTileBytes = 128 * DPAD * 2;        // one 128-row tile of Q, K or V
  static constexpr int kKStages = DPAD == 128 ? 3 : 4;
  static constexpr int kVStages = DPAD == 128 ? 2 : 4;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + NQ * kTileBytes;
  static constexpr int kOffV = kOffK + kKStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kVStages * kTileBytes;
  // barriers: q_full[NQ] k_full[KS] k_empty[KS] v_full[VS] v_empty[VS]
  //           s_full[NQ] p_ready[NQ] o_done[NQ] mma_done
  static constexpr int kNumBars = 4 * NQ + 2 * kKStages + 2 * kVStages + 1;
  static constexpr int kOffMisc = kOffBar + 8 * kNumBars;
  static constexpr int kSmemBytes = kOffMisc + 16;
  static constexpr int kTmemCols = (128 * NQ + DPAD * NQ) <= 256 ? 256 : 512;
  static constexpr int kColO = 128 * NQ;
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

template <int NQ, int DPAD, bool BF16>
__global__ void __launch_bounds__(FwdCfg<NQ, DPAD>::kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ FwdArgs args) {
  using C = FwdCfg<NQ, DPAD>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- which (sequence, head, query rows) this CTA owns ----
  const int mblk = gridDim.x - 1 - blockIdx.x;  // longest causal rows first
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  // Q and K sides are addressed independently: packed (rows from the
  // cumulative lengths, TMA batch coordinate 0), padded (dense rows, lengths
  // from the per-batch array) or dense.
  int32_t sq = args.Sq, sk = args.Sk, qrow0 = 0, krow0 = 0, bq = b, bk = b;
  if (args.q_packed) {
    qrow0 = args.cu_q[b];
    sq = args.cu_q[b + 1] - qrow0;
    bq = 0;
  } else if (args.q_padded) {
    sq = min(max(args.cu_q[b], 0), args.Sq);
  }
  if (args.k_packed) {
    krow0 = args.cu_k[b];
    sk = args.cu_k[b + 1] - krow0;
    bk = 0;
  } else if (args.k_padded) {
    sk = min(max(args.cu_k[b], 0), args.Sk);
  }
  const int32_t m0 = mblk * 128 * NQ;
  if (m0 >= sq) return;
  const SeqWindow win = seq_window(args.wl, args.wr, args.bottom_right != 0, sq, sk);
  int32_t nb, ne;
  fwd_tile_range(win, sq, sk, m0, 128 * NQ, &nb, &ne);
  const int n_tiles = ne - nb;

  // Output addressing for row i (sequence-local) of this head.
  auto o_row_ptr = [&](int32_t i) -> uint8_t* {
    int64_t off = args.q_packed ? (int64_t)(qrow0 + i) * args.o_stride[2]
                              : (int64_t)b * args.o_stride[0] + (int64_t)i * args.o_stride[2];
    off += (int64_t)h * args.o_stride[1];
    return reinterpret_cast<uint8_t*>(args.o) + 2 * off;
  };
  auto lse_ptr = [&](int32_t i) -> float* {
    int64_t idx;
    if (args.q_packed)
      idx = args.lse_th ? (int64_t)(qrow0 + i) * args.H + h : (int64_t)h * args.total_q + qrow0 + i;
    else
      idx = args.lse_th ? ((int64_t)b * args.Sq + i) * args.H + h
                        : ((int64_t)b * args.H + h) * args.Sq + i;
    return args.lse + idx;
  };

  if (n_tiles <= 0) {
    // Every row of these tiles is fully masked: O = 0 (only the first D
    // columns are written) and LSE = -inf.
    const int rows = min(128 * NQ, sq - m0);
    for (int idx = threadIdx.x; idx < rows * (args.D / 8); idx += blockDim.x) {
      const int r = idx / (args.D / 8), c = idx % (args.D / 8);
      st_global_v4(o_row_ptr(m0 + r) + 16 * c, 0u, 0u, 0u, 0u);
    }
    if (args.lse)
      for (int r = threadIdx.x; r < rows; r += blockDim.x) *lse_ptr(m0 + r) = -INFINITY;
    return;
  }

  if (sbase & 1023) {  // the swizzled tiles need 1 KiB alignment
    if (threadIdx.x == 0) atomicOr(args.status, 1u << kSiteTeardown);
    return;
  }

  // ---- shared memory carve-up ----
  const uint32_t sQ = sbase + C::kOffQ, sK = sbase + C::kOffK, sV = sbase + C::kOffV;
  const uint32_t bar0 = sbase + C::kOffBar;
  auto q_full = [&](int t) { return bar0 + 8 * t; };
  auto k_full = [&](int s) { return bar0 + 8 * (NQ + s); };
  auto k_empty = [&](int s) { return bar0 + 8 * (NQ + C::kKStages + s); };
  auto v_full = [&](int s) { return bar0 + 8 * (NQ + 2 * C::kKStages + s); };
  auto v_empty = [&](int s) { return bar0 + 8 * (NQ + 2 * C::kKStages + C::kVStages + s); };
  const int bs = NQ + 2 * C::kKStages + 2 * C::kVStages;
  auto s_full = [&](int t) { return bar0 + 8 * (bs + t); };
  auto p_ready = [&](int t) { return bar0 + 8 * (bs + NQ + t); };
  auto o_done = [&](int t) { return bar0 + 8 * (bs + 2 * NQ + t); };
  const uint32_t mma_done = bar0 + 8 * (bs + 3 * NQ);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  if (threadIdx.x == 0) {
    for (int t = 0; t < NQ; ++t) {
      mbar_init(q_full(t), 1);
      mbar_init(s_full(t), 1);
      mbar_init(p_ready(t), 128);
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

  if (warp >= C::kSoftmaxWarps) {
  // The producer / MMA warpgroup gives registers back to the softmax groups.
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::kLowRegs));
  if (warp == C::kLoadWarp) {
    // ===================== TMA producer =====================
    if (lane == 0) {
      prefetch_tmap(&args.tq);
      prefetch_tmap(&args.tk);
      prefetch_tmap(&args.tv);
      for (int t = 0; t < NQ; ++t) {
        mbar_expect_tx(q_full(t), C::kTileBytes);
        for (int blk = 0; blk < C::kBlocks; ++blk)
          tma_load_4d(sQ + t * C::kTileBytes + blk * 16384, &args.tq, q_full(t), 64 * blk,
                      qrow0 + m0 + 128 * t, h, bq);
      }
      int issued = 0;
      for (int it = 0; it < n_tiles; ++it) {
        const int krow = krow0 + (nb + it) * 128;
        const int ks = it % C::kKStages, kr = it / C::kKStages;
        if (kr > 0 && !mbar_wait(k_empty(ks), (kr - 1) & 1, abort_flag, args.status, kSiteLoad))
          break;
        mbar_expect_tx(k_full(ks), C::kTileBytes);
        for (int blk = 0; blk < C::kBlocks; ++blk)
          tma_load_4d(sK + ks * C::kTileBytes + blk * 16384, &args.tk, k_full(ks), 64 * blk, krow,
                      h, bk);
        const int vs = it % C::kVStages, vr = it / C::kVStages;
        if (vr > 0 && !mbar_wait(v_empty(vs), (vr - 1) & 1, abort_flag, args.status, kSiteLoad)) {
          issued = 2 * it + 1;
          break;
        }
        mbar_expect_tx(v_full(vs), C::kTileBytes);
        for (int blk = 0; blk < C::kBlocks; ++blk)
          tma_load_4d(sV + vs * C::kTileBytes + blk * 16384, &args.tv, v_full(vs), 64 * blk, krow,
                      h, bk);
        issued = 2 * it + 2;
      }
      if (*abort_flag) {
        // Drain: wait (bounded) for every copy still in flight.
        const int nk = (issued + 1) / 2, nv = issued / 2;
        for (int it = max(0, nk - C::kKStages); it < nk; ++it)
          mbar_wait(k_full(it % C::kKStages), (it / C::kKStages) & 1, abort_flag, args.status,
                    kSiteTeardown);
        for (int it = max(0, nv - C::kVStages); it < nv; ++it)
          mbar_wait(v_full(it % C::kVStages), (it / C::kVStages) & 1, abort_flag, args.status,
                    kSiteTeardown);
      }
    }
  } else if (warp == C::kMmaWarp) {
    // ===================== MMA issuer =====================
    // Shared-memory descriptors are built once per tile and advanced by adding
    // (byte offset >> 4) to their start-address field, so issuing an MMA
    // costs a 64-bit add, not a rebuilt descriptor.
    if (lane == 0) {
      const uint32_t idesc_s = make_idesc(BF16, 128, 128, false, false, args.negate != 0);
      const uint32_t idesc_o = make_idesc(BF16, 128, args.D, false, true);
      // descriptor words: hi is fixed per layout, lo carries the start address
      const uint32_t kHiK = (uint32_t)(make_sdesc(0, 16, 1024) >> 32);
      const uint32_t kHiV = (uint32_t)(make_sdesc(0, 16384, 1024) >> 32);
      const uint32_t dQ = (uint32_t)make_sdesc(sQ, 16, 1024), dK = (uint32_t)make_sdesc(sK, 16, 1024);
      const uint32_t dV = (uint32_t)make_sdesc(sV, 16384, 1024);
      constexpr uint32_t kTile16 = C::kTileBytes >> 4;
      bool ok = true;
      for (int t = 0; t < NQ && ok; ++t)
        ok = mbar_wait(q_full(t), 0, abort_flag, args.status, kSiteMma);
      // O_t (+)= P_t V: P from TMEM (16 columns of 32 bits per 16 keys... 8
      // columns per K step of 16 keys), V MN-major, next 16 keys = +2048 bytes.
      // The issue loop is instantiated twice, with the V padding clears (K
      // side padded) and without them, so other calls run code that carries
      // no trace of the clears.
      auto issue_all = [&](auto padding) {
        // Padded batches: rows of a V tile past seqlen_k hold the caller's
        // padding, not TMA zero fill; P is 0 there, but 0 * NaN is not, so the
        // rows are zeroed before the tensor cores read the tile.
        auto clear_v_padding = [&](int it_v) {
          if constexpr (decltype(padding)::value) {
            const int r0 = sk - (nb + it_v) * 128;
            if (r0 < 128) {
              zero_tile_rows(sV + (it_v % C::kVStages) * C::kTileBytes, r0, C::kBlocks);
              fence_proxy_async_smem();
            }
          } else {
            (void)it_v;
          }
        };
        auto issue_pv = [=](int t, int it_prev) {
          fwd_issue_pv(tmem + C::kColO + DPAD * t, tmem + 128 * t,
                       dV + (uint32_t)(it_prev % C::kVStages) * kTile16, kHiV, idesc_o, it_prev > 0);
          tc_commit(bar0 + 8 * (bs + 2 * NQ + t));  // o_done(t)
        };
        // S_t = Q_t K^T: both K-major; 16-column K steps are +32 bytes inside a
        // 64-column block, blocks 16 KiB apart.  Padded head-dim columns are
        // zero in both operands (TMA fill), so all DPAD/16 steps are issued.
        auto issue_s = [=](int t, int ks) {
          fwd_issue_s<DPAD / 16>(tmem + 128 * t, dQ + (uint32_t)t * kTile16,
                                 dK + (uint32_t)ks * kTile16, kHiK, idesc_s);
          tc_commit(bar0 + 8 * (bs + t));  // s_full(t)
        };
        for (int it = 0; it < n_tiles && ok; ++it) {
          const int ks = it % C::kKStages;
          if (!(ok = mbar_wait(k_full(ks), (it / C::kKStages) & 1, abort_flag, args.status, kSiteMma)))
            break;
          for (int t = 0; t < NQ && ok; ++t) {
            if (it > 0) {
              if (!(ok = mbar_wait(p_ready(t), (it - 1) & 1, abort_flag, args.status, kSiteMma))) break;
              if (t == 0) {
                const int vs = (it - 1) % C::kVStages;
                if (!(ok = mbar_wait(v_full(vs), ((it - 1) / C::kVStages) & 1, abort_flag,
                                     args.status, kSiteMma)))
                  break;
                clear_v_padding(it - 1);
              }
              tc_fence_after();
              issue_pv(t, it - 1);
              if (t == NQ - 1) tc_commit(v_empty((it - 1) % C::kVStages));
            }
            issue_s(t, ks);
          }
          if (!ok) break;
          tc_commit(k_empty(ks));
        }
        if (ok) {
          const int last = n_tiles - 1;
          for (int t = 0; t < NQ && ok; ++t) {
            if (!(ok = mbar_wait(p_ready(t), last & 1, abort_flag, args.status, kSiteMma))) break;
            if (t == 0) {
              const int vs = last % C::kVStages;
              if (!(ok = mbar_wait(v_full(vs), (last / C::kVStages) & 1, abort_flag, args.status,
                                   kSiteMma)))
                break;
              clear_v_padding(last);
            }
            tc_fence_after();
            issue_pv(t, last);
          }
        }
      };
      if (args.k_padded)
        issue_all(Flag<true>{});
      else
        issue_all(Flag<false>{});
      // Everything issued has completed before TMEM is released.
      tc_commit(mma_done);
      mbar_wait(mma_done, 0, abort_flag, args.status, kSiteTeardown);
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::kHighRegs));
    // ===================== softmax / correction / epilogue =====================
    const int t = warp / 4;               // query tile of this warp group
    const int quad = warp % 4;            // TMEM lane quadrant
    const int r = quad * 32 + lane;       // row within the tile
    const int32_t i = m0 + 128 * t + r;   // sequence-local query row
    const int32_t lo = row_lo(win, i), hi = row_hi(win, i, sk);
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off + 128 * t;
    const uint32_t tO = tmem + lane_off + C::kColO + DPAD * t;
    const float sl2 = args.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int it = 0; it < n_tiles; ++it) {
      ok = mbar_wait(s_full(t), it & 1, abort_flag, args.status, kSiteSoftmax);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      // The whole score row in one TMEM load.
      uint32_t raw[128];
      tmem_ld128(tS, raw);
      float s[128];
#pragma unroll
      for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(raw[c]);
      const int32_t n0 = (nb + it) * 128;
      const bool full = tile_is_full(win, sq, sk, m0 + 128 * t, n0);
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
      const float m_tile = (mx == -INFINITY) ? -INFINITY : mx * sl2;
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
      const float rowsum = (la + lb) + (lc + ld);
      l = alpha * l + rowsum;
      if (it > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        // O_t must hold PV of the previous tile before it is rescaled.
        ok = mbar_wait(o_done(t), (it - 1) & 1, abort_flag, args.status, kSiteSoftmax);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        for (int c = 0; c < args.D / 16; ++c) {
          uint32_t raw[16];
          tmem_ld16(tO + 16 * c, raw);
#pragma unroll
          for (int e = 0; e < 16; ++e) raw[e] = __float_as_uint(__uint_as_float(raw[e]) * alpha);
          tmem_st16(tO + 16 * c, raw);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_ready(t));
    }
    if (ok) {
      ok = mbar_wait(o_done(t), (n_tiles - 1) & 1, abort_flag, args.status, kSiteEpilogue);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const bool valid = i < sq;
      uint8_t* orow = valid ? o_row_ptr(i) : nullptr;
      for (int c = 0; c < args.D / 16; ++c) {
        uint32_t raw[16];
        tmem_ld16(tO + 16 * c, raw);
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          pk[e] = pack2<BF16>(__uint_as_float(raw[2 * e]) * inv, __uint_as_float(raw[2 * e + 1]) * inv);
        if (valid) {
          st_global_v4(orow + 32 * c, pk[0], pk[1], pk[2], pk[3]);
          st_global_v4(orow + 32 * c + 16, pk[4], pk[5], pk[6], pk[7]);
        }
      }
      if (valid && args.lse)
        *lse_ptr(i) = l > 0.f ? (m_used + __log2f(l)) * 0.69314718055994531f : -INFINITY;
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

template <int NQ, int DPAD, bool BF16>
static cudaError_t launch(const FwdArgs& args, int n_mblocks, cudaStream_t stream) {
  using C = FwdCfg<NQ, DPAD>;
  static_assert(C::kSmemBytes <= 232448, "shared memory budget");
  static_assert(NQ * 128 * C::kHighRegs + 128 * C::kLowRegs <= C::kThreads * C::kLaunchRegs,
                "register split exceeds the launch budget");
  auto kern = attn_fwd_kernel<NQ, DPAD, BF16>;
  // The setmaxnreg split assumes every thread starts with kLaunchRegs
  // registers; with fewer, the raising warpgroups would wait forever, so
  // refuse to launch instead.
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs < C::kLaunchRegs) return cudaErrorLaunchOutOfResources;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(n_mblocks, args.H, args.B);
  kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(args);
  return cudaGetLastError();
}

cudaError_t launch_fwd(const FwdArgs& args, cudaStream_t stream) {
  constexpr int NQ = 2;
  const int rows = 128 * NQ;
  const int n_mblocks = (args.Sq + rows - 1) / rows;
  if (n_mblocks == 0 || args.H == 0 || args.B == 0) return cudaSuccess;
  const bool bf16 = args.bf16 != 0;
  if (args.D <= 64)
    return bf16 ? launch<NQ, 64, true>(args, n_mblocks, stream)
                : launch<NQ, 64, false>(args, n_mblocks, stream);
  return bf16 ? launch<NQ, 128, true>(args, n_mblocks, stream)
              : launch<NQ, 128, false>(args, n_mblocks, stream);
}

}  // namespace attn
