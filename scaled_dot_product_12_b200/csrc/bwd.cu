// FlashAttention backward for sm_100a: gradient of <dO, O> for the masked
// softmax attention the forward computes.
//
// Three launches on the caller's stream:
//  1. attn_bwd_pre_kernel   delta = rowsum(dO o O) in fp32 (the 0.14b release
//                           notes, "Minor Changes", name this step
//                           bwd_preprocess, with varlen folded in) and a
//                           cleared fp32 dQ accumulator;
//  2. attn_bwd_kernel       one CTA per (128-key tile, head, sequence); it
//                           keeps K, V and the dK, dV accumulators on chip and
//                           walks the 128-query tiles whose window reaches its
//                           keys: S^T = K Q^T and dP^T = V dO^T, each with one
//                           extra K step that subtracts the per-query
//                           LSE*log2(e)/c resp. delta inside the product, P^T
//                           and dS^T = P^T o (dP^T - delta) in TMEM,
//                           dV += P^T dO, dK += dS^T Q, and the dQ tile added
//                           into the fp32 accumulator by TMA bulk reductions.
//                           dO has strides of its own (the 0.14b notes,
//                           "Kernel Bug Fixes", record a kernel that addressed
//                           dO with O's strides);
//  3. attn_dq_convert_kernel  dQ = sm_scale * accumulator in the input dtype.
// Warp roles of (2): warps 0-7 P / dS in two groups of query columns (one key
// row per thread) and the dK / dV epilogue, warps 8-11 dQ drain, warp 12 TMA,
// warp 13 MMA, warps 14-15 idle (they complete the TMA/MMA warpgroup, whose
// registers go to the others through setmaxnreg).
#include <cuda_runtime.h>

#include <type_traits>

#include "common.cuh"
#include "fwd.h"
#include "mask.cuh"

namespace attn {

// ---------------------------------------------------------------------------
// 1. preprocess: TPR threads per (head, row) -- 8 when the head dims are at
// most 64, else 16 -- each one 16-byte chunk of O and dO and 32 bytes of the
// accumulator.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int64_t row_offset(const int64_t* st, int64_t row, int h, int Sq,
                                              bool packed) {
  if (packed) return row * st[2] + (int64_t)h * st[1];
  const int64_t b = row / Sq, s = row % Sq;
  return b * st[0] + (int64_t)h * st[1] + s * st[2];
}

template <bool BF16, int TPR>
__global__ void __launch_bounds__(256) attn_bwd_pre_kernel(const __grid_constant__ BwdArgs a) {
  constexpr int kGroups = 256 / TPR;  // (head, row) groups per block and pass
  const int64_t n_groups = (int64_t)a.H * a.rows;
  const int sub = threadIdx.x & (TPR - 1);
  const int chunks = (a.Dv + 7) / 8;  // of O and dO, 8 columns each; the last may be partial
  for (int64_t g = (int64_t)blockIdx.x * kGroups + threadIdx.x / TPR; g < n_groups;
       g += (int64_t)gridDim.x * kGroups) {
    const int h = (int)(g / a.rows);
    const int64_t row = g % a.rows;
    float acc = 0.f;
    if (sub < chunks) {
      const uint16_t* orow = reinterpret_cast<const uint16_t*>(a.o) +
                             row_offset(a.o_stride, row, h, a.Sq, a.q_packed) + 8 * sub;
      const uint16_t* drow = reinterpret_cast<const uint16_t*>(a.dout) +
                             row_offset(a.do_stride, row, h, a.Sq, a.q_packed) + 8 * sub;
      uint32_t ow[4], dw[4];
      if (8 * sub + 8 <= a.Dv) {
        const uint4 ov = *reinterpret_cast<const uint4*>(orow);
        const uint4 dv = *reinterpret_cast<const uint4*>(drow);
        ow[0] = ov.x, ow[1] = ov.y, ow[2] = ov.z, ow[3] = ov.w;
        dw[0] = dv.x, dw[1] = dv.y, dw[2] = dv.z, dw[3] = dv.w;
      } else {  // columns past Dv are not read
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c0 = 8 * sub + 2 * e;
          const uint32_t o0 = c0 < a.Dv ? orow[2 * e] : 0u, o1 = c0 + 1 < a.Dv ? orow[2 * e + 1] : 0u;
          const uint32_t d0 = c0 < a.Dv ? drow[2 * e] : 0u, d1 = c0 + 1 < a.Dv ? drow[2 * e + 1] : 0u;
          ow[e] = o0 | (o1 << 16);
          dw[e] = d0 | (d1 << 16);
        }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 x = unpack2<BF16>(ow[e]), y = unpack2<BF16>(dw[e]);
        acc = fmaf(x.x, y.x, acc);
        acc = fmaf(x.y, y.y, acc);
      }
    }
    if (sub < a.DA / 8) {
      float4* z = reinterpret_cast<float4*>(a.dq_acc + g * a.DA + 8 * sub);
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (a.order && sub == 0) reinterpret_cast<int4*>(a.order)[g] = make_int4(0, 0, 0, 0);
    }
#pragma unroll
    for (int m = TPR / 2; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
    if (sub == 0) a.delta[g] = acc;
  }
}

// Eight fp32 values (u, v) times s as 16-bit values at dst, only the first
// `ncols` of them (dst is 16-byte aligned when ncols >= 8).
template <bool BF16>
__device__ __forceinline__ void store_chunk8(uint8_t* dst, float4 u, float4 v, float s, int ncols) {
  const uint32_t w[4] = {pack2<BF16>(u.x * s, u.y * s), pack2<BF16>(u.z * s, u.w * s),
                         pack2<BF16>(v.x * s, v.y * s), pack2<BF16>(v.z * s, v.w * s)};
  if (ncols >= 8) {
    st_global_v4(dst, w[0], w[1], w[2], w[3]);
    return;
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    if (2 * e + 1 < ncols)
      *reinterpret_cast<uint32_t*>(dst + 4 * e) = w[e];
    else if (2 * e < ncols)
      *reinterpret_cast<uint16_t*>(dst + 4 * e) = (uint16_t)(w[e] & 0xFFFFu);
  }
}

// ---------------------------------------------------------------------------
// 3. dQ conversion.
// ---------------------------------------------------------------------------
template <bool BF16>
__global__ void __launch_bounds__(256) attn_dq_convert_kernel(const __grid_constant__ BwdArgs a) {
  const int chunks = (a.D + 7) / 8;
  const int64_t n = (int64_t)a.H * a.rows * chunks;
  for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < n;
       x += (int64_t)gridDim.x * blockDim.x) {
    const int64_t g = x / chunks;
    const int c = (int)(x % chunks);
    const int h = (int)(g / a.rows);
    const int64_t row = g % a.rows;
    if (a.q_padded) {  // rows past a batch's seqlen_q are padding: not written
      const int32_t len = min(max(a.cu_q[row / a.Sq], 0), a.Sq);
      if (row % a.Sq >= len) continue;
    }
    const float4* src = reinterpret_cast<const float4*>(a.dq_acc + g * a.DA + 8 * c);
    const float4 u = src[0], v = src[1];
    const float s = a.sm_scale;
    uint8_t* dst = reinterpret_cast<uint8_t*>(a.dq) +
                   2 * (row_offset(a.dq_stride, row, h, a.Sq, a.q_packed) + 8 * c);
    store_chunk8<BF16>(dst, u, v, s, a.D - 8 * c);
  }
}

// The same for a stacked Q side whose sequences may leave rows unused
// (lengths from seqused, positions from an array): block row b of the grid
// converts sequence b's used rows only, so rows outside every sequence are
// not written.
template <bool BF16>
__global__ void __launch_bounds__(256) attn_dq_convert_seq_kernel(const __grid_constant__ BwdArgs a) {
  const int b = blockIdx.x;
  int32_t row0, len;
  stacked_bounds(a.cu_q, a.q_used ? a.used_q : nullptr, a.q_offsets != 0, b, a.total_q, &row0,
                 &len);
  const int chunks = (a.D + 7) / 8;
  const int64_t n = (int64_t)a.H * len * chunks;
  for (int64_t x = (int64_t)blockIdx.y * blockDim.x + threadIdx.x; x < n;
       x += (int64_t)gridDim.y * blockDim.x) {
    const int c = (int)(x % chunks);
    const int64_t hr = x / chunks;
    const int h = (int)(hr / len);
    const int64_t row = row0 + hr % len;
    const int64_t g = (int64_t)h * a.rows + row;
    const float4* src = reinterpret_cast<const float4*>(a.dq_acc + g * a.DA + 8 * c);
    const float4 u = src[0], v = src[1];
    const float s = a.sm_scale;
    uint8_t* dst = reinterpret_cast<uint8_t*>(a.dq) +
                   2 * (row_offset(a.dq_stride, row, h, a.Sq, true) + 8 * c);
    store_chunk8<BF16>(dst, u, v, s, a.D - 8 * c);
  }
}

// ---------------------------------------------------------------------------
// 2. main backward
// ---------------------------------------------------------------------------
template <int DPAD, bool BIAS = false>
struct BwdCfg {
  // Warps 0-7: two P/dS groups (query columns 0-63 and 64-127 of every key
  // row); 8-11: dQ drain; 12: TMA; 13: MMA; 14-15 idle.  16 warps, four per
  // sub-partition, launch with 128 registers per thread; the TMA/MMA
  // warpgroup then gives registers to the P/dS and drain warpgroups
  // (setmaxnreg), so the drain can hold a whole 128-column dQ tile and
  // release its TMEM columns right after reading them.
  static constexpr int kThreads = 512;
  static constexpr int kLaunchRegs = 128;
  static constexpr int kProducerRegs = 96;
  static constexpr int kDrainRegs = 144;
  static constexpr int kPdsRegs = 136;
  static constexpr int kLoadWarp = 12;
  static constexpr int kMmaWarp = 13;
  static constexpr int kBlocks = DPAD / 64;
  static constexpr int kTileBytes = 128 * DPAD * 2;
  static constexpr int kQStages = 2;
  // The dQ tile is staged in shared memory for TMA bulk reductions (4 warps x
  // kDqBufs buffers x 32x32 fp32); at head dim 128 dO gets one ring stage and
  // each drain warp one staging buffer, to make room.
  static constexpr bool kStageDq = true;
  static constexpr int kDOStages = (DPAD == 128) ? 1 : 2;
  static constexpr int kDqBufs = (DPAD == 128) ? 1 : 2;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kTileBytes;
  static constexpr int kOffQ = kOffV + kTileBytes;
  static constexpr int kOffDO = kOffQ + kQStages * kTileBytes;
  static constexpr int kOffDS = kOffDO + kDOStages * kTileBytes;  // 128 x 128 16-bit
  static constexpr int kOffDQ = kOffDS + 128 * 128 * 2;
  static constexpr int kDqStageBytes = kStageDq ? 4 * kDqBufs * 32 * 32 * 4 : 0;
  // Operands of one extra 16-wide K step appended to the S^T and dP^T
  // products, which subtracts the per-query constants inside the MMA (no-
  // swizzle K-major, 128 rows x 16 bf16 = 4 KiB each): [0] ones on the key
  // side, [1] -LSE/c terms of the next S^T tile, [2] -delta terms of the next
  // dP^T tile, on the query side.
  static constexpr int kXBytes = 128 * 16 * 2;
  static constexpr int kOffX = kOffDQ + kDqStageBytes;
  // With a bias at head dim 64, the bias tile of the current query tile
  // (128 queries x 128 keys, 16-bit, two 128-byte swizzled 64-key blocks) is
  // staged by TMA; at 128 there is no room and the P / dS warps load it.
  static constexpr bool kStageBias = BIAS && DPAD == 64;
  static constexpr int kBiasTileBytes = kStageBias ? 128 * 128 * 2 : 0;
  static constexpr int kOffBias = kOffX + 3 * kXBytes;
  static constexpr int kOffBar = kOffBias + kBiasTileBytes;
  // kv_full, q_full[QS], q_empty[QS], do_full[DS], do_empty[DS], s_full,
  // dp_full, p_ready, ds_ready, dq_mma, dq_free, acc_done, x_ready,
  // delta_ready[2], b_full, b_empty
  static constexpr int kNumBars = 1 + 2 * kQStages + 2 * kDOStages + 12;
  // With dropout, delta is not folded into dP^T: each P/dS group stages the
  // delta values of its 64 query columns, two tiles deep.
  static constexpr int kOffDelta = kOffBar + 8 * kNumBars;
  static constexpr int kOffMisc = kOffDelta + 2 * 2 * 64 * 4;
  static constexpr int kSmemBytes = kOffMisc + 16;
  static constexpr int kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + DPAD;
  static constexpr bool kAliasDQ = (DPAD == 128);  // dQ tile reuses the dP^T columns
  static constexpr int kColDQ = kAliasDQ ? kColDP : 256 + 2 * DPAD;
  static constexpr bool kDqTransposed = (DPAD == 128);  // dQ^T = K^T dS^T, lane = head dim
  static constexpr int kTmemCols = 512;
};

// D = A B^T with both operands K-major (A: 128 rows, B: 128 rows, K = head
// dim): 16-column K steps are +32 bytes inside a 64-column block, blocks
// 16 KiB apart; padded head-dim columns are zero in both operands.
template <int KSTEPS>
__device__ __forceinline__ void bwd_issue_kmajor(uint32_t d, uint32_t a_lo, uint32_t b_lo,
                                                 uint32_t hi, uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < KSTEPS; ++kk) {
    const uint32_t o = (uint32_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
    mma_ss2(d, a_lo + o, hi, b_lo + o, hi, idesc, kk > 0 ? 1u : 0u);
  }
}
// D (+)= A(TMEM, 128 lanes x 128 K as 16-bit pairs) B(MN-major smem), K = 128.
__device__ __forceinline__ void bwd_issue_ts(uint32_t d, uint32_t a, uint32_t b_lo, uint32_t hi,
                                             uint32_t idesc, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    mma_ts2(d, a + 8 * kk, b_lo + (uint32_t)(kk * 2048 >> 4), hi, idesc,
            (accumulate || kk > 0) ? 1u : 0u);
}
// Same with A split in two: queries 0-63 at columns [a, a+32), queries
// 64-127 at [a+64, a+96) (each P/dS group writes inside its own columns).
__device__ __forceinline__ void bwd_issue_ts_halves(uint32_t d, uint32_t a, uint32_t b_lo,
                                                    uint32_t hi, uint32_t idesc, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    mma_ts2(d, a + 8 * kk + (kk >= 4 ? 32 : 0), b_lo + (uint32_t)(kk * 2048 >> 4), hi, idesc,
            (accumulate || kk > 0) ? 1u : 0u);
}
// D = A B with both operands MN-major in smem, K = 128 (16 rows = 2048 bytes).
__device__ __forceinline__ void bwd_issue_mn(uint32_t d, uint32_t a_lo, uint32_t b_lo, uint32_t hi,
                                             uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t o = (uint32_t)(kk * 2048 >> 4);
    mma_ss2(d, a_lo + o, hi, b_lo + o, hi, idesc, kk > 0 ? 1u : 0u);
  }
}

template <int DPAD, bool BF16, bool DROPOUT, bool BIAS>
__global__ void __launch_bounds__(512, 1) attn_bwd_kernel(const __grid_constant__ BwdArgs a) {
  using C = BwdCfg<DPAD, BIAS>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int ntile = blockIdx.x;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  // Q and K sides are addressed independently (see the forward kernel).
  int32_t sq = a.Sq, sk = a.Sk, qrow0 = 0, krow0 = 0, bq = b, bk = b;
  if (a.q_packed) {
    stacked_bounds(a.cu_q, a.q_used ? a.used_q : nullptr, a.q_offsets != 0, b, a.total_q, &qrow0, &sq);
    bq = 0;
  } else if (a.q_padded) {
    sq = min(max(a.cu_q[b], 0), a.Sq);
  }
  if (a.k_packed) {
    stacked_bounds(a.cu_k, a.k_used ? a.used_k : nullptr, a.k_offsets != 0, b, a.total_k, &krow0, &sk);
    bk = 0;
  } else if (a.k_padded) {
    sk = min(max(a.cu_k[b], 0), a.Sk);
  }
  const int32_t n0 = ntile * 128;
  if (n0 >= sk) return;
  if (sbase & 1023) {  // the swizzled tiles need 1 KiB alignment
    if (threadIdx.x == 0) atomicOr(a.status, 1u << kSiteTeardown);
    return;
  }
  const SeqWindow win = seq_window(a.wl, a.wr, a.bottom_right != 0, sq, sk);
  int32_t mb, me;
  bwd_tile_range(win, sq, sk, n0, &mb, &me);
  const int n_it = me - mb;

  auto kv_row_ptr = [&](void* base, const int64_t* st, int32_t j) -> uint8_t* {
    int64_t off = a.k_packed ? (int64_t)(krow0 + j) * st[2]
                           : (int64_t)b * st[0] + (int64_t)j * st[2];
    off += (int64_t)h * st[1];
    return reinterpret_cast<uint8_t*>(base) + 2 * off;
  };

  // dbias rows [r_begin, r_end) of this key tile's columns (those below
  // seqlen_k) set to 0: the query rows no visited query tile holds, whose
  // pairs with these keys are all masked.  Threads t of nt share the rows,
  // 16 per row.
  auto zero_dbias_rows = [&](int32_t r_begin, int32_t r_end, int t, int nt) {
    if constexpr (BIAS) {
      if (!a.dbias) return;
      // (never past the bias tensor's Sq x Sk, whatever the sequence lengths)
      const int ncols = min(128, min(sk, a.Sk) - n0);
      r_end = min(r_end, a.Sq);
      uint16_t* base = reinterpret_cast<uint16_t*>(a.dbias) + (int64_t)b * a.dbias_stride[0] +
                       (int64_t)h * a.dbias_stride[1] + n0;
      for (int64_t x = t; x < (int64_t)(r_end - r_begin) * 16; x += nt) {
        const int32_t i = r_begin + (int32_t)(x >> 4);
        const int c = (int)(x & 15);
        if (8 * c >= ncols) continue;
        uint16_t* p = base + (int64_t)i * a.dbias_stride[2] + 8 * c;
        if (8 * c + 8 <= ncols) {
          st_global_v4(p, 0u, 0u, 0u, 0u);
        } else {
          for (int e = 0; e < ncols - 8 * c; ++e) p[e] = 0;
        }
      }
    } else {
      (void)r_begin, (void)r_end, (void)t, (void)nt;
    }
  };

  if (n_it <= 0) {
    // No query sees these keys: dK = dV = 0 (and dbias = 0 in their columns).
    const int rows = min(128, sk - n0);
    for (int r = threadIdx.x / 4; r < rows; r += blockDim.x / 4) {
      zero_row16(kv_row_ptr(a.dk, a.dk_stride, n0 + r), a.D, threadIdx.x & 3, 4);
      zero_row16(kv_row_ptr(a.dv, a.dv_stride, n0 + r), a.Dv, threadIdx.x & 3, 4);
    }
    zero_dbias_rows(0, sq, threadIdx.x, blockDim.x);
    return;
  }

  const uint32_t sK = sbase + C::kOffK, sV = sbase + C::kOffV, sQ = sbase + C::kOffQ,
                 sDO = sbase + C::kOffDO, sDS = sbase + C::kOffDS, sDQ = sbase + C::kOffDQ;
  const uint32_t sXA = sbase + C::kOffX, sXQ = sXA + C::kXBytes, sXD = sXA + 2 * C::kXBytes;
  const uint32_t bar0 = sbase + C::kOffBar;
  const uint32_t kv_full = bar0;
  auto q_full = [&](int s) { return bar0 + 8 * (1 + s); };
  auto q_empty = [&](int s) { return bar0 + 8 * (1 + C::kQStages + s); };
  auto do_full = [&](int s) { return bar0 + 8 * (1 + 2 * C::kQStages + s); };
  auto do_empty = [&](int s) { return bar0 + 8 * (1 + 2 * C::kQStages + C::kDOStages + s); };
  const uint32_t s_full = bar0 + 8 * (1 + 2 * C::kQStages + 2 * C::kDOStages);
  const uint32_t dp_full = s_full + 8, p_ready = s_full + 16, ds_ready = s_full + 24,
                 dq_mma = s_full + 32, dq_free = s_full + 40, acc_done = s_full + 48,
                 x_ready = s_full + 56;
  auto delta_ready = [&](int g) { return s_full + 64 + 8 * g; };
  const uint32_t b_full = s_full + 80, b_empty = s_full + 88;  // staged bias tile
  const uint32_t sBias = sbase + C::kOffBias;
  (void)b_full, (void)b_empty, (void)sBias;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < C::kQStages; ++s) {
      mbar_init(q_full(s), 1);
      mbar_init(q_empty(s), 1);
    }
    for (int s = 0; s < C::kDOStages; ++s) {
      mbar_init(do_full(s), 1);
      mbar_init(do_empty(s), 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_ready, 8);  // one arrival per P/dS warp
    mbar_init(ds_ready, 8);
    mbar_init(dq_mma, 1);
    mbar_init(dq_free, 4);  // one per drain warp
    mbar_init(acc_done, 1);
    mbar_init(x_ready, 8);
    mbar_init(delta_ready(0), 4);  // one per warp of the group
    mbar_init(delta_ready(1), 4);
    mbar_init(b_full, 1);
    mbar_init(b_empty, 8);  // one per P / dS warp
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

  if (warp >= 12) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::kProducerRegs));
  if (warp == C::kLoadWarp) {
    // ===================== TMA producer =====================
    if (lane == 0) {
      prefetch_tmap(&a.tq);
      prefetch_tmap(&a.tk);
      prefetch_tmap(&a.tv);
      prefetch_tmap(&a.tdo);
      mbar_expect_tx(kv_full, 2 * C::kTileBytes);
      for (int blk = 0; blk < C::kBlocks; ++blk) {
        tma_load_4d(sK + blk * 16384, &a.tk, kv_full, 64 * blk, krow0 + n0, h, bk);
        tma_load_4d(sV + blk * 16384, &a.tv, kv_full, 64 * blk, krow0 + n0, h, bk);
      }
      int nq = 0, ndo = 0;
      for (int it = 0; it < n_it; ++it) {
        const int qs = it % C::kQStages, round = it / C::kQStages;
        const int qrow = qrow0 + (mb + it) * 128;
        if (round > 0 && !mbar_wait(q_empty(qs), (round - 1) & 1, abort_flag, a.status, kSiteLoad))
          break;
        mbar_expect_tx(q_full(qs), C::kTileBytes);
        for (int blk = 0; blk < C::kBlocks; ++blk)
          tma_load_4d(sQ + qs * C::kTileBytes + blk * 16384, &a.tq, q_full(qs), 64 * blk, qrow, h,
                      bq);
        ++nq;
        const int ds = it % C::kDOStages, dround = it / C::kDOStages;
        if (dround > 0 &&
            !mbar_wait(do_empty(ds), (dround - 1) & 1, abort_flag, a.status, kSiteLoad))
          break;
        mbar_expect_tx(do_full(ds), C::kTileBytes);
        for (int blk = 0; blk < C::kBlocks; ++blk)
          tma_load_4d(sDO + ds * C::kTileBytes + blk * 16384, &a.tdo, do_full(ds), 64 * blk, qrow,
                      h, bq);
        ++ndo;
      }
      if (*abort_flag) {
        mbar_drain(kv_full, 0, a.status);
        for (int it = max(0, nq - C::kQStages); it < nq; ++it)
          mbar_drain(q_full(it % C::kQStages), (it / C::kQStages) & 1, a.status);
        for (int it = max(0, ndo - C::kDOStages); it < ndo; ++it)
          mbar_drain(do_full(it % C::kDOStages), (it / C::kDOStages) & 1, a.status);
      }
    }
  } else if (warp == C::kMmaWarp) {
    // ===================== MMA issuer =====================
    // Order per query tile `it`:  dV(it), S(it+1), dK(it), dQ(it), dP(it+1).
    // S(it+1) reuses the S/P columns as soon as dV(it) has read P(it); the
    // P / dS warps work on tile it+1's P while dK(it) and dQ(it) run.
    if (lane == 0) {
      const uint32_t idesc_kk = make_idesc(BF16, 128, 128, false, false);   // S^T, dP^T
      const uint32_t idesc_dv = make_idesc(BF16, 128, a.Dv16, false, true);  // dV (A in TMEM)
      const uint32_t idesc_dk = make_idesc(BF16, 128, a.D16, false, true);   // dK (A in TMEM)
      // dQ: with a 128-wide head dim the transposed product dQ^T = K^T dS^T
      // (TMEM lane = head-dim index, column = query) lets the drain add whole
      // 128-byte rows; otherwise dQ = dS K (lane = query).
      const uint32_t idesc_dq = C::kDqTransposed ? make_idesc(BF16, 128, 128, true, true)
                                                 : make_idesc(BF16, 128, a.D16, true, true);
      // Descriptor words: the high word is fixed per layout; the low word
      // carries the start address and is advanced by (bytes >> 4).
      const uint32_t hiK = (uint32_t)(make_sdesc(0, 16, 1024) >> 32);    // K-major
      const uint32_t hiM = (uint32_t)(make_sdesc(0, 16384, 1024) >> 32); // MN-major
      const uint32_t loK = (uint32_t)make_sdesc(sK, 16, 1024), loV = (uint32_t)make_sdesc(sV, 16, 1024);
      const uint32_t loQ = (uint32_t)make_sdesc(sQ, 16, 1024), loDO = (uint32_t)make_sdesc(sDO, 16, 1024);
      const uint32_t loKm = (uint32_t)make_sdesc(sK, 16384, 1024);
      const uint32_t loQm = (uint32_t)make_sdesc(sQ, 16384, 1024);
      const uint32_t loDOm = (uint32_t)make_sdesc(sDO, 16384, 1024);
      const uint32_t loDSm = (uint32_t)make_sdesc(sDS, 16384, 1024);
      constexpr uint32_t kTile16 = C::kTileBytes >> 4;
      // The extra K step: always bf16 operands (a separate instruction, so
      // independent of the inputs' type), accumulating into the same tile.
      const uint32_t idesc_x = make_idesc(true, 128, 128, false, false);
      const uint64_t dXA = make_sdesc_plain(sXA, 128, 256), dXQ = make_sdesc_plain(sXQ, 128, 256),
                     dXD = make_sdesc_plain(sXD, 128, 256);
      // The issue loop is instantiated twice, with the padding clears (some
      // side leaves rows unused: padded, or stacked with used lengths) and
      // without them, so dense and packed calls run code that carries no
      // trace of the clears.
      auto issue_all = [&](auto padding) {
        // Tile rows past seqlen_q / seqlen_k may hold the caller's padding (a
        // padded batch, the unused rows of a slot, a gap between stacked
        // sequences), not TMA zero fill; P and dS are 0 there, but 0 * NaN is
        // not, so those rows are zeroed before the tensor cores first read a
        // tile.
        auto clear_padding = [&](bool side_padded, uint32_t tile, int r0) {
          if constexpr (decltype(padding)::value) {
            if (side_padded && r0 < 128) {
              zero_tile_rows(tile, r0, C::kBlocks);
              fence_proxy_async_smem();
            }
          } else {
            (void)side_padded, (void)tile, (void)r0;
          }
        };
        bool ok = mbar_wait(kv_full, 0, abort_flag, a.status, kSiteMma) &&
                  mbar_wait(q_full(0), 0, abort_flag, a.status, kSiteMma) &&
                  mbar_wait(x_ready, 0, abort_flag, a.status, kSiteMma);
        if (ok) {
          clear_padding(a.k_padded || a.k_used, sK, sk - n0);
          clear_padding(a.k_padded || a.k_used, sV, sk - n0);
          clear_padding(a.q_padded || a.q_used, sQ, sq - mb * 128);
          tc_fence_after();
          bwd_issue_kmajor<DPAD / 16>(tmem + C::kColS, loK, loQ, hiK, idesc_kk);
          mma_ss(tmem + C::kColS, dXA, dXQ, idesc_x, true);
          tc_commit(s_full);
          ok = mbar_wait(do_full(0), 0, abort_flag, a.status, kSiteMma);
        }
        if (ok) {
          clear_padding(a.q_padded || a.q_used, sDO, sq - mb * 128);
          tc_fence_after();
          bwd_issue_kmajor<DPAD / 16>(tmem + C::kColDP, loV, loDO, hiK, idesc_kk);
          mma_ss(tmem + C::kColDP, dXA, dXD, idesc_x, true);
          tc_commit(dp_full);
        }
        for (int it = 0; it < n_it && ok; ++it) {
          const int qs = it % C::kQStages, dos = it % C::kDOStages;
          const int nx = it + 1, nqs = nx % C::kQStages, ndos = nx % C::kDOStages;
          const uint32_t npar = (nx / C::kQStages) & 1, ndpar = (nx / C::kDOStages) & 1;
          // dV += P^T dO  (P^T from TMEM, dO MN-major)
          if (!(ok = mbar_wait(p_ready, it & 1, abort_flag, a.status, kSiteMma))) break;
          tc_fence_after();
          bwd_issue_ts_halves(tmem + C::kColDV, tmem + C::kColS, loDOm + dos * kTile16, hiM, idesc_dv,
                              it > 0);
          tc_commit(do_empty(dos));
          if (nx < n_it) {
            if (!(ok = mbar_wait(q_full(nqs), npar, abort_flag, a.status, kSiteMma))) break;
            clear_padding(a.q_padded || a.q_used, sQ + nqs * C::kTileBytes, sq - (mb + nx) * 128);
            tc_fence_after();
            bwd_issue_kmajor<DPAD / 16>(tmem + C::kColS, loK, loQ + nqs * kTile16, hiK, idesc_kk);
            mma_ss(tmem + C::kColS, dXA, dXQ, idesc_x, true);
            tc_commit(s_full);
          }
          // dK += dS^T Q
          if (!(ok = mbar_wait(ds_ready, it & 1, abort_flag, a.status, kSiteMma))) break;
          tc_fence_after();
          bwd_issue_ts_halves(tmem + C::kColDK, tmem + C::kColDP, loQm + qs * kTile16, hiM, idesc_dk,
                              it > 0);
          tc_commit(q_empty(qs));
          // dQ tile (into the dP columns when aliased: in order after dK read them)
          if (!C::kAliasDQ && it > 0 &&
              !(ok = mbar_wait(dq_free, (it - 1) & 1, abort_flag, a.status, kSiteMma)))
            break;
          if (C::kDqTransposed)
            bwd_issue_mn(tmem + C::kColDQ, loKm, loDSm, hiM, idesc_dq);   // K^T dS^T
          else
            bwd_issue_mn(tmem + C::kColDQ, loDSm, loKm, hiM, idesc_dq);   // dS K
          tc_commit(dq_mma);
          if (nx < n_it) {
            if (!(ok = mbar_wait(do_full(ndos), ndpar, abort_flag, a.status, kSiteMma))) break;
            if (C::kAliasDQ && !(ok = mbar_wait(dq_free, it & 1, abort_flag, a.status, kSiteMma)))
              break;
            clear_padding(a.q_padded || a.q_used, sDO + ndos * C::kTileBytes, sq - (mb + nx) * 128);
            tc_fence_after();
            bwd_issue_kmajor<DPAD / 16>(tmem + C::kColDP, loV, loDO + ndos * kTile16, hiK, idesc_kk);
            mma_ss(tmem + C::kColDP, dXA, dXD, idesc_x, true);
            tc_commit(dp_full);
          }
        }
        tc_commit(acc_done);
        // every MMA issued has completed before TMEM can be released (on an
        // abort too, when the other warps skip their wait on acc_done)
        mbar_drain(acc_done, 0, a.status);
      };
      if (a.q_padded || a.k_padded || a.q_used || a.k_used)
        issue_all(Flag<true>{});
      else
        issue_all(Flag<false>{});
    }
  } else if (BIAS) {
    if (C::kStageBias && warp == 14) {
      // ===================== bias tile producer (head dim 64) =====================
      // The bias tile of each visited query tile (query rows x this CTA's
      // keys) into shared memory, refilled as soon as the P / dS warps have
      // read the previous one.
      if (lane == 0 && a.bias) {
        prefetch_tmap(&a.tb);
        const int cb = a.bias_b_bcast ? 0 : b, ch = a.bias_h_bcast ? 0 : h;
        int it = 0;
        for (; it < n_it; ++it) {
          if (it > 0 && !mbar_wait(b_empty, (uint32_t)((it - 1) & 1), abort_flag, a.status, kSiteLoad))
            break;
          mbar_expect_tx(b_full, C::kBiasTileBytes);
          for (int blk = 0; blk < 2; ++blk)
            tma_load_4d(sBias + blk * 16384, &a.tb, b_full, n0 + 64 * blk, (mb + it) * 128, ch, cb);
        }
        if (*abort_flag && it > 0) mbar_drain(b_full, (uint32_t)((it - 1) & 1), a.status);
      }
    } else {
      // dbias of the query rows outside the visited tiles
      const int t = C::kStageBias ? lane : (warp - 14) * 32 + lane;
      const int nt = C::kStageBias ? 32 : 64;
      zero_dbias_rows(0, min(mb * 128, sq), t, nt);
      zero_dbias_rows(min(me * 128, sq), sq, t, nt);
    }
  }
  } else if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::kPdsRegs));
    // ===================== P, dS and the dK / dV epilogue =====================
    // Group `half` owns query columns [64 half, 64 half + 64) of every key row.
    const int half = warp >> 2, quad = warp & 3;
    const int r = quad * 32 + lane;  // key row within the tile (TMEM lane)
    const int32_t j = n0 + r;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::kColS, tDP = tmem + lane_off + C::kColDP;
    const int qo = 64 * half;          // first query column of this group
    const uint32_t po = 64 * half;     // its P / dS columns (16-bit pairs)
    const float sl2 = a.scale_log2;  // c = sm_scale * log2(e), |c| >= 2^-100
    // Queries that see key j: j - R <= i <= j + L, 0 <= i < sq (none if j >= sk).
    int32_t qa = j - win.R, qz = j + win.L;
    if (qa < 0) qa = 0;
    if (qz > sq - 1) qz = sq - 1;
    if (j >= sk) qz = qa - 1;
    // Bias and dbias columns of key j (null past the sequence, or when not
    // given): element (i, j) at col + i * stride.
    const uint16_t* bcol = nullptr;
    const uint16_t* bwarp = nullptr;  // this warp's first key column (L2 prefetch)
    uint16_t* dbcol = nullptr;
    const int32_t sqb = min(sq, a.Sq);  // bias rows: never past the tensor's Sq
    (void)sqb, (void)bwarp;
    if constexpr (BIAS) {
      const int32_t j0 = n0 + quad * 32;
      if (a.bias && j0 < min(sk, a.Sk))
        bwarp = reinterpret_cast<const uint16_t*>(a.bias) + (int64_t)b * a.bias_stride[0] +
                (int64_t)h * a.bias_stride[1] + j0;
      if (j < sk && j < a.Sk && a.bias)
        bcol = reinterpret_cast<const uint16_t*>(a.bias) + (int64_t)b * a.bias_stride[0] +
               (int64_t)h * a.bias_stride[1] + j;
      if (j < sk && j < a.Sk && a.dbias)
        dbcol = reinterpret_cast<uint16_t*>(a.dbias) + (int64_t)b * a.dbias_stride[0] +
                (int64_t)h * a.dbias_stride[1] + j;
    }
    // Per-query values of a tile, one per thread: group 0 fetches LSE, group
    // 1 fetches delta, for query row r (0 past the sequence).
    auto row_val = [&](int it) -> float {
      const int32_t i = (mb + it) * 128 + r;
      if (i >= sq) return 0.f;
      if (half == 0) {
        int64_t li;
        if (a.q_packed)
          li = a.lse_th ? (int64_t)(qrow0 + i) * a.H + h : (int64_t)h * a.total_q + qrow0 + i;
        else
          li = a.lse_th ? ((int64_t)b * a.Sq + i) * a.H + h : ((int64_t)b * a.H + h) * a.Sq + i;
        return a.lse[li];
      }
      const int64_t row = a.q_packed ? (int64_t)(qrow0 + i) : (int64_t)b * a.Sq + i;
      return a.delta[(int64_t)h * a.rows + row];
    };
    // The per-query constants enter the products through the extra K step:
    // thread r writes query r's row of the query-side operand, the value as
    // three bf16 terms (hi + mid + lo equals the fp32 value) in columns 0-2
    // against ones in columns 0-2 of the key-side operand; columns 3-15 are 0.
    // Group 0 writes -LSE*log2(e)/c (S^T*c - LSE*log2(e) == c*(S^T - that)),
    // group 1 writes -delta.  Rows whose LSE is not finite (no allowed key)
    // get 0: their P is zero through the column mask.
    const uint32_t xrow = (uint32_t)((r >> 3) * 256 + (r & 7) * 16);  // core matrix (r/8, 0)
    const float inv_c = 1.f / sl2;
    auto folded = [&](float v) -> float {
      if (half == 1) return DROPOUT ? 0.f : -v;  // with dropout delta is applied per element
      return (v == -INFINITY || v == INFINITY || v != v) ? 0.f : -(v * 1.4426950408889634f) * inv_c;
    };
    auto put_row = [&](uint32_t base, float x) {
      const uint32_t w_hi = pack2<true>(x, 0.f);
      const float t0 = __uint_as_float(w_hi << 16);
      const float r1 = x - t0;
      const uint32_t w_mid = pack2<true>(r1, 0.f);
      const float t1 = __uint_as_float(w_mid << 16);
      const uint32_t w_lo = pack2<true>(r1 - t1, 0.f);
      asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(base + xrow),
                   "r"((w_hi & 0xFFFFu) | (w_mid << 16)), "r"(w_lo & 0xFFFFu)
                   : "memory");
    };
    // Dropout: this group's delta values for tile `it` into its staging slot
    // (threads 0-63 of the group write query columns qo .. qo + 63), then the
    // group's delta_ready barrier.  Every warp of the group arrives once per
    // tile (after all its lanes) and waits for that tile before reading, so
    // the barrier never runs two phases ahead of a reader, and a slot is
    // rewritten only two tiles later, after all of its readers have moved on.
    const uint32_t sDelta = sbase + C::kOffDelta + half * 2 * 64 * 4;
    auto stage_delta = [&](int it) {
      if constexpr (DROPOUT) {
        if (r < 64) {
          const int32_t i = (mb + it) * 128 + qo + r;
          float d = 0.f;
          if (i < sq) {
            const int64_t row = a.q_packed ? (int64_t)(qrow0 + i) : (int64_t)b * a.Sq + i;
            d = a.delta[(int64_t)h * a.rows + row];
          }
          asm volatile("st.shared.f32 [%0], %1;" ::"r"(sDelta + (it & 1) * 256 + r * 4), "f"(d)
                       : "memory");
        }
        mbar_arrive_warp(delta_ready(half));
      } else {
        (void)it;
      }
    };
    // Dropout: keep bits of this key row against the 32 query columns of
    // chunk c of tile it.  Key j, query i take word (j mod 4) of Philox on the
    // counter (j div 4, i, b H + h, offset).
    const uint32_t bh = (uint32_t)(b * a.H + h);
    auto keep_bits = [&](int it, int c) -> uint32_t {
      uint32_t bits = 0;
      if constexpr (DROPOUT) {
        const uint32_t i0 = (uint32_t)((mb + it) * 128 + qo + 32 * c);
        const int word = j & 3;
#pragma unroll 4
        for (int k = 0; k < 32; ++k) {
          const uint4 wd = philox4x32_10(make_uint4((uint32_t)(j >> 2), i0 + k, bh, a.philox_offset),
                                         a.seed_lo, a.seed_hi);
          const uint32_t x = word == 0 ? wd.x : word == 1 ? wd.y : word == 2 ? wd.z : wd.w;
          bits |= (x < a.keep_below ? 1u : 0u) << k;
        }
      } else {
        (void)it, (void)c;
      }
      return bits;
    };
    {
      // Constant parts, then tile 0's terms; the MMA issuer waits on x_ready.
      const uint32_t one2 = pack2<true>(1.f, 1.f), one_ = pack2<true>(1.f, 0.f);
      if (half == 0) {
        st_shared_v4(sXA + xrow, one2, one_, 0u, 0u);
        st_shared_v4(sXA + xrow + 128, 0u, 0u, 0u, 0u);
      }
      const uint32_t xb = half == 0 ? sXQ : sXD;
      st_shared_v4(xb + xrow, 0u, 0u, 0u, 0u);
      st_shared_v4(xb + xrow + 128, 0u, 0u, 0u, 0u);
      put_row(xb, folded(row_val(0)));
      fence_proxy_async_smem();
      mbar_arrive_warp(x_ready);
    }
    float v_next = n_it > 1 ? row_val(1) : 0.f;  // this group's value for tile it + 1
    // Bias: raw 16-bit values of key j for 16 queries from i0 (0 past the
    // sequence), two sub-chunks in flight.
    uint32_t braw[2][BIAS ? 16 : 1];
    auto load_bias16 = [&](uint32_t (&dst)[BIAS ? 16 : 1], int32_t i0) {
      if constexpr (BIAS && !C::kStageBias) {
        const uint16_t* p = bcol ? bcol + (int64_t)i0 * a.bias_stride[2] : nullptr;
#pragma unroll
        for (int k = 0; k < 16; ++k)
          dst[k] = (p && i0 + k < sqb) ? (uint32_t)__ldg(p + (int64_t)k * a.bias_stride[2]) : 0u;
      } else {
        (void)dst, (void)i0;
      }
    };
    load_bias16(braw[0], mb * 128 + qo);
    bool ok = true;
    for (int it = 0; it < n_it && ok; ++it) {
      const int32_t m0 = (mb + it) * 128;
      const bool full = tile_is_full(win, sq, sk, m0, n0);
      const int32_t ca = qa - m0, cz = qz - m0;  // allowed columns [ca, cz]
      // ---- phase 1: P^T = exp2(c * (S^T - LSE*log2(e)/c)), masked ----
      ok = mbar_wait(s_full, it & 1, abort_flag, a.status, kSiteSoftmax);
      if (C::kStageBias && ok && a.bias)
        ok = mbar_wait(b_full, it & 1, abort_flag, a.status, kSiteSoftmax);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      // P is kept as the rounded 16-bit pairs the dV product uses (with
      // dropout: the undropped P for dS, while the dV product gets the kept
      // elements only; its factor 1 / (1 - p) is applied at the store).
      uint32_t pk[32];
      uint32_t keep[2] = {0xFFFFFFFFu, 0xFFFFFFFFu};
      if constexpr (DROPOUT) stage_delta(it);
      if constexpr (BIAS && !C::kStageBias) {
        // the next tile's bias into L2: this warp's 32 key columns (64
        // bytes of a row) for the group's 64 query rows, two rows per lane
        if (bwarp && it + 1 < n_it) {
          const int32_t i1 = m0 + 128 + qo;
#pragma unroll
          for (int k = lane; k < 64; k += 32)
            if (i1 + k < sqb)
              asm volatile("prefetch.global.L2 [%0];" ::"l"(bwarp + (int64_t)(i1 + k) * a.bias_stride[2]));
        }
      }
      if constexpr (C::kStageBias) {
        // Staged bias tile: (query q of the tile, key r) at 64-key block
        // r / 64, row q, 16-byte chunk ((r % 64) / 8) xor (q % 8), 2 bytes r % 8.
        const uint32_t bcol_s = sBias + (r >> 6) * 16384 + (r & 7) * 2;
        const uint32_t bchunk = (uint32_t)((r & 63) >> 3);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if constexpr (DROPOUT) keep[c] = keep_bits(it, c);
          uint32_t sr[32];
          tmem_ld32(tS + qo + 32 * c, sr);
          uint32_t chunk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int q0 = qo + 32 * c + 2 * e, q1 = q0 + 1;
            float b0 = 0.f, b1 = 0.f;
            if (a.bias) {
              uint16_t h0, h1;
              asm volatile("ld.shared.u16 %0, [%1];"
                           : "=h"(h0)
                           : "r"(bcol_s + q0 * 128 + ((bchunk ^ (q0 & 7)) << 4)));
              asm volatile("ld.shared.u16 %0, [%1];"
                           : "=h"(h1)
                           : "r"(bcol_s + q1 * 128 + ((bchunk ^ (q1 & 7)) << 4)));
              b0 = h16_to_f32<BF16>(h0) * 1.4426950408889634f;
              b1 = h16_to_f32<BF16>(h1) * 1.4426950408889634f;
            }
            float v0 = ex2(fmaf(__uint_as_float(sr[2 * e]), sl2, b0));
            float v1 = ex2(fmaf(__uint_as_float(sr[2 * e + 1]), sl2, b1));
            if (!full) {
              v0 = (q0 < ca || q0 > cz) ? 0.f : v0;
              v1 = (q1 < ca || q1 > cz) ? 0.f : v1;
            }
            pk[16 * c + e] = pack2<BF16>(v0, v1);
            if constexpr (DROPOUT) {
              v0 = (keep[c] >> (2 * e)) & 1u ? v0 : 0.f;
              v1 = (keep[c] >> (2 * e + 1)) & 1u ? v1 : 0.f;
              chunk[e] = pack2<BF16>(v0, v1);
            } else {
              chunk[e] = pk[16 * c + e];
            }
          }
          tmem_st16(tS + po + 16 * c, chunk);
        }
        // the bias tile has been read: the producer can load the next one
        if (a.bias) mbar_arrive_warp(b_empty);
      } else if constexpr (BIAS) {
        // Sub-chunks of 16 queries; each one's bias values are requested one
        // sub-chunk ahead (the first of the next tile at the end of this
        // one), so the loads overlap the exponentials.
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if constexpr (DROPOUT) keep[c] = keep_bits(it, c);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int sc = 2 * c + hh;
            if (sc < 3)
              load_bias16(braw[(sc + 1) & 1], m0 + qo + 16 * (sc + 1));
            else if (it + 1 < n_it)
              load_bias16(braw[0], m0 + 128 + qo);
            uint32_t sr[16], half8[8];
            tmem_ld16(tS + qo + 16 * sc, sr);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int q0 = qo + 16 * sc + 2 * e, q1 = q0 + 1;
              const float b0 = h16_to_f32<BF16>(braw[sc & 1][2 * e]) * 1.4426950408889634f;
              const float b1 = h16_to_f32<BF16>(braw[sc & 1][2 * e + 1]) * 1.4426950408889634f;
              float v0 = ex2(fmaf(__uint_as_float(sr[2 * e]), sl2, b0));
              float v1 = ex2(fmaf(__uint_as_float(sr[2 * e + 1]), sl2, b1));
              if (!full) {
                v0 = (q0 < ca || q0 > cz) ? 0.f : v0;
                v1 = (q1 < ca || q1 > cz) ? 0.f : v1;
              }
              pk[16 * c + 8 * hh + e] = pack2<BF16>(v0, v1);
              if constexpr (DROPOUT) {
                const int kb = 16 * hh + 2 * e;  // bit of the 32-query chunk
                v0 = (keep[c] >> kb) & 1u ? v0 : 0.f;
                v1 = (keep[c] >> (kb + 1)) & 1u ? v1 : 0.f;
                half8[e] = pack2<BF16>(v0, v1);
              } else {
                half8[e] = pk[16 * c + 8 * hh + e];
              }
            }
            tmem_st8(tS + po + 16 * c + 8 * hh, half8);
          }
        }
      } else {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        if constexpr (DROPOUT) keep[c] = keep_bits(it, c);
        uint32_t sr[32];
        tmem_ld32(tS + qo + 32 * c, sr);
        uint32_t chunk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int q0 = qo + 32 * c + 2 * e, q1 = q0 + 1;
          float v0 = ex2(__uint_as_float(sr[2 * e]) * sl2);
          float v1 = ex2(__uint_as_float(sr[2 * e + 1]) * sl2);
          if (!full) {
            v0 = (q0 < ca || q0 > cz) ? 0.f : v0;
            v1 = (q1 < ca || q1 > cz) ? 0.f : v1;
          }
          pk[16 * c + e] = pack2<BF16>(v0, v1);
          if constexpr (DROPOUT) {
            v0 = (keep[c] >> (2 * e)) & 1u ? v0 : 0.f;
            v1 = (keep[c] >> (2 * e + 1)) & 1u ? v1 : 0.f;
            chunk[e] = pack2<BF16>(v0, v1);
          } else {
            chunk[e] = pk[16 * c + e];
          }
        }
        tmem_st16(tS + po + 16 * c, chunk);
      }
      }
      if (half == 0) {
        // S^T(it) has been read: the operand can take tile it+1's terms.
        if (it + 1 < n_it) put_row(sXQ, folded(v_next));
        if (it + 2 < n_it) v_next = row_val(it + 2);
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive_warp(p_ready);
      // ---- phase 2: dS^T = P^T o (dP^T - delta), into TMEM and shared memory ----
      ok = mbar_wait(dp_full, it & 1, abort_flag, a.status, kSiteSoftmax) &&
           (it == 0 || mbar_wait(dq_mma, (it - 1) & 1, abort_flag, a.status, kSiteSoftmax)) &&
           (!DROPOUT || mbar_wait(delta_ready(half), it & 1, abort_flag, a.status, kSiteSoftmax));
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t dr[32];
        tmem_ld32(tDP + qo + 32 * c, dr);  // 32 queries of dP^T - delta (raw dP^T with dropout)
        uint32_t dd[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 pe = unpack2<BF16>(pk[16 * c + e]);
          float d0, d1;
          if constexpr (DROPOUT) {
            // dS = P o (m s dP - delta): a dropped element keeps -P delta
            float2 dl;
            asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];"
                         : "=f"(dl.x), "=f"(dl.y)
                         : "r"(sDelta + (it & 1) * 256 + (32 * c + 2 * e) * 4));
            const float s0 = (keep[c] >> (2 * e)) & 1u ? a.drop_scale * __uint_as_float(dr[2 * e]) : 0.f;
            const float s1 =
                (keep[c] >> (2 * e + 1)) & 1u ? a.drop_scale * __uint_as_float(dr[2 * e + 1]) : 0.f;
            d0 = pe.x * (s0 - dl.x);
            d1 = pe.y * (s1 - dl.y);
          } else {
            d0 = pe.x * __uint_as_float(dr[2 * e]);
            d1 = pe.y * __uint_as_float(dr[2 * e + 1]);
          }
          dd[e] = pack2<BF16>(d0, d1);
          if constexpr (BIAS) {
            // dbias(i, j) = dS (queries past seqlen_q are not written)
            const int32_t i = m0 + qo + 32 * c + 2 * e;
            if (dbcol && i < sqb) {
              uint16_t* p = dbcol + (int64_t)i * a.dbias_stride[2];
              p[0] = (uint16_t)(dd[e] & 0xFFFFu);
              if (i + 1 < sqb) p[a.dbias_stride[2]] = (uint16_t)(dd[e] >> 16);
            }
          }
        }
        tmem_st16(tDP + po + 16 * c, dd);
        // dS (query-contiguous rows of this key) into the MN-major smem tile:
        // 64-query block `half`, 16-byte chunks 4c..4c+3 of row r, swizzled.
        const uint32_t rowb = sDS + half * 16384 + r * 128;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int chunk = (c * 4 + u) ^ (r & 7);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(rowb + chunk * 16),
                       "r"(dd[4 * u]), "r"(dd[4 * u + 1]), "r"(dd[4 * u + 2]), "r"(dd[4 * u + 3])
                       : "memory");
        }
      }
      if (half == 1) {
        // dP^T(it) (delta subtracted in the MMA) has been read: next tile's terms.
        if (it + 1 < n_it) put_row(sXD, folded(v_next));
        if (it + 2 < n_it) v_next = row_val(it + 2);
      }
      fence_proxy_async_smem();
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive_warp(ds_ready);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(acc_done, 0, abort_flag, a.status, kSiteEpilogue));
    if (ok) {
      // Group 0 stores dV, group 1 stores dK (scaled by sm_scale).
      tc_fence_after();
      const bool valid = j < sk;
      uint8_t* row = valid ? (half == 0 ? kv_row_ptr(a.dv, a.dv_stride, j)
                                        : kv_row_ptr(a.dk, a.dk_stride, j))
                           : nullptr;
      const float mul = half == 0 ? (DROPOUT ? a.drop_scale : 1.f) : a.sm_scale;
      const uint32_t tacc = tmem + lane_off + (half == 0 ? C::kColDV : C::kColDK);
      const int ncols = half == 0 ? a.Dv : a.D;  // dV has V's head dim, dK Q's
      for (int c = 0; c < (ncols + 15) / 16; ++c) {
        uint32_t rv[16], pv[8];
        tmem_ld16(tacc + 16 * c, rv);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          pv[e] = pack2<BF16>(__uint_as_float(rv[2 * e]) * mul, __uint_as_float(rv[2 * e + 1]) * mul);
        if (valid) st_row16(row, c, pv, ncols);
      }
    }
  } else {
    // ===================== dQ drain (warps 8-11) =====================
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::kDrainRegs));
    const int quad = warp & 3;
    const uint32_t tDQ = tmem + ((uint32_t)(quad * 32) << 16) + C::kColDQ;
    const uint32_t stage = sDQ + quad * (C::kDqBufs * 4096);
    int nbox = 0;  // boxes staged so far: cycles through the kDqBufs buffers across tiles
    for (int it = 0; it < n_it; ++it) {
      bool ok = mbar_wait(dq_mma, it & 1, abort_flag, a.status, kSiteDq);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const int32_t m0 = (mb + it) * 128;
      const int64_t row0 = a.q_packed ? (int64_t)(qrow0 + m0) : (int64_t)b * a.Sq + m0;
      // Each warp stages 32 x 32 fp32 boxes (32 rows of the accumulator x 32
      // head-dim columns, 128-byte swizzled like the tensor map) in one of its
      // two buffers and adds them with a TMA bulk reduction.  Rows of queries
      // outside the sequence hold exact zeros (their dS is 0), so whole boxes
      // can be added; columns past D are clipped by the tensor map.
      const int grow = (int)((int64_t)h * a.rows + row0);
      // Deterministic mode: the key tiles that visit this query tile form one
      // run [n_lo, ...]; this warp adds its column quarter of the tile after
      // the n - n_lo key tiles before it have added theirs (a counter per
      // head, tile and quarter), so every element's fp32 sum is taken in key
      // tile order whatever order the CTAs run in.
      int* order = a.order ? a.order + 4 * (int64_t)grow + quad : nullptr;
      auto wait_turn = [&]() -> bool {  // called after the tile left TMEM
        if (!order) return true;
        int lo_n = 0, hi_n = ntile;  // smallest n' with m < m_end(n'), n' in [0, ntile]
        while (lo_n < hi_n) {
          const int mid = (lo_n + hi_n) >> 1;
          int32_t mb2, me2;
          bwd_tile_range(win, sq, sk, mid * 128, &mb2, &me2);
          if (me2 > mb + it) hi_n = mid; else lo_n = mid + 1;
        }
        bool in_time = true;
        if (lane == 0) in_time = wait_counter(order, ntile - lo_n, abort_flag, a.status, kSiteDq);
        return __shfl_sync(0xffffffffu, in_time ? 1 : 0, 0) != 0;
      };
      auto issue_box = [&](uint32_t buf, int col, int row) {
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_2d(&a.tdq, buf, col, row);
          bulk_commit();
        }
      };
      auto next_buf = [&]() -> uint32_t {
        const uint32_t buf = stage + (nbox % C::kDqBufs) * 4096;
        ++nbox;
        if (lane == 0) bulk_wait_read<C::kDqBufs - 1>();
        __syncwarp();
        return buf;
      };
      if (C::kDqTransposed) {
        // lane = head-dim index d (this warp: columns 32 quad .. +31), TMEM
        // column = query.  Box rows are queries; each lane writes one float
        // per row.  The whole tile is read into registers first, so its TMEM
        // columns (shared with dP^T) are released before any staging.
        const bool active = 32 * quad < a.D;
        uint32_t v0[64], v1[64];
        tmem_ld64(tDQ, v0);
        tmem_ld64(tDQ + 64, v1);
        tc_fence_before();
        mbar_arrive_warp(dq_free);
        if (!wait_turn()) break;
        if (active) {
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const uint32_t buf = next_buf();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const uint32_t off = e * 128 + ((((uint32_t)lane >> 2) ^ (e & 7)) << 4) + (lane & 3) * 4;
              const uint32_t val = c4 < 2 ? v0[32 * c4 + e] : v1[32 * (c4 - 2) + e];
              asm volatile("st.shared.b32 [%0], %1;" ::"r"(buf + off), "r"(val) : "memory");
            }
            issue_box(buf, 32 * quad, grow + 32 * c4);
          }
        }
      } else {
        // lane = query row (this warp: rows 32 quad .. +31), TMEM column =
        // head-dim index.  Each lane writes its row's 32 floats of a box.  The
        // whole tile (at most 64 columns here) is read before any staging.
        constexpr int kChunks = DPAD / 32;
        uint32_t v[kChunks][32];
#pragma unroll
        for (int cc = 0; cc < kChunks; ++cc)
          if (32 * cc < a.D) tmem_ld32(tDQ + 32 * cc, v[cc]);
        tc_fence_before();
        mbar_arrive_warp(dq_free);
        if (!wait_turn()) break;
#pragma unroll
        for (int cc = 0; cc < kChunks; ++cc) {
          if (32 * cc >= a.D) break;
          const uint32_t buf = next_buf();
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t off = lane * 128 + (((uint32_t)k ^ (lane & 7)) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(buf + off),
                         "r"(v[cc][4 * k]), "r"(v[cc][4 * k + 1]), "r"(v[cc][4 * k + 2]),
                         "r"(v[cc][4 * k + 3])
                         : "memory");
          }
          issue_box(buf, 32 * cc, grow + 32 * quad);
        }
      }
      if (order && lane == 0) {
        // this warp's additions are complete before the next key tile's
        bulk_wait<0>();
        release_counter(order);
      }
    }
    // The staged tiles must stay in place until the TMA has added them.
    if (C::kStageDq && lane == 0) bulk_wait<0>();
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == C::kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int DPAD, bool BF16, bool DROPOUT, bool BIAS>
static cudaError_t launch_main(const BwdArgs& a, cudaStream_t stream) {
  using C = BwdCfg<DPAD, BIAS>;
  static_assert(C::kSmemBytes <= 232448, "shared memory budget");
  // One warp of each warpgroup per sub-partition: P/dS, P/dS, drain, TMA/MMA.
  static_assert(2 * C::kPdsRegs + C::kDrainRegs + C::kProducerRegs <= 4 * C::kLaunchRegs,
                "register split exceeds the launch budget");
  auto kern = attn_bwd_kernel<DPAD, BF16, DROPOUT, BIAS>;
  static std::atomic<uint64_t> prepared{0};
  const dim3 grid((a.Sk + 127) / 128, a.H, a.B);
  return prepared_launch(kern, prepared, a.dev, C::kSmemBytes, C::kLaunchRegs, [&] {
    kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(a);
  });
}

template <bool BF16>
static cudaError_t launch_all(const BwdArgs& a, cudaStream_t stream, int sms) {
  const int64_t groups = (int64_t)a.H * a.rows;
  if (groups > 0) {
    const bool narrow = a.Dv <= 64 && a.DA <= 64;  // 8 threads cover a row
    const int per_block = narrow ? 32 : 16;
    const int64_t want = (groups + per_block - 1) / per_block;
    const int grid = (int)(want < (int64_t)sms * 16 ? want : (int64_t)sms * 16);
    if (narrow)
      attn_bwd_pre_kernel<BF16, 8><<<grid, 256, 0, stream>>>(a);
    else
      attn_bwd_pre_kernel<BF16, 16><<<grid, 256, 0, stream>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (a.Sk > 0 && a.H > 0 && a.B > 0) {
    cudaError_t e = cudaSuccess;
    if (a.main_events[0] && (e = cudaEventRecord(a.main_events[0], stream)) != cudaSuccess) return e;
    // all tiles take the wider of the two head dims (TMA zero-fills the rest)
    const bool narrow = a.D <= 64 && a.Dv <= 64;
    const bool bias = a.bias || a.dbias;
    auto by_bias = [&](auto dpad, auto drop) -> cudaError_t {
      constexpr int P = decltype(dpad)::value;
      constexpr bool DR = decltype(drop)::value;
      return bias ? launch_main<P, BF16, DR, true>(a, stream) : launch_main<P, BF16, DR, false>(a, stream);
    };
    auto by_drop = [&](auto dpad) -> cudaError_t {
      return a.dropout ? by_bias(dpad, Flag<true>{}) : by_bias(dpad, Flag<false>{});
    };
    e = narrow ? by_drop(std::integral_constant<int, 64>{})
               : by_drop(std::integral_constant<int, 128>{});
    if (e != cudaSuccess) return e;
    if (a.main_events[1] && (e = cudaEventRecord(a.main_events[1], stream)) != cudaSuccess) return e;
  }
  if (groups > 0 && a.q_used) {
    // per sequence: Sq (the largest seqlen_q) bounds each sequence's rows
    const int64_t want = ((int64_t)a.H * a.Sq * ((a.D + 7) / 8) + 255) / 256;
    const dim3 grid((unsigned)a.B, (unsigned)(want < 64 ? (want > 0 ? want : 1) : 64));
    attn_dq_convert_seq_kernel<BF16><<<grid, 256, 0, stream>>>(a);
    return cudaGetLastError();
  }
  if (groups > 0) {
    const int64_t n = groups * ((a.D + 7) / 8);
    const int64_t want = (n + 255) / 256;
    const int grid = (int)(want < (int64_t)sms * 16 ? want : (int64_t)sms * 16);
    attn_dq_convert_kernel<BF16><<<grid, 256, 0, stream>>>(a);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

cudaError_t launch_bwd(const BwdArgs& a, cudaStream_t stream) {
  const int sms = a.sms > 0 ? a.sms : 148;
  return a.bf16 ? launch_all<true>(a, stream, sms) : launch_all<false>(a, stream, sms);
}

}  // namespace attn
