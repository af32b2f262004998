// Kernel argument blocks shared by the host launcher (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace attn {

// Tensor maps are 4-D (D, rows, heads, batch): dense BHSD uses rows = Sq or
// Sk and batch = B; packed 1THD uses rows = total tokens and batch = 1.
// Boxes are 64 columns x 128 rows with 128-byte swizzle.
struct FwdArgs {
  CUtensorMap tq, tk, tv;
  CUtensorMap tk2;  // K with 64 x 64 boxes (the CTA-pair kernel loads half key tiles)
  void* o;
  float* lse;
  int64_t o_stride[3];
  const int32_t* cu_q;
  const int32_t* cu_k;
  int32_t B, H, Sq, Sk, D;
  int32_t D16;  // D rounded up to 16 (MMA N; the columns past D are zero)
  int32_t Dv, Dv16;  // head dim of V and O, and rounded up to 16
  int32_t wl, wr, bottom_right, lse_th, bf16, negate;
  int32_t units_by_cost;  // number units query block slowest (any mask), else fastest
  // Per side (Q: Q, O, LSE; K: K, V): stacked 1THD (positions in cu_q / cu_k:
  // B + 1 cumulative entries, or B start rows with *_offsets; lengths from
  // the cumulative differences, or from used_q / used_k with *_used), or
  // padded BHSD with per-batch lengths in cu_q / cu_k (B entries); neither:
  // dense BHSD.
  int32_t q_packed, k_packed, q_padded, k_padded;
  int32_t q_used, k_used, q_offsets, k_offsets;
  const int32_t* used_q;
  const int32_t* used_k;
  int64_t total_q, total_k;  // rows of packed tensors (sequence bounds are clamped to them)
  float scale_log2;  // |sm_scale| * log2(e)
  uint32_t* status;
  int32_t dev, sms;  // the stream's device and its SM count (host side only)
  // Dropout: an element is kept iff its Philox word < keep_below; kept
  // elements are scaled by drop_scale = 1 / (1 - p).
  int32_t dropout;
  uint32_t keep_below, seed_lo, seed_hi, philox_offset;
  float drop_scale;
  // Additive bias: element (b, h, i, j) of sequence b at bias + b*s[0] +
  // h*s[1] + i*s[2] + j (16-bit, the dtype of Q), or null.  The forward
  // stages it through `tb`, a 4-D map (Sk, Sq, heads, batches) whose head /
  // batch extent is 1 where that stride is 0 (the *_bcast flags: coordinate 0).
  const void* bias;
  int64_t bias_stride[3];
  CUtensorMap tb;
  int32_t bias_b_bcast, bias_h_bcast;
};

struct BwdArgs {
  CUtensorMap tq, tk, tv, tdo;
  CUtensorMap tdq;  // fp32 dQ accumulator as 2-D (D, H*rows), 32 x 32 boxes
  const void* o;
  const void* dout;
  const float* lse;
  void* dq;
  void* dk;
  void* dv;
  int64_t o_stride[3], do_stride[3], dq_stride[3], dk_stride[3], dv_stride[3];
  const int32_t* cu_q;
  const int32_t* cu_k;
  int32_t B, H, Sq, Sk, D;
  int32_t D16;  // D rounded up to 16 (MMA N; the columns past D are zero)
  int32_t Dv, Dv16;  // head dim of V, O, dO and dV, and rounded up to 16
  int32_t DA;   // row pitch of the fp32 dQ accumulator: D rounded up to 8
  int32_t wl, wr, bottom_right, lse_th, bf16;
  // Per side, as in FwdArgs (Q: Q, O, LSE, dO, dQ; K: K, V, dK, dV).
  int32_t q_packed, k_packed, q_padded, k_padded;
  int32_t q_used, k_used, q_offsets, k_offsets;
  const int32_t* used_q;
  const int32_t* used_k;
  int64_t total_q, total_k;  // rows of packed tensors (sequence bounds are clamped to them)
  int64_t rows;           // rows of the workspace: B*Sq, or total_q when Q is packed
  float sm_scale;
  float scale_log2;       // sm_scale * log2(e) (sign kept)
  float* delta;           // workspace: [H][rows]
  float* dq_acc;          // workspace: [H][rows][DA]
  int32_t* order;         // workspace: [H][rows][4] order counters (deterministic dQ), or null
  uint32_t* status;
  int32_t dev, sms;            // the stream's device and its SM count (host side only)
  cudaEvent_t main_events[2];  // optional, recorded around the main kernel
  int32_t dropout;             // as in FwdArgs
  uint32_t keep_below, seed_lo, seed_hi, philox_offset;
  float drop_scale;
  // Bias as in FwdArgs (null: zero) and its gradient dS, addressed the same
  // way through dbias_stride (null: not written).
  const void* bias;
  void* dbias;
  int64_t bias_stride[3], dbias_stride[3];
  CUtensorMap tb;  // as in FwdArgs (head dim 64 stages the bias tiles)
  int32_t bias_b_bcast, bias_h_bcast;
};

cudaError_t launch_fwd(const FwdArgs& args, cudaStream_t stream);
// The CTA-pair forward (dense, no mask, bias or dropout, the wider head dim
// in (64, 128], Dv a multiple of 16).
bool fwd_pair_eligible(const FwdArgs& args);
cudaError_t launch_fwd_pair(const FwdArgs& args, cudaStream_t stream);

// Checks a kernel's register count at launch (the setmaxnreg splits assume
// `min_regs` per thread; with fewer, the warpgroups that raise their count
// would wait forever) and sets its dynamic shared-memory limit, once per
// device: `done` holds one bit per device index below 64 (others are prepared
// on every call).
template <class Kern>
cudaError_t prepare_kernel(Kern kern, std::atomic<uint64_t>& done, int dev, int smem_bytes,
                           int min_regs) {
  const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t)1 << dev : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs < min_regs) return cudaErrorLaunchOutOfResources;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
  if (e != cudaSuccess) return e;
  done.fetch_or(bit, std::memory_order_release);
  return cudaSuccess;
}

// Launches `launch()` after prepare_kernel; if the launch is refused while the
// preparation was taken from the cache (the device's context was reset since,
// which drops the attribute), prepares again and launches once more.
template <class Kern, class Launch>
cudaError_t prepared_launch(Kern kern, std::atomic<uint64_t>& done, int dev, int smem_bytes,
                            int min_regs, Launch&& launch) {
  const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t)1 << dev : 0;
  const bool cached = bit && (done.load(std::memory_order_acquire) & bit);
  cudaError_t e = prepare_kernel(kern, done, dev, smem_bytes, min_regs);
  if (e != cudaSuccess) return e;
  launch();
  e = cudaGetLastError();
  if (e != cudaSuccess && cached) {
    done.fetch_and(~bit, std::memory_order_acq_rel);
    e = prepare_kernel(kern, done, dev, smem_bytes, min_regs);
    if (e != cudaSuccess) return e;
    launch();
    e = cudaGetLastError();
  }
  return e;
}
cudaError_t launch_bwd(const BwdArgs& args, cudaStream_t stream);

}  // namespace attn
