// Kernel argument blocks shared by the host launcher (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace attn {

// Tensor maps are 4-D (D, rows, heads, batch): dense BHSD uses rows = Sq or
// Sk and batch = B; packed 1THD uses rows = total tokens and batch = 1.
// Boxes are 64 columns x 128 rows with 128-byte swizzle.
struct FwdArgs {
  CUtensorMap tq, tk, tv;
  void* o;
  float* lse;
  int64_t o_stride[3];
  const int32_t* cu_q;
  const int32_t* cu_k;
  int32_t B, H, Sq, Sk, D;
  int32_t wl, wr, bottom_right, lse_th, bf16, negate;
  // Per side (Q: Q, O, LSE; K: K, V): packed 1THD with cumulative lengths in
  // cu_q / cu_k (B + 1 entries), or padded BHSD with per-batch lengths (B
  // entries); neither: dense BHSD.
  int32_t q_packed, k_packed, q_padded, k_padded;
  int64_t total_q;
  float scale_log2;  // |sm_scale| * log2(e)
  uint32_t* status;
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
  int32_t wl, wr, bottom_right, lse_th, bf16;
  // Per side, as in FwdArgs (Q: Q, O, LSE, dO, dQ; K: K, V, dK, dV).
  int32_t q_packed, k_packed, q_padded, k_padded;
  int64_t total_q, rows;  // rows of the workspace: B*Sq, or total_q when Q is packed
  float sm_scale;
  float scale_log2;       // sm_scale * log2(e) (sign kept)
  float* delta;           // workspace: [H][rows]
  float* dq_acc;          // workspace: [H][rows][D]
  uint32_t* status;
  cudaEvent_t main_events[2];  // optional, recorded around the main kernel
};

cudaError_t launch_fwd(const FwdArgs& args, cudaStream_t stream);
cudaError_t launch_bwd(const BwdArgs& args, cudaStream_t stream);

}  // namespace attn
