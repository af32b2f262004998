/*
 * attn.h -- C ABI of libattn.so: FlashAttention forward and backward for
 * NVIDIA B200 (sm_100a) with the Generalized Sliding Window mask.
 *
 * What the calls compute.  For every sequence b and head h, with
 * c = sm_scale and the window of the sequence (below):
 *     S_ij = c * <q_i, k_j> (+ bias_ij, optional),  LSE_i = ln sum_{allowed j} exp(S_ij),
 *     P_ij = exp(S_ij - LSE_i) on allowed j (0 elsewhere),  O_i = sum_j P_ij v_j.
 * A row with no allowed key gets O_i = 0 and LSE_i = -inf.  attn_bwd returns
 * the gradient of <dO, O> with respect to Q, K and V (and the bias):
 *     dV = P^T dO,  dS = P o (dO V^T - rowsum(dO o O)),  dQ = c dS K,  dK = c dS^T Q,
 *     dbias = dS.
 * The aotriton README (section "Kernel Support") names this kernel family:
 * FlashAttention after Tri Dao, which reaches the plain definition above.
 *
 * The window (AOTriton 0.10b release notes, "Major Changes from Release 0.9
 * Beta": causal masks are sliding windows and both window sides may be
 * negative; AOTriton 0.15b release notes, "Bottom-Right Aligned Sliding
 * Windows"): with d = seqlen_k - seqlen_q of the sequence,
 *   - window_left == ATTN_CAUSAL_TOP_LEFT:     key j allowed iff j <= i
 *   - window_left == ATTN_CAUSAL_BOTTOM_RIGHT: key j allowed iff j <= i + d
 *     (window_right is ignored for both sentinels, and the diagonal bit
 *     never shifts a sentinel)
 *   - otherwise (L, R) = (window_left, window_right) under the TOP_LEFT
 *     diagonal and (window_left - d, window_right + d) under BOTTOM_RIGHT;
 *     ATTN_WINDOW_INF on a side leaves it unbounded (and is not shifted);
 *     key j allowed iff i - L <= j <= i + R (both ends inclusive).
 * Negative windows are legal; an empty window masks its rows fully.
 *
 * Conventions of every call (AOTriton 0.14b release notes, "Runtime Bug
 * Fixes": the device is taken from the stream, calls do not rely on a
 * caller-held lock and keep no per-thread caches):
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream of the calling thread's current device).  The device is
 *     the stream's device, whatever the calling thread's current device is.
 *   - The caller owns every buffer, the backward workspace included; the
 *     library allocates no device memory and holds no per-call state, so
 *     calls from several host threads are safe.
 *   - Return value: a cudaError_t code.  0 = success.
 *     ATTN_ERROR_INVALID_VALUE (cudaErrorInvalidValue) for: a wrong
 *     struct_size / version, reserved VarlenBits set, an unsupported mode,
 *     dtype or head dimension, a NULL required pointer, a base address not
 *     16-byte aligned, a stride whose byte size is not a multiple of 16, a
 *     backward workspace that is too small, or a backward with H * rows_q
 *     (rows_q = B*Sq, or total_q for a packed Q side) of 2^31 - 256 or more.  ATTN_ERROR_NO_KERNEL_IMAGE
 *     (cudaErrorNoKernelImageForDevice) on a GPU other than sm_100.  Launch
 *     errors are passed through.  A failing call writes nothing.
 *   - Tensors: fp16 or bf16 (ATTN_DTYPE_*), the head dimension contiguous
 *     (stride 1), any D in [1, 128]; V, O, dO and dV may have a head
 *     dimension Dv of their own (version 2; AOTriton 0.15b release notes,
 *     "Kernel Bug Fixes", name Hdim_vo apart from Hdim_qk).  Strides are in ELEMENTS, and every
 *     stride's byte size must be a multiple of 16: a D that is not a multiple
 *     of 8 lives in rows the caller pads (e.g. a [..., 72] buffer viewed as
 *     [..., 67]); columns past D are never read into a result or written.
 *       dense  (BHSD):  element (b, h, s, d) at base + b*stride[0] + h*stride[1]
 *                       + s*stride[2] + d
 *       packed (1THD):  element (t, h, d) at base + t*stride[2] + h*stride[1] + d
 *                       (stride[0] is ignored); token t of sequence b is row
 *                       cu_seqlens[b] + t.
 *   - LSE is fp32 in the layout chosen by the VarlenBits lse_layout field:
 *       HT dense [B, H, Sq], HT packed [H, total_q],
 *       TH dense [B, Sq, H], TH packed [total_q, H]   (all contiguous).
 *   - A device-side wait that runs past its iteration limit does not hang or
 *     trap: the kernel records it in a status word and returns early (the
 *     output is then invalid).  attn_device_status() reads and clears it.
 */
#ifndef ATTN_H_
#define ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported symbols keep default visibility even when the library is built
 * with -fvisibility=hidden. */
#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

/* Version 2 adds the fields after cu_seqlens_k (forward) / main_kernel_events
 * (backward), version 3 the bias fields after flags.  A caller built against
 * an older version passes that version and its struct size
 * (ATTN_FWD_PARAMS_V1_SIZE, ATTN_FWD_PARAMS_V2_SIZE and the backward
 * counterparts); the fields it does not know then read as zero. */
#define ATTN_PARAMS_VERSION 3u

/* Return codes (numeric values of cudaError_t). */
#define ATTN_SUCCESS 0
#define ATTN_ERROR_INVALID_VALUE 1
#define ATTN_ERROR_NO_KERNEL_IMAGE 209

/* Element types of Q, K, V, O, dO, dQ, dK, dV. */
#define ATTN_DTYPE_FP16 0
#define ATTN_DTYPE_BF16 1

/* Window encodings (values chosen by this library; the pages name the
 * sentinel idea, not the numbers). */
#define ATTN_WINDOW_INF 2147483647
#define ATTN_CAUSAL_TOP_LEFT (-2147483647 - 1)
#define ATTN_CAUSAL_BOTTOM_RIGHT (-2147483647)

/*
 * VarlenBits, one uint32_t (AOTriton 0.14b release notes, "VarlenBits
 * supersedes VarlenType"; bit 18 from the 0.15b notes, "API Changes"):
 *   bits  7:0  Q-side VarlenMode    bits 15:8  K-side VarlenMode
 *   bits 17:16 lse_layout (0 = HT, 1 = TH; 2 and 3 are rejected)
 *   bit  18    principal diagonal (0 = TOP_LEFT, 1 = BOTTOM_RIGHT)
 *   bits 31:19 reserved, must be 0.
 * VarlenMode (one byte): bit 0 stacked (0 = BHSD, 1 = 1THD), bits 2:1 length
 * (0 uniform, 1 cumulative sums, 2 per-sequence array), bits 4:3 position
 * (0 uniform, 1 reuse the cumulative sums, 2 second array), bits 7:5
 * reserved.  Each side takes one of five modes on its own (the Q side
 * addresses Q, O, LSE, dO and dQ; the K side K, V, dK and dV):
 *   ATTN_VARLEN_MODE_DENSE   BHSD, every batch Sq queries / Sk keys;
 *   ATTN_VARLEN_MODE_PACKED  1THD, that side's cu_seqlens array holds B + 1
 *                            cumulative lengths (the positions reuse them);
 *   ATTN_VARLEN_MODE_PADDED  BHSD sized [B, H, Sq, D] / [B, H, Sk, D], with
 *                            per-batch lengths: that side's cu_seqlens array
 *                            holds B lengths (not cumulative; clamped to
 *                            [0, Sq] / [0, Sk]);
 *   ATTN_VARLEN_MODE_PACKED_USED (version 2)
 *                            1THD whose sequence b occupies rows
 *                            [cu_seqlens[b], cu_seqlens[b + 1]) (B + 1
 *                            cumulative entries, the positions) of which the
 *                            first seqused[b] are used (a packed cache whose
 *                            slots are longer than their contents);
 *   ATTN_VARLEN_MODE_PACKED_OFFSETS (version 2)
 *                            1THD whose sequence b starts at row
 *                            cu_seqlens[b] (B entries: a second array of
 *                            positions, in any order) and has seqused[b]
 *                            rows; the used ranges must not overlap.
 * In every mode with lengths, rows of a tensor that lie outside every used
 * range are padding: never written, and their contents (NaN included) do not
 * reach any result.  Lengths and positions are clamped on the device to the
 * tensor (and, for PACKED_USED, to the slot).  A batch index b names the same
 * sequence on both sides.  Any other mode returns ATTN_ERROR_INVALID_VALUE.
 */
#define ATTN_VARLEN_MODE(stacked, length, position) \
  ((uint32_t)(stacked) | ((uint32_t)(length) << 1) | ((uint32_t)(position) << 3))
#define ATTN_VARLEN_MODE_DENSE ATTN_VARLEN_MODE(0, 0, 0)
#define ATTN_VARLEN_MODE_PACKED ATTN_VARLEN_MODE(1, 1, 1)
#define ATTN_VARLEN_MODE_PADDED ATTN_VARLEN_MODE(0, 2, 0)
#define ATTN_VARLEN_MODE_PACKED_USED ATTN_VARLEN_MODE(1, 2, 1)
#define ATTN_VARLEN_MODE_PACKED_OFFSETS ATTN_VARLEN_MODE(1, 2, 2)
#define ATTN_LSE_HT 0u
#define ATTN_LSE_TH 1u
#define ATTN_DIAGONAL_TOP_LEFT 0u
#define ATTN_DIAGONAL_BOTTOM_RIGHT 1u
#define ATTN_VARLEN_BITS(qmode, kmode, lse_layout, diagonal)                      \
  ((uint32_t)(qmode) | ((uint32_t)(kmode) << 8) | ((uint32_t)(lse_layout) << 16) | \
   ((uint32_t)(diagonal) << 18))

/*
 * Forward parameters.  Sizes: dense -- B batches of Sq queries and Sk keys;
 * packed -- B sequences, Sq / Sk the largest seqlen_q / seqlen_k (they size
 * the launch; a sequence longer than them is an error of the caller, whose
 * results are then unspecified, though nothing outside the tensors, the
 * bias included, is read or written), total_q / total_k the rows of the
 * packed tensors, cu_seqlens_q / _k device arrays of B + 1 int32 cumulative
 * lengths starting at 0 (each entry is clamped to [0, total_q] / [0,
 * total_k] on the device, so an array that runs past the tensors shortens
 * the sequences concerned; nothing outside the tensors is read or written);
 * padded -- dense tensors of B batches with Sq / Sk rows, cu_seqlens_q / _k
 * device arrays of B int32 lengths (seqlen_q / seqlen_k of each batch);
 * PACKED_USED / PACKED_OFFSETS -- as packed, with the positions in
 * cu_seqlens_q / _k and the lengths in seqused_q / _k (see VarlenBits).
 *
 * Dropout (version 2; AOTriton 0.10b release notes, "Major Changes from
 * Release 0.9 Beta": Philox with 32-bit words in groups of four; 0.14b notes,
 * "Minor Changes from Release 0.13 Beta": the four words of a counter in
 * generation order): with 0 < dropout_p < 1, element (i, j) of P (query row
 * i and key j counted within their sequence, head index bh = b * H + h) is
 * kept iff word (j mod 4) of Philox4x32-10 on the counter
 * (j div 4, i, bh, philox_offset) under the key (low, high 32 bits of
 * philox_seed) is below floor((1 - dropout_p) * 2^32); kept elements are
 * scaled by 1 / (1 - dropout_p).  LSE is that of the softmax without
 * dropout.  The backward regenerates the same mask from the same fields.
 *
 * Additive bias (version 3; AOTriton 0.10b release notes, "Known Problems",
 * and 0.14b notes, "Kernel Bug Fixes", where the bias is converted to fp32
 * before it is added): with bias != NULL the logits are
 *     S_ij = c * <q_i, k_j> + bias(b, h, i, j)
 * on allowed pairs (the bias never unmasks a pair), with LSE, P and O taken
 * from these S.  bias has the dtype of Q; element (b, h, i, j), i and j
 * counted within sequence b (i < seqlen_q <= Sq, j < seqlen_k <= Sk), is at
 * bias + b*bias_stride[0] + h*bias_stride[1] + i*bias_stride[2] + j in every
 * varlen mode (a [B, H, Sq, Sk] tensor; elements past a sequence's lengths
 * are not read).  bias_stride[0] and [1] may be 0 (one bias for all batches
 * or heads); every stride's byte size is a multiple of 16 and the base is
 * 16-byte aligned.  Bias entries must be finite.
 */
typedef struct attn_fwd_params {
  uint32_t struct_size; /* sizeof(attn_fwd_params) */
  uint32_t version;     /* ATTN_PARAMS_VERSION */
  int32_t dtype;        /* ATTN_DTYPE_FP16 or ATTN_DTYPE_BF16 */
  int32_t B, H, Sq, Sk, D;
  int64_t total_q, total_k; /* packed only */
  const void* q;            /* [B,H,Sq,D] or [total_q,H,D] */
  const void* k;            /* [B,H,Sk,D] or [total_k,H,D] */
  const void* v;            /* like k */
  void* o;                  /* like q, written */
  float* lse;               /* written; may be NULL (then not written) */
  int64_t q_stride[3], k_stride[3], v_stride[3], o_stride[3]; /* batch, head, seq */
  float sm_scale;           /* any finite value, zero and negative included */
  int32_t window_left, window_right;
  uint32_t varlen_bits;
  const int32_t* cu_seqlens_q; /* packed / padded only, device memory */
  const int32_t* cu_seqlens_k;
  /* ---- version 2 ---- */
  const int32_t* seqused_q;    /* PACKED_USED / PACKED_OFFSETS: B lengths, device memory */
  const int32_t* seqused_k;
  int32_t Dv;                  /* head dim of V and O, in [1, 128]; 0 = D */
  float dropout_p;             /* [0, 1); 0 = no dropout */
  uint64_t philox_seed;
  uint32_t philox_offset;
  uint32_t flags;              /* none defined for the forward: must be 0 */
  /* ---- version 3 ---- */
  const void* bias;            /* NULL: no bias */
  int64_t bias_stride[3];      /* batch, head, query row (elements) */
} attn_fwd_params;
#define ATTN_FWD_PARAMS_V1_SIZE ((uint32_t)offsetof(attn_fwd_params, seqused_q))
#define ATTN_FWD_PARAMS_V2_SIZE ((uint32_t)offsetof(attn_fwd_params, bias))

/*
 * Backward parameters: the forward's fields plus the forward output O, its
 * LSE (same layout as written by attn_fwd, required), the incoming gradient
 * dO (its own strides: it need not share O's), the outputs dQ / dK / dV and
 * a caller-owned device workspace of attn_bwd_workspace_size() bytes,
 * 256-byte aligned.  The workspace holds, after the call, the fp32 rowsums
 * delta = rowsum(dO o O) [H][rows] followed by the fp32 dQ accumulator
 * [H][rows][D], rows = B*Sq (dense) or total_q (packed), and with
 * ATTN_BWD_DETERMINISTIC the int32 order counters [H][rows][4].
 *
 * Bias (version 3): the forward's bias (same fields, required to recompute
 * P when the forward had one) and an optional output dbias, the gradient of
 * <dO, O> with respect to the bias: dbias(b, h, i, j) = dS_ij on allowed
 * pairs, 0 on masked pairs of the sequence, in the dtype of Q and addressed
 * like the bias through dbias_stride (all of them positive where the extent
 * is above 1: one element per (b, h, i, j); a caller that broadcast the bias
 * sums the result itself).  Elements past a sequence's lengths are not
 * written.  dbias without bias is the gradient at a zero bias.
 */
typedef struct attn_bwd_params {
  uint32_t struct_size; /* sizeof(attn_bwd_params) */
  uint32_t version;     /* ATTN_PARAMS_VERSION */
  int32_t dtype;
  int32_t B, H, Sq, Sk, D;
  int64_t total_q, total_k;
  const void* q;
  const void* k;
  const void* v;
  const void* o;
  const void* dout;
  const float* lse;
  void* dq;
  void* dk;
  void* dv;
  int64_t q_stride[3], k_stride[3], v_stride[3], o_stride[3], do_stride[3];
  int64_t dq_stride[3], dk_stride[3], dv_stride[3];
  float sm_scale;
  int32_t window_left, window_right;
  uint32_t varlen_bits;
  const int32_t* cu_seqlens_q;
  const int32_t* cu_seqlens_k;
  void* workspace;
  size_t workspace_bytes;
  /* Optional measurement hook: two cudaEvent_t created by the caller on the
   * stream's device, recorded on `stream` immediately before and after the
   * main backward kernel (so the caller can time it alone).  NULL: none. */
  void* main_kernel_events[2];
  /* ---- version 2 ---- */
  const int32_t* seqused_q;
  const int32_t* seqused_k;
  int32_t Dv;                  /* head dim of V, O, dO and dV; 0 = D */
  float dropout_p;             /* the forward's dropout fields */
  uint64_t philox_seed;
  uint32_t philox_offset;
  uint32_t flags;              /* ATTN_BWD_DETERMINISTIC or 0 */
  /* ---- version 3 ---- */
  const void* bias;            /* the forward's bias, or NULL */
  void* dbias;                 /* written when not NULL */
  int64_t bias_stride[3], dbias_stride[3];
} attn_bwd_params;
#define ATTN_BWD_PARAMS_V1_SIZE ((uint32_t)offsetof(attn_bwd_params, seqused_q))
#define ATTN_BWD_PARAMS_V2_SIZE ((uint32_t)offsetof(attn_bwd_params, bias))

/* attn_bwd_params.flags: add the dQ contributions of the key tiles in a
 * fixed order, so that repeated calls give bit-identical dQ (AOTriton 0.15b
 * release notes, "Known Problems", record run-to-run differences of the
 * backward).  Costs some speed and H * rows * 16 bytes more workspace. */
#define ATTN_BWD_DETERMINISTIC 1u

/* Forward: writes O and (unless lse is NULL) LSE.  One kernel launch. */
ATTN_API int attn_fwd(const attn_fwd_params* params, void* stream);

/* Backward: writes dQ, dK, dV (and the workspace).  Three kernel launches on
 * `stream`: rowsum(dO o O) with the dQ accumulator cleared, the main
 * backward, and the dQ conversion. */
ATTN_API int attn_bwd(const attn_bwd_params* params, void* stream);

/* Bytes of device workspace attn_bwd needs for these sizes (host only; reads
 * the size fields, no pointer).  0 if the sizes are invalid. */
ATTN_API size_t attn_bwd_workspace_size(const attn_bwd_params* params);

/*
 * attn_bwd without a caller-provided workspace (the pages have no counterpart
 * of this call; it serves callers of this library that cannot allocate device
 * memory: hosts that own all device memory and hand a kernel library no
 * allocator, and latency-critical paths where cudaMalloc's implicit
 * synchronisation is not acceptable).
 *
 * The backward's scratch memory (fp32 row sums and the fp32 dQ accumulator)
 * comes from a device array compiled into the library, ATTN_STATIC_WORKSPACE_BYTES
 * bytes, which every GPU that loads the library holds until the process exits.
 * The caller passes inputs and outputs only; params->workspace and
 * params->workspace_bytes are ignored.  The call allocates nothing.
 *   - params must be of the current version (struct_size ==
 *     sizeof(attn_bwd_params)); older struct sizes are rejected with
 *     ATTN_ERROR_INVALID_VALUE.
 *   - Sizes whose attn_bwd_workspace_size() exceeds ATTN_STATIC_WORKSPACE_BYTES
 *     are rejected with cudaErrorMemoryAllocation (2) before any GPU work;
 *     otherwise the return codes are those of attn_bwd.
 *   - Every call looks up the device address of the array on the stream's
 *     device (so a reset of the device's context, which can move it, is
 *     harmless); the first call on a device may also load the library's
 *     device code there, so make that first call before any stream capture.
 *   - Every call on a device shares the one array and leaves its contents
 *     there; each call clears the accumulator it needs before use.  Calls whose
 *     work overlaps on the GPU (different streams without ordering between
 *     them) race on the array and give wrong results: order them.
 */
#define ATTN_STATIC_WORKSPACE_BYTES (64u << 20)
ATTN_API int attn_bwd_static_workspace(const attn_bwd_params* params, void* stream);

/* Number of allowed (query, key) pairs of one sequence under a window, the
 * unit of the FLOP counts (4*D per pair forward, 10*D backward).  Host only. */
ATTN_API int64_t attn_allowed_pairs(int32_t seqlen_q, int32_t seqlen_k, int32_t window_left,
                           int32_t window_right, uint32_t bottom_right);

/*
 * The kernels' tile plan, computed on the host by the same code the kernels
 * run, for tests and tools.  For the query tile [m0, m0 + 128) of a sequence
 * (seqlen_q, seqlen_k) it writes the half-open range of 128-key tiles the
 * forward visits, *n_begin / *n_end, and for each tile n in the range
 * full_mask[n - n_begin] = 1 if no element of the tile is masked (the kernel
 * then skips the element test), 0 otherwise; full_mask needs room for
 * ceil(seqlen_k / 128) bytes.  Returns 0, or ATTN_ERROR_INVALID_VALUE.
 */
ATTN_API int attn_tile_plan(int32_t seqlen_q, int32_t seqlen_k, int32_t window_left,
                   int32_t window_right, uint32_t bottom_right, int32_t m0, int32_t* n_begin,
                   int32_t* n_end, uint8_t* full_mask);

/* The backward's mirror: for the key tile [n0, n0 + 128), the half-open range
 * of 128-query tiles that see any of its keys. */
ATTN_API int attn_tile_plan_bwd(int32_t seqlen_q, int32_t seqlen_k, int32_t window_left,
                       int32_t window_right, uint32_t bottom_right, int32_t n0,
                       int32_t* m_begin, int32_t* m_end);

/* Reads and clears the device status word of the stream's device (waits for
 * the stream).  *status = 0 when every device-side wait finished in time;
 * otherwise bit k marks wait site k that gave up.  Returns a cudaError_t.
 * There is one status word per device, shared by every caller and stream on
 * that device: a bit set by one caller's kernel is seen (and cleared) by
 * whichever caller reads it first, so callers that run concurrently on one
 * device and need to attribute a failure must order their reads. */
ATTN_API int attn_device_status(void* stream, uint32_t* status);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_H_ */
