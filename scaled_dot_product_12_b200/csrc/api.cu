// C ABI of libattn.so (declared and documented in include/attn.h): parameter
// validation, tensor-map encoding and kernel launches.  Host code only.
//
// The interface follows the V3 shape the AOTriton 0.10b release notes print
// ("Major Changes from Release 0.9 Beta": attn_fwd(params, version, stream)),
// the versioned-params rule of the 0.15b notes ("API Changes": a struct
// version field; reserved VarlenBits rejected with an invalid-value error) and
// the runtime rules of the 0.14b notes ("Runtime Bug Fixes": the device comes
// from the stream, no reliance on a caller-held lock, no per-thread caches,
// errors are returned, not hidden).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "../../include/attn.h"
#include "fwd.h"
#include "mask.cuh"

namespace {

__device__ uint32_t g_status;  // bits set by device-side waits that gave up

constexpr int kMaxDevices = 64;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// Per-device facts that outlive a context reset (compute capability, SM
// count), filled once under a lock.  The status word's device address is not
// cached: a reset of the device's primary context can move it, so every call
// looks it up (cheap once the module is loaded).
struct DeviceInfo {
  bool ready = false;
  bool sm100 = false;
  int sms = 0;
  uint32_t* status = nullptr;
};
std::mutex g_dev_mu;
DeviceInfo g_dev[kMaxDevices];

cudaError_t device_info(int dev, DeviceInfo* out) {
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo& d = g_dev[dev];
    if (!d.ready) {
      int major = 0, minor = 0, sms = 0;
      cudaError_t e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
      if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
      if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      if (e != cudaSuccess) return e;
      d.sm100 = (major == 10 && minor == 0);
      d.sms = sms;
      d.ready = true;
    }
    *out = d;
  }
  if (!out->sm100) return cudaSuccess;
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_status);  // current device == dev here
  if (e != cudaSuccess) return e;
  out->status = static_cast<uint32_t*>(p);
  return cudaSuccess;
}

// Runs `fn` with the stream's device current, restoring the caller's device;
// a failure to restore it is reported when the call itself succeeded.
template <class F>
cudaError_t on_stream_device(cudaStream_t stream, F&& fn) {
  int cur = 0, dev = 0;
  cudaError_t e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return e;
  dev = cur;
  if (stream != nullptr) {
    e = cudaStreamGetDevice(stream, &dev);
    if (e != cudaSuccess) return e;
  }
  if (dev != cur && (e = cudaSetDevice(dev)) != cudaSuccess) return e;
  DeviceInfo info;
  e = device_info(dev, &info);
  if (e == cudaSuccess) e = info.sm100 ? fn(dev, info) : cudaErrorNoKernelImageForDevice;
  if (dev != cur) {
    const cudaError_t r = cudaSetDevice(cur);
    if (e == cudaSuccess) e = r;
  }
  return e;
}

constexpr uint32_t kReservedBits = 0xFFF80000u;  // bits 31:19
constexpr uint32_t kModeReserved = 0xE0u;        // bits 7:5 of a VarlenMode

// Addressing of each side (Q: Q, O, LSE, dO, dQ; K: K, V, dK, dV).
struct Mode {
  bool q_packed, k_packed;    // 1THD (stacked), positions from cu_seqlens
  bool q_used, k_used;        // stacked, lengths from seqused
  bool q_offsets, k_offsets;  // stacked, cu_seqlens holds B start rows (not cumulative)
  bool q_padded, k_padded;    // BHSD with per-batch lengths
  bool lse_th;
  bool bottom_right;
};

bool decode_bits(uint32_t bits, Mode* m) {
  if (bits & kReservedBits) return false;
  const uint32_t qm = bits & 0xFFu, km = (bits >> 8) & 0xFFu, lse = (bits >> 16) & 3u;
  if ((qm | km) & kModeReserved) return false;
  auto known = [](uint32_t x) {
    return x == ATTN_VARLEN_MODE_DENSE || x == ATTN_VARLEN_MODE_PACKED ||
           x == ATTN_VARLEN_MODE_PADDED || x == ATTN_VARLEN_MODE_PACKED_USED ||
           x == ATTN_VARLEN_MODE_PACKED_OFFSETS;
  };
  if (!known(qm) || !known(km)) return false;  // each side on its own
  if (lse > 1) return false;
  auto stacked = [](uint32_t x) { return (x & 1u) != 0; };
  m->q_packed = stacked(qm);
  m->k_packed = stacked(km);
  m->q_used = (qm == ATTN_VARLEN_MODE_PACKED_USED || qm == ATTN_VARLEN_MODE_PACKED_OFFSETS);
  m->k_used = (km == ATTN_VARLEN_MODE_PACKED_USED || km == ATTN_VARLEN_MODE_PACKED_OFFSETS);
  m->q_offsets = (qm == ATTN_VARLEN_MODE_PACKED_OFFSETS);
  m->k_offsets = (km == ATTN_VARLEN_MODE_PACKED_OFFSETS);
  m->q_padded = (qm == ATTN_VARLEN_MODE_PADDED);
  m->k_padded = (km == ATTN_VARLEN_MODE_PADDED);
  m->lse_th = (lse == ATTN_LSE_TH);
  m->bottom_right = ((bits >> 18) & 1u) != 0;
  return true;
}

// Copies a params struct of any version into a full current one (callers of
// an older version get zeros in the fields they do not know).
template <class P>
bool normalize(const P* in, uint32_t v1_size, uint32_t v2_size, P* out) {
  if (!in) return false;
  if (in->version == ATTN_PARAMS_VERSION && in->struct_size == sizeof(P)) {
    std::memcpy(out, in, sizeof(P));
    return true;
  }
  const uint32_t known = in->version == 1u ? v1_size : in->version == 2u ? v2_size : 0u;
  if (known != 0u && in->struct_size == known) {
    std::memset(out, 0, sizeof(P));
    std::memcpy(out, in, known);
    out->struct_size = sizeof(P);
    out->version = ATTN_PARAMS_VERSION;
    return true;
  }
  return false;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A tensor described by base + strides (elements) of a 16-bit type.  Checks
// the strides the kernels (and TMA) rely on: multiples of 16 bytes, positive
// where the extent is above 1.
bool strides_ok(const int64_t* st, bool packed, int64_t nb, int64_t nh, int64_t nrows) {
  const int64_t lim = (int64_t)1 << 38;
  auto ok = [&](int64_t s, int64_t extent) {
    if (extent <= 1) return true;
    return s > 0 && s < lim && ((s * 2) % 16) == 0;
  };
  if (!packed && !ok(st[0], nb)) return false;
  return ok(st[1], nh) && ok(st[2], nrows);
}

// Strides (elements) of a [B, H, Sq, Sk] bias: byte sizes multiples of 16,
// batch and head strides may be 0 (broadcast) when `broadcast` allows it,
// the row stride positive where there is more than one row.
bool bias_strides_ok(const int64_t* st, int64_t nb, int64_t nh, int64_t nrows, bool broadcast) {
  const int64_t lim = (int64_t)1 << 38;
  auto ok = [&](int64_t s, int64_t extent, bool zero_ok) {
    if (extent <= 1) return true;
    if (s == 0) return zero_ok;
    return s > 0 && s < lim && ((s * 2) % 16) == 0;
  };
  return ok(st[0], nb, broadcast) && ok(st[1], nh, broadcast) && ok(st[2], nrows, false);
}

cudaError_t make_map(CUtensorMap* map, const void* base, int D, int64_t rows, int H, int B,
                     const int64_t* st, bool packed, int box_rows = 128) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  const int64_t rows_c = rows > 0 ? rows : 1;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)rows_c, (cuuint64_t)(H > 0 ? H : 1),
                        (cuuint64_t)(packed ? 1 : (B > 0 ? B : 1))};
  // Strides (bytes) of dims 1..3; a dimension of extent 1 gets a harmless
  // placeholder stride so the encoder accepts it.
  auto pick = [&](int64_t s, uint64_t extent) -> cuuint64_t {
    if (extent > 1) return (cuuint64_t)(s * 2);
    return 16;
  };
  cuuint64_t strides[3] = {pick(st[2], dims[1]), pick(st[1], dims[2]),
                           packed ? (cuuint64_t)16 : pick(st[0], dims[3])};
  cuuint32_t box[4] = {64, (cuuint32_t)box_rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 4, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// 4-D map over a [B, H, Sq, Sk] bias (the strides checked by
// bias_strides_ok): dimensions (Sk, Sq, H, B), 64 x 128 boxes with 128-byte
// swizzle, a head or batch dimension of stride 0 (broadcast) or extent 1 given
// extent 1 (the kernel then uses coordinate 0: *h_bcast / *b_bcast).
cudaError_t make_bias_map(CUtensorMap* map, const void* base, int Sq, int Sk, int H, int B,
                          const int64_t* st, int32_t* h_bcast, int32_t* b_bcast) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  const bool hb = H <= 1 || st[1] == 0, bb = B <= 1 || st[0] == 0;
  cuuint64_t dims[4] = {(cuuint64_t)(Sk > 0 ? Sk : 1), (cuuint64_t)(Sq > 0 ? Sq : 1),
                        (cuuint64_t)(hb ? 1 : H), (cuuint64_t)(bb ? 1 : B)};
  cuuint64_t strides[3] = {dims[1] > 1 ? (cuuint64_t)(st[2] * 2) : 16,
                           hb ? 16 : (cuuint64_t)(st[1] * 2), bb ? 16 : (cuuint64_t)(st[0] * 2)};
  cuuint32_t box[4] = {64, 128, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 4, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  *h_bcast = hb ? 1 : 0;
  *b_bcast = bb ? 1 : 0;
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// 2-D fp32 map over the dQ accumulator [H*rows][D] (row pitch DA*4 bytes),
// 32 x 32 boxes with 128-byte swizzle: the backward adds staged dQ tiles
// through it.
cudaError_t make_dq_map(CUtensorMap* map, float* base, int D, int DA, int64_t rows_total) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)(rows_total > 0 ? rows_total : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)DA * 4};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Checks shared by forward and backward (on a normalized struct).
template <class P>
bool common_ok(const P* p, Mode* m, uint32_t known_flags, bool check_pointers = true,
               bool dropout_built = true) {
  if (p->dtype != ATTN_DTYPE_FP16 && p->dtype != ATTN_DTYPE_BF16) return false;
  if (p->D < 1 || p->D > 128) return false;
  if (p->B < 0 || p->H < 0 || p->Sq < 0 || p->Sk < 0) return false;
  if (p->Sq >= attn::kBig || p->Sk >= attn::kBig) return false;
  if (!std::isfinite(p->sm_scale)) return false;
  if (!decode_bits(p->varlen_bits, m)) return false;
  if (m->q_packed && (p->total_q < 0 || p->total_q >= attn::kBig)) return false;
  if (m->k_packed && (p->total_k < 0 || p->total_k >= attn::kBig)) return false;
  if ((p->flags & ~known_flags) != 0) return false;
  if (p->Dv < 0 || p->Dv > 128) return false;  // 0: V and O share D
  if (!(p->dropout_p >= 0.f && p->dropout_p < 1.f)) return false;  // NaN fails too
  if (p->dropout_p != 0.f && !dropout_built) return false;
  // Stacked and padded sides read their positions / lengths from the device
  // arrays.
  if (check_pointers && p->B > 0) {
    if ((m->q_packed || m->q_padded) && !p->cu_seqlens_q) return false;
    if ((m->k_packed || m->k_padded) && !p->cu_seqlens_k) return false;
    if (m->q_used && !p->seqused_q) return false;
    if (m->k_used && !p->seqused_k) return false;
  }
  return true;
}

bool has_work(int B, int H, int64_t rows_q) { return B > 0 && H > 0 && rows_q > 0; }

// Dropout fields of the kernel arguments: keep iff the Philox word is below
// floor((1 - p) 2^32); a p so small that every word is kept is no dropout.
template <class Args, class P>
void set_dropout(Args& a, const P* p) {
  const double keep = std::floor((1.0 - (double)p->dropout_p) * 4294967296.0);
  a.dropout = p->dropout_p > 0.f && keep < 4294967296.0;
  a.keep_below = a.dropout ? (uint32_t)keep : 0u;
  a.drop_scale = a.dropout ? (float)(1.0 / (1.0 - (double)p->dropout_p)) : 1.f;
  a.seed_lo = (uint32_t)(p->philox_seed & 0xFFFFFFFFu);
  a.seed_hi = (uint32_t)(p->philox_seed >> 32);
  a.philox_offset = p->philox_offset;
}

}  // namespace

extern "C" {

int attn_fwd(const attn_fwd_params* params, void* stream_ptr) {
  attn_fwd_params full;
  if (!normalize(params, ATTN_FWD_PARAMS_V1_SIZE, ATTN_FWD_PARAMS_V2_SIZE, &full)) return cudaErrorInvalidValue;
  const attn_fwd_params* p = &full;
  Mode m;
  if (!common_ok(p, &m, /*known_flags=*/0u)) return cudaErrorInvalidValue;
  const int64_t rows_q = m.q_packed ? p->total_q : (int64_t)p->B * p->Sq;
  const int64_t rows_k = m.k_packed ? p->total_k : (int64_t)p->B * p->Sk;
  if (!has_work(p->B, p->H, rows_q)) return cudaSuccess;
  if (!p->q || !p->o) return cudaErrorInvalidValue;
  if (rows_k > 0 && (!p->k || !p->v)) return cudaErrorInvalidValue;
  if (!aligned16(p->q) || !aligned16(p->o) || (rows_k > 0 && (!aligned16(p->k) || !aligned16(p->v))))
    return cudaErrorInvalidValue;
  if (p->lse && (reinterpret_cast<uintptr_t>(p->lse) & 3u)) return cudaErrorInvalidValue;
  const int64_t nq = m.q_packed ? p->total_q : p->Sq, nk = m.k_packed ? p->total_k : p->Sk;
  if (!strides_ok(p->q_stride, m.q_packed, p->B, p->H, nq) ||
      !strides_ok(p->o_stride, m.q_packed, p->B, p->H, nq) ||
      !strides_ok(p->k_stride, m.k_packed, p->B, p->H, nk) ||
      !strides_ok(p->v_stride, m.k_packed, p->B, p->H, nk))
    return cudaErrorInvalidValue;
  if (p->bias && (!aligned16(p->bias) || !bias_strides_ok(p->bias_stride, p->B, p->H, p->Sq, true)))
    return cudaErrorInvalidValue;

  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  return on_stream_device(stream, [&](int dev, const DeviceInfo& info) -> cudaError_t {
    attn::FwdArgs a;
    std::memset(&a, 0, sizeof(a));
    const void* kbase = rows_k > 0 ? p->k : p->q;
    const void* vbase = rows_k > 0 ? p->v : p->q;
    const int Dv = p->Dv ? p->Dv : p->D;
    a.o = p->o;
    a.lse = p->lse;
    for (int i = 0; i < 3; ++i) a.o_stride[i] = p->o_stride[i];
    a.cu_q = p->cu_seqlens_q;
    a.cu_k = p->cu_seqlens_k;
    a.B = p->B;
    a.H = p->H;
    a.Sq = p->Sq;
    a.Sk = p->Sk;
    a.D = p->D;
    a.D16 = (p->D + 15) / 16 * 16;
    a.Dv = Dv;
    a.Dv16 = (Dv + 15) / 16 * 16;
    a.wl = p->window_left;
    a.wr = p->window_right;
    a.bottom_right = m.bottom_right;
    a.q_packed = m.q_packed;
    a.k_packed = m.k_packed;
    a.q_padded = m.q_padded;
    a.k_padded = m.k_padded;
    a.q_used = m.q_used;
    a.k_used = m.k_used;
    a.q_offsets = m.q_offsets;
    a.k_offsets = m.k_offsets;
    a.used_q = p->seqused_q;
    a.used_k = p->seqused_k;
    a.lse_th = m.lse_th;
    a.bf16 = p->dtype == ATTN_DTYPE_BF16;
    a.negate = p->sm_scale < 0.f;
    // unit costs differ under any window; equal without one
    a.units_by_cost = !(p->window_left == ATTN_WINDOW_INF && p->window_right == ATTN_WINDOW_INF);
    a.total_q = p->total_q;
    a.total_k = p->total_k;
    a.scale_log2 = std::fabs(p->sm_scale) * 1.4426950408889634f;
    a.status = info.status;
    a.dev = dev;
    a.sms = info.sms;
    set_dropout(a, p);
    a.bias = p->bias;
    for (int i = 0; i < 3; ++i) a.bias_stride[i] = p->bias_stride[i];
    // K is read in 128-row tiles by the one-CTA kernel and in 64-row halves
    // by the CTA-pair kernel: only the map of the kernel that runs is encoded.
    const bool pair = attn::fwd_pair_eligible(a);
    cudaError_t e = make_map(&a.tq, p->q, p->D, nq, p->H, p->B, p->q_stride, m.q_packed);
    if (e == cudaSuccess)
      e = pair ? make_map(&a.tk2, kbase, p->D, nk, p->H, p->B, p->k_stride, m.k_packed, 64)
               : make_map(&a.tk, kbase, p->D, nk, p->H, p->B, p->k_stride, m.k_packed);
    if (e == cudaSuccess) e = make_map(&a.tv, vbase, Dv, nk, p->H, p->B, p->v_stride, m.k_packed);
    if (e == cudaSuccess && p->bias)
      e = make_bias_map(&a.tb, p->bias, p->Sq, p->Sk, p->H, p->B, p->bias_stride, &a.bias_h_bcast,
                        &a.bias_b_bcast);
    if (e != cudaSuccess) return e;
    return attn::launch_fwd(a, stream);
  });
}

namespace {
// Workspace of the backward: delta [H][rows] fp32 (256-byte aligned), the dQ
// accumulator [H][rows][D] fp32, and with ATTN_BWD_DETERMINISTIC the order
// counters [H][rows][4] int32.
struct BwdWorkspace {
  size_t delta_bytes, acc_bytes, order_bytes;
  size_t total() const { return delta_bytes + acc_bytes + order_bytes; }
};
BwdWorkspace bwd_workspace(const attn_bwd_params* p, const Mode& m) {
  const int64_t rows = m.q_packed ? p->total_q : (int64_t)p->B * p->Sq;
  const int64_t n = (int64_t)p->H * rows;
  BwdWorkspace w;
  w.delta_bytes = ((size_t)n * 4 + 255) & ~(size_t)255;
  w.acc_bytes = (size_t)n * ((p->D + 7) / 8 * 8) * 4;
  w.order_bytes = (p->flags & ATTN_BWD_DETERMINISTIC) ? (size_t)n * 16 : 0;
  return w;
}
constexpr uint32_t kBwdFlags = ATTN_BWD_DETERMINISTIC;  // flags the backward accepts
constexpr bool kBwdDropout = true;                       // backward dropout kernels built
}  // namespace

size_t attn_bwd_workspace_size(const attn_bwd_params* params) {
  attn_bwd_params full;
  if (!normalize(params, ATTN_BWD_PARAMS_V1_SIZE, ATTN_BWD_PARAMS_V2_SIZE, &full)) return 0;
  Mode m;
  if (!common_ok(&full, &m, kBwdFlags, /*check_pointers=*/false, kBwdDropout)) return 0;
  return bwd_workspace(&full, m).total();
}

int attn_bwd(const attn_bwd_params* params, void* stream_ptr) {
  attn_bwd_params full;
  if (!normalize(params, ATTN_BWD_PARAMS_V1_SIZE, ATTN_BWD_PARAMS_V2_SIZE, &full)) return cudaErrorInvalidValue;
  const attn_bwd_params* p = &full;
  Mode m;
  if (!common_ok(p, &m, kBwdFlags, true, kBwdDropout)) return cudaErrorInvalidValue;
  const int64_t rows_q = m.q_packed ? p->total_q : (int64_t)p->B * p->Sq;
  const int64_t rows_k = m.k_packed ? p->total_k : (int64_t)p->B * p->Sk;
  if (!has_work(p->B, p->H, rows_q) && !(p->B > 0 && p->H > 0 && rows_k > 0)) return cudaSuccess;
  const void* need16[] = {p->q, p->o, p->dout, p->dq};
  for (const void* x : need16)
    if (rows_q > 0 && (!x || !aligned16(x))) return cudaErrorInvalidValue;
  const void* need16k[] = {p->k, p->v, p->dk, p->dv};
  for (const void* x : need16k)
    if (rows_k > 0 && (!x || !aligned16(x))) return cudaErrorInvalidValue;
  if (rows_q > 0 && (!p->lse || (reinterpret_cast<uintptr_t>(p->lse) & 3u)))
    return cudaErrorInvalidValue;
  // The dQ accumulator is reduced into through a 2-D tensor map whose row
  // coordinate (head * rows + row) is a signed 32-bit TMA coordinate.
  if ((int64_t)p->H * rows_q >= ((int64_t)1 << 31) - 256) return cudaErrorInvalidValue;
  const BwdWorkspace wl = bwd_workspace(p, m);
  const size_t ws = wl.total();
  if (ws > 0 && (!p->workspace || p->workspace_bytes < ws ||
                 (reinterpret_cast<uintptr_t>(p->workspace) & 255u)))
    return cudaErrorInvalidValue;
  const int64_t nq = m.q_packed ? p->total_q : p->Sq, nk = m.k_packed ? p->total_k : p->Sk;
  const int64_t* sq_list[] = {p->q_stride, p->o_stride, p->do_stride, p->dq_stride};
  for (const int64_t* st : sq_list)
    if (!strides_ok(st, m.q_packed, p->B, p->H, nq)) return cudaErrorInvalidValue;
  const int64_t* sk_list[] = {p->k_stride, p->v_stride, p->dk_stride, p->dv_stride};
  for (const int64_t* st : sk_list)
    if (!strides_ok(st, m.k_packed, p->B, p->H, nk)) return cudaErrorInvalidValue;
  if (p->bias && (!aligned16(p->bias) || !bias_strides_ok(p->bias_stride, p->B, p->H, p->Sq, true)))
    return cudaErrorInvalidValue;
  if (p->dbias &&
      (!aligned16(p->dbias) || !bias_strides_ok(p->dbias_stride, p->B, p->H, p->Sq, false)))
    return cudaErrorInvalidValue;

  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  return on_stream_device(stream, [&](int dev, const DeviceInfo& info) -> cudaError_t {
    attn::BwdArgs a;
    std::memset(&a, 0, sizeof(a));
    const void* qbase = rows_q > 0 ? p->q : p->k;
    const void* dobase = rows_q > 0 ? p->dout : p->k;
    const void* kbase = rows_k > 0 ? p->k : p->q;
    const void* vbase = rows_k > 0 ? p->v : p->q;
    const int Dv = p->Dv ? p->Dv : p->D;
    cudaError_t e = make_map(&a.tq, qbase, p->D, nq, p->H, p->B, p->q_stride, m.q_packed);
    if (e == cudaSuccess)
      e = make_map(&a.tdo, dobase, Dv, nq, p->H, p->B, p->do_stride, m.q_packed);
    if (e == cudaSuccess) e = make_map(&a.tk, kbase, p->D, nk, p->H, p->B, p->k_stride, m.k_packed);
    if (e == cudaSuccess) e = make_map(&a.tv, vbase, Dv, nk, p->H, p->B, p->v_stride, m.k_packed);
    if (e != cudaSuccess) return e;
    a.o = p->o;
    a.dout = p->dout;
    a.lse = p->lse;
    a.dq = p->dq;
    a.dk = p->dk;
    a.dv = p->dv;
    for (int i = 0; i < 3; ++i) {
      a.o_stride[i] = p->o_stride[i];
      a.do_stride[i] = p->do_stride[i];
      a.dq_stride[i] = p->dq_stride[i];
      a.dk_stride[i] = p->dk_stride[i];
      a.dv_stride[i] = p->dv_stride[i];
    }
    a.cu_q = p->cu_seqlens_q;
    a.cu_k = p->cu_seqlens_k;
    a.B = p->B;
    a.H = p->H;
    a.Sq = p->Sq;
    a.Sk = p->Sk;
    a.D = p->D;
    a.D16 = (p->D + 15) / 16 * 16;
    a.Dv = Dv;
    a.Dv16 = (Dv + 15) / 16 * 16;
    a.wl = p->window_left;
    a.wr = p->window_right;
    a.bottom_right = m.bottom_right;
    a.q_packed = m.q_packed;
    a.k_packed = m.k_packed;
    a.q_padded = m.q_padded;
    a.k_padded = m.k_padded;
    a.q_used = m.q_used;
    a.k_used = m.k_used;
    a.q_offsets = m.q_offsets;
    a.k_offsets = m.k_offsets;
    a.used_q = p->seqused_q;
    a.used_k = p->seqused_k;
    a.lse_th = m.lse_th;
    a.bf16 = p->dtype == ATTN_DTYPE_BF16;
    a.total_q = p->total_q;
    a.total_k = p->total_k;
    a.rows = rows_q;
    a.DA = (p->D + 7) / 8 * 8;
    a.sm_scale = p->sm_scale;
    // c = sm_scale * log2(e); the kernel subtracts LSE*log2(e)/c inside the
    // S^T product, so |c| is kept at least 2^-100.  Below that c * S^T is far
    // under the rounding of LSE*log2(e) and P is unchanged in fp32.
    a.scale_log2 = p->sm_scale * 1.4426950408889634f;
    if (std::fabs(a.scale_log2) < 0x1p-100f) a.scale_log2 = std::signbit(a.scale_log2) ? -0x1p-100f : 0x1p-100f;
    a.delta = static_cast<float*>(p->workspace);
    a.dq_acc = reinterpret_cast<float*>(static_cast<uint8_t*>(p->workspace) + wl.delta_bytes);
    a.order = wl.order_bytes ? reinterpret_cast<int32_t*>(static_cast<uint8_t*>(p->workspace) +
                                                          wl.delta_bytes + wl.acc_bytes)
                             : nullptr;
    e = make_dq_map(&a.tdq, a.dq_acc, p->D, a.DA, (int64_t)p->H * rows_q);
    if (e != cudaSuccess) return e;
    a.status = info.status;
    a.dev = dev;
    a.sms = info.sms;
    set_dropout(a, p);
    a.bias = p->bias;
    a.dbias = p->dbias;
    for (int i = 0; i < 3; ++i) {
      a.bias_stride[i] = p->bias_stride[i];
      a.dbias_stride[i] = p->dbias_stride[i];
    }
    if (p->bias) {
      e = make_bias_map(&a.tb, p->bias, p->Sq, p->Sk, p->H, p->B, p->bias_stride, &a.bias_h_bcast,
                        &a.bias_b_bcast);
      if (e != cudaSuccess) return e;
    }
    a.main_events[0] = static_cast<cudaEvent_t>(p->main_kernel_events[0]);
    a.main_events[1] = static_cast<cudaEvent_t>(p->main_kernel_events[1]);
    return attn::launch_bwd(a, stream);
  });
}

int64_t attn_allowed_pairs(int32_t seqlen_q, int32_t seqlen_k, int32_t window_left,
                           int32_t window_right, uint32_t bottom_right) {
  if (seqlen_q <= 0 || seqlen_k <= 0 || seqlen_q >= attn::kBig || seqlen_k >= attn::kBig) return 0;
  const attn::SeqWindow w =
      attn::seq_window(window_left, window_right, bottom_right != 0, seqlen_q, seqlen_k);
  int64_t total = 0;
  for (int32_t i = 0; i < seqlen_q; ++i) {
    const int32_t lo = attn::row_lo(w, i), hi = attn::row_hi(w, i, seqlen_k);
    if (hi >= lo) total += hi - lo + 1;
  }
  return total;
}

int attn_tile_plan(int32_t seqlen_q, int32_t seqlen_k, int32_t window_left, int32_t window_right,
                   uint32_t bottom_right, int32_t m0, int32_t* n_begin, int32_t* n_end,
                   uint8_t* full_mask) {
  if (!n_begin || !n_end || seqlen_q < 0 || seqlen_k < 0 || seqlen_q >= attn::kBig ||
      seqlen_k >= attn::kBig || m0 < 0)
    return cudaErrorInvalidValue;
  const attn::SeqWindow w =
      attn::seq_window(window_left, window_right, bottom_right != 0, seqlen_q, seqlen_k);
  attn::fwd_tile_range(w, seqlen_q, seqlen_k, m0, attn::kTileM, n_begin, n_end);
  if (full_mask)
    for (int32_t n = *n_begin; n < *n_end; ++n)
      full_mask[n - *n_begin] =
          attn::tile_is_full(w, seqlen_q, seqlen_k, m0, n * attn::kTileN) ? 1 : 0;
  return cudaSuccess;
}

int attn_tile_plan_bwd(int32_t seqlen_q, int32_t seqlen_k, int32_t window_left,
                       int32_t window_right, uint32_t bottom_right, int32_t n0, int32_t* m_begin,
                       int32_t* m_end) {
  if (!m_begin || !m_end || seqlen_q < 0 || seqlen_k < 0 || seqlen_q >= attn::kBig ||
      seqlen_k >= attn::kBig || n0 < 0)
    return cudaErrorInvalidValue;
  const attn::SeqWindow w =
      attn::seq_window(window_left, window_right, bottom_right != 0, seqlen_q, seqlen_k);
  attn::bwd_tile_range(w, seqlen_q, seqlen_k, n0, m_begin, m_end);
  return cudaSuccess;
}

int attn_device_status(void* stream_ptr, uint32_t* status) {
  if (!status) return cudaErrorInvalidValue;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  return on_stream_device(stream, [&](int, const DeviceInfo& info) -> cudaError_t {
    uint32_t host = 0;
    cudaError_t e = cudaMemcpyAsync(&host, info.status, 4, cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return e;
    *status = host;
    e = cudaMemsetAsync(info.status, 0, 4, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    return e;
  });
}

}  // extern "C"
