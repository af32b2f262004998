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

// Per-device facts, filled once under a lock: is it sm_100, and where is its
// copy of the status word.
struct DeviceInfo {
  bool ready = false;
  bool sm100 = false;
  uint32_t* status = nullptr;
};
std::mutex g_dev_mu;
DeviceInfo g_dev[kMaxDevices];

cudaError_t device_info(int dev, DeviceInfo* out) {
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    int major = 0, minor = 0;
    cudaError_t e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e != cudaSuccess) return e;
    d.sm100 = (major == 10 && minor == 0);
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_status);  // current device == dev here
    if (e != cudaSuccess) return e;
    d.status = static_cast<uint32_t*>(p);
    d.ready = true;
  }
  *out = d;
  return cudaSuccess;
}

// Runs `fn` with the stream's device current, restoring the caller's device.
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
  if (e == cudaSuccess) e = info.sm100 ? fn(info) : cudaErrorNoKernelImageForDevice;
  if (dev != cur) cudaSetDevice(cur);
  return e;
}

constexpr uint32_t kReservedBits = 0xFFF80000u;  // bits 31:19
constexpr uint32_t kModeReserved = 0xE0u;        // bits 7:5 of a VarlenMode

// Addressing of each side (Q: Q, O, LSE, dO, dQ; K: K, V, dK, dV).
struct Mode {
  bool q_packed, k_packed;  // 1THD with cumulative lengths
  bool q_padded, k_padded;  // BHSD with per-batch lengths
  bool lse_th;
  bool bottom_right;
};

bool decode_bits(uint32_t bits, Mode* m) {
  if (bits & kReservedBits) return false;
  const uint32_t qm = bits & 0xFFu, km = (bits >> 8) & 0xFFu, lse = (bits >> 16) & 3u;
  if ((qm | km) & kModeReserved) return false;
  auto known = [](uint32_t x) {
    return x == ATTN_VARLEN_MODE_DENSE || x == ATTN_VARLEN_MODE_PACKED || x == ATTN_VARLEN_MODE_PADDED;
  };
  if (!known(qm) || !known(km)) return false;  // each side on its own: dense, packed or padded
  if (lse > 1) return false;
  m->q_packed = (qm == ATTN_VARLEN_MODE_PACKED);
  m->k_packed = (km == ATTN_VARLEN_MODE_PACKED);
  m->q_padded = (qm == ATTN_VARLEN_MODE_PADDED);
  m->k_padded = (km == ATTN_VARLEN_MODE_PADDED);
  m->lse_th = (lse == ATTN_LSE_TH);
  m->bottom_right = ((bits >> 18) & 1u) != 0;
  return true;
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

cudaError_t make_map(CUtensorMap* map, const void* base, int D, int64_t rows, int H, int B,
                     const int64_t* st, bool packed) {
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
  cuuint32_t box[4] = {64, 128, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 4, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// 2-D fp32 map over the dQ accumulator [H*rows][D] (row pitch D*4 bytes),
// 32 x 32 boxes with 128-byte swizzle: the backward adds staged dQ tiles
// through it.
cudaError_t make_dq_map(CUtensorMap* map, float* base, int D, int64_t rows_total) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)(rows_total > 0 ? rows_total : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)D * 4};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Checks shared by forward and backward.
template <class P>
bool common_ok(const P* p, size_t want_size, Mode* m, bool check_pointers = true) {
  if (!p || p->struct_size != want_size || p->version != ATTN_PARAMS_VERSION) return false;
  if (p->dtype != ATTN_DTYPE_FP16 && p->dtype != ATTN_DTYPE_BF16) return false;
  if (p->D < 16 || p->D > 128 || (p->D % 16) != 0) return false;
  if (p->B < 0 || p->H < 0 || p->Sq < 0 || p->Sk < 0) return false;
  if (p->Sq >= attn::kBig || p->Sk >= attn::kBig) return false;
  if (!std::isfinite(p->sm_scale)) return false;
  if (!decode_bits(p->varlen_bits, m)) return false;
  if (m->q_packed && (p->total_q < 0 || p->total_q >= attn::kBig)) return false;
  if (m->k_packed && (p->total_k < 0 || p->total_k >= attn::kBig)) return false;
  // Packed and padded sides read their lengths from the device arrays.
  if (check_pointers && p->B > 0) {
    if ((m->q_packed || m->q_padded) && !p->cu_seqlens_q) return false;
    if ((m->k_packed || m->k_padded) && !p->cu_seqlens_k) return false;
  }
  return true;
}

bool has_work(int B, int H, int64_t rows_q) { return B > 0 && H > 0 && rows_q > 0; }

}  // namespace

extern "C" {

int attn_fwd(const attn_fwd_params* p, void* stream_ptr) {
  Mode m;
  if (!common_ok(p, sizeof(attn_fwd_params), &m)) return cudaErrorInvalidValue;
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

  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  return on_stream_device(stream, [&](const DeviceInfo& info) -> cudaError_t {
    attn::FwdArgs a;
    std::memset(&a, 0, sizeof(a));
    const void* kbase = rows_k > 0 ? p->k : p->q;
    const void* vbase = rows_k > 0 ? p->v : p->q;
    cudaError_t e = make_map(&a.tq, p->q, p->D, nq, p->H, p->B, p->q_stride, m.q_packed);
    if (e == cudaSuccess) e = make_map(&a.tk, kbase, p->D, nk, p->H, p->B, p->k_stride, m.k_packed);
    if (e == cudaSuccess) e = make_map(&a.tv, vbase, p->D, nk, p->H, p->B, p->v_stride, m.k_packed);
    if (e != cudaSuccess) return e;
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
    a.wl = p->window_left;
    a.wr = p->window_right;
    a.bottom_right = m.bottom_right;
    a.q_packed = m.q_packed;
    a.k_packed = m.k_packed;
    a.q_padded = m.q_padded;
    a.k_padded = m.k_padded;
    a.lse_th = m.lse_th;
    a.bf16 = p->dtype == ATTN_DTYPE_BF16;
    a.negate = p->sm_scale < 0.f;
    a.total_q = p->total_q;
    a.scale_log2 = std::fabs(p->sm_scale) * 1.4426950408889634f;
    a.status = info.status;
    return attn::launch_fwd(a, stream);
  });
}

size_t attn_bwd_workspace_size(const attn_bwd_params* p) {
  Mode m;
  if (!common_ok(p, sizeof(attn_bwd_params), &m, /*check_pointers=*/false)) return 0;
  const int64_t rows = m.q_packed ? p->total_q : (int64_t)p->B * p->Sq;
  const int64_t n = (int64_t)p->H * rows;
  const size_t delta_bytes = ((size_t)n * 4 + 255) & ~(size_t)255;
  return delta_bytes + (size_t)n * p->D * 4;
}

int attn_bwd(const attn_bwd_params* p, void* stream_ptr) {
  Mode m;
  if (!common_ok(p, sizeof(attn_bwd_params), &m)) return cudaErrorInvalidValue;
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
  const size_t ws = attn_bwd_workspace_size(p);
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

  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  return on_stream_device(stream, [&](const DeviceInfo& info) -> cudaError_t {
    attn::BwdArgs a;
    std::memset(&a, 0, sizeof(a));
    const void* qbase = rows_q > 0 ? p->q : p->k;
    const void* dobase = rows_q > 0 ? p->dout : p->k;
    const void* kbase = rows_k > 0 ? p->k : p->q;
    const void* vbase = rows_k > 0 ? p->v : p->q;
    cudaError_t e = make_map(&a.tq, qbase, p->D, nq, p->H, p->B, p->q_stride, m.q_packed);
    if (e == cudaSuccess)
      e = make_map(&a.tdo, dobase, p->D, nq, p->H, p->B, p->do_stride, m.q_packed);
    if (e == cudaSuccess) e = make_map(&a.tk, kbase, p->D, nk, p->H, p->B, p->k_stride, m.k_packed);
    if (e == cudaSuccess) e = make_map(&a.tv, vbase, p->D, nk, p->H, p->B, p->v_stride, m.k_packed);
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
    a.wl = p->window_left;
    a.wr = p->window_right;
    a.bottom_right = m.bottom_right;
    a.q_packed = m.q_packed;
    a.k_packed = m.k_packed;
    a.q_padded = m.q_padded;
    a.k_padded = m.k_padded;
    a.lse_th = m.lse_th;
    a.bf16 = p->dtype == ATTN_DTYPE_BF16;
    a.total_q = p->total_q;
    a.rows = rows_q;
    a.sm_scale = p->sm_scale;
    // c = sm_scale * log2(e); the kernel subtracts LSE*log2(e)/c inside the
    // S^T product, so |c| is kept at least 2^-100.  Below that c * S^T is far
    // under the rounding of LSE*log2(e) and P is unchanged in fp32.
    a.scale_log2 = p->sm_scale * 1.4426950408889634f;
    if (std::fabs(a.scale_log2) < 0x1p-100f) a.scale_log2 = std::signbit(a.scale_log2) ? -0x1p-100f : 0x1p-100f;
    const size_t delta_bytes = ((size_t)p->H * rows_q * 4 + 255) & ~(size_t)255;
    a.delta = static_cast<float*>(p->workspace);
    a.dq_acc = reinterpret_cast<float*>(static_cast<uint8_t*>(p->workspace) + delta_bytes);
    e = make_dq_map(&a.tdq, a.dq_acc, p->D, (int64_t)p->H * rows_q);
    if (e != cudaSuccess) return e;
    a.status = info.status;
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
  return on_stream_device(stream, [&](const DeviceInfo& info) -> cudaError_t {
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
