// kvq_api.cu -- the C ABI of libkvq: argument checks, TMA descriptors,
// dispatch to the per-d kernels.  Declarations and contracts: include/kvq.h.
#include <cuda.h>
#include <cmath>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "kvq.h"
#include "kvq_launch.h"

namespace {

using kvq::vpw_of;

constexpr int kMaxDevices = 64;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

kvq_status check_shape(int32_t d, int32_t group, kvq_rot rot) {
  if (rot != KVQ_ROT_SRFT && rot != KVQ_ROT_SRHT) return KVQ_ERR_BAD_ROT;
  if (d != 64 && d != 128 && d != 256) return KVQ_ERR_BAD_DIM;
  if ((group != 32 && group != 64 && group != 128 && group != 256) || group > d)
    return KVQ_ERR_BAD_GROUP;
  return KVQ_OK;
}

// Per-device facts, looked up once: SM count and whether the device is
// compute capability 10.0 (the only one this sm_100a build runs on).
struct DeviceInfo {
  int sm_count = 0;
  bool ok = false;
};

kvq_status device_info(DeviceInfo* out) {
  static DeviceInfo info[kMaxDevices];
  static bool done[kMaxDevices];
  static std::mutex mu;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
  std::lock_guard<std::mutex> g(mu);
  if (!done[dev]) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return KVQ_ERR_CUDA;
    }
    info[dev].sm_count = sms;
    info[dev].ok = (major == 10 && minor == 0);
    done[dev] = true;
  }
  *out = info[dev];
  return info[dev].ok ? KVQ_OK : KVQ_ERR_UNSUPPORTED_DEVICE;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    cudaGetLastError();
  });
  return fn;
}

// Tiled tensor map: dims/box innermost first; strides in bytes for dims 1..
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, uint32_t rank, const void* base,
              const uint64_t* dims, const uint64_t* strides, const uint32_t* box,
              CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const uint32_t es[5] = {1, 1, 1, 1, 1};
  uint64_t dummy = 16;
  return fn(m, dt, rank, const_cast<void*>(base), dims, rank > 1 ? strides : &dummy, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

CUtensorMapSwizzle code_swizzle(int d) {
  return d == 64 ? CU_TENSOR_MAP_SWIZZLE_32B
                 : (d == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
}

// fp16 rows [rows][d] with row pitch `pitch` bytes, box {64, VPW}.
bool map_x(CUtensorMap* m, const void* base, int d, uint64_t rows, uint64_t pitch) {
  const uint64_t dims[2] = {uint64_t(d), rows};
  const uint64_t strides[1] = {pitch};
  const uint32_t box[2] = {64, uint32_t(vpw_of(d))};
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, base, dims, strides, box,
                  CU_TENSOR_MAP_SWIZZLE_128B);
}

// packed-code rows [rows][d/2] with row pitch `pitch` bytes, box {d/2, VPW}.
// codes of other widths: rows of d*bits/8 bytes, moved as slabs of 128, 64
// or 32 bytes with the matching swizzle (one unswizzled box for 48-byte rows);
// must agree with Cfg::SW in kvq_codec.cuh.
bool map_qb(CUtensorMap* m, const void* base, int d, int bits, uint64_t rows) {
  const uint64_t qp = uint64_t(d) * uint64_t(bits) / 8;
  const uint32_t sw = qp % 128 == 0 ? 128 : (qp % 64 == 0 ? 64 : (qp % 32 == 0 ? 32 : 0));
  const CUtensorMapSwizzle mode = sw == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : sw == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                  : sw == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                             : CU_TENSOR_MAP_SWIZZLE_NONE;
  const uint64_t dims[2] = {qp, rows};
  const uint64_t strides[1] = {qp};
  const uint32_t box[2] = {sw ? sw : uint32_t(qp), uint32_t(vpw_of(d))};
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, mode);
}

bool map_q(CUtensorMap* m, const void* base, int d, uint64_t rows, uint64_t pitch) {
  const uint64_t dims[2] = {uint64_t(d / 2), rows};
  const uint64_t strides[1] = {pitch};
  const uint32_t box[2] = {uint32_t(d / 2), uint32_t(vpw_of(d))};
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, code_swizzle(d));
}

// scales as one flat f32 array of `count` elements, box {VPW * d/g}.
bool map_s(CUtensorMap* m, const void* base, int d, int group, uint64_t count) {
  const uint64_t dims[1] = {count};
  const uint32_t box[1] = {uint32_t(vpw_of(d) * (d / group))};
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 1, base, dims, nullptr, box,
                  CU_TENSOR_MAP_SWIZZLE_NONE);
}

kvq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA; }

constexpr int64_t kMaxRows = (int64_t(1) << 31) - 1;

bool bits_ok(int32_t d, int32_t bits) {
  return bits == 4 || bits == 6 || bits == 8 || (bits == 3 && d >= 128);
}

kvq_status rot_quant_fwd(const uint16_t* x, int64_t n_vec, int32_t d, int32_t group,
                         const int8_t* signs, const float* lambda, kvq_rot rot, uint8_t* packed,
                         float* scales, kvq_stream stream, int32_t bits = 4) {
  if (kvq_status s = check_shape(d, group, rot)) return s;
  if (!bits_ok(d, bits)) return KVQ_ERR_BAD_BITS;
  if (n_vec < 0 || n_vec > kMaxRows) return KVQ_ERR_BAD_SIZE;
  if (!x || !signs || !packed || !scales) return KVQ_ERR_NULL;
  if (!aligned(x, 16) || !aligned(packed, 16) || !aligned(scales, 16) ||
      (lambda && !aligned(lambda, 8)))
    return KVQ_ERR_MISALIGNED;
  if (n_vec == 0) return KVQ_OK;
  DeviceInfo dev;
  if (kvq_status s = device_info(&dev)) return s;
  CUtensorMap tmX, tmQ;
  if (!map_x(&tmX, x, d, uint64_t(n_vec), uint64_t(2 * d)) ||
      !(bits == 4 ? map_q(&tmQ, packed, d, uint64_t(n_vec), uint64_t(d / 2))
                  : map_qb(&tmQ, packed, d, bits, uint64_t(n_vec))))
    return KVQ_ERR_CUDA;
  kvq::FwdLaunch L{&tmX, &tmQ, signs, lambda, bits, scales, n_vec, dev.sm_count,
                   reinterpret_cast<cudaStream_t>(stream)};
  cudaError_t e = d == 64    ? kvq::launch_fwd<64>(group, rot, L)
                  : d == 128 ? kvq::launch_fwd<128>(group, rot, L)
                             : kvq::launch_fwd<256>(group, rot, L);
  return from_cuda(e);
}

kvq_status dequant_rot_inv(const uint8_t* packed, const float* scales, int64_t n_vec, int32_t d,
                           int32_t group, const int8_t* signs, const float* lambda, kvq_rot rot,
                           uint16_t* out, kvq_stream stream, int32_t bits = 4) {
  if (kvq_status s = check_shape(d, group, rot)) return s;
  if (!bits_ok(d, bits)) return KVQ_ERR_BAD_BITS;
  if (n_vec < 0 || n_vec > kMaxRows || n_vec * (d / group) > kMaxRows) return KVQ_ERR_BAD_SIZE;
  if (!packed || !scales || !signs || !out) return KVQ_ERR_NULL;
  if (!aligned(packed, 16) || !aligned(scales, 16) || !aligned(out, 16) ||
      (lambda && !aligned(lambda, 8)))
    return KVQ_ERR_MISALIGNED;
  if (n_vec == 0) return KVQ_OK;
  DeviceInfo dev;
  if (kvq_status s = device_info(&dev)) return s;
  CUtensorMap tmQ, tmS, tmX;
  if (!(bits == 4 ? map_q(&tmQ, packed, d, uint64_t(n_vec), uint64_t(d / 2))
                  : map_qb(&tmQ, packed, d, bits, uint64_t(n_vec))) ||
      !map_s(&tmS, scales, d, group, uint64_t(n_vec) * uint64_t(d / group)) ||
      !map_x(&tmX, out, d, uint64_t(n_vec), uint64_t(2 * d)))
    return KVQ_ERR_CUDA;
  kvq::InvLaunch L{&tmQ, &tmS, &tmX, signs, lambda, bits, n_vec, dev.sm_count,
                   reinterpret_cast<cudaStream_t>(stream)};
  cudaError_t e = d == 64    ? kvq::launch_inv<64>(group, rot, L)
                  : d == 128 ? kvq::launch_inv<128>(group, rot, L)
                             : kvq::launch_inv<256>(group, rot, L);
  return from_cuda(e);
}

}  // namespace

extern "C" {

kvq_status kvq_rot_quant_fwd(const uint16_t* x, int64_t n_vec, int32_t d, int32_t group,
                             const int8_t* signs, kvq_rot rot, uint8_t* packed, float* scales,
                             kvq_stream stream) {
  return rot_quant_fwd(x, n_vec, d, group, signs, nullptr, rot, packed, scales, stream);
}

kvq_status kvq_dequant_rot_inv(const uint8_t* packed, const float* scales, int64_t n_vec,
                               int32_t d, int32_t group, const int8_t* signs, kvq_rot rot,
                               uint16_t* out, kvq_stream stream) {
  return dequant_rot_inv(packed, scales, n_vec, d, group, signs, nullptr, rot, out, stream);
}

kvq_status kvq_rot_quant_fwd_lambda(const uint16_t* x, int64_t n_vec, int32_t d, int32_t group,
                                    const int8_t* signs, const float* lambda, kvq_rot rot,
                                    uint8_t* packed, float* scales, kvq_stream stream) {
  if (!lambda) return KVQ_ERR_NULL;
  return rot_quant_fwd(x, n_vec, d, group, signs, lambda, rot, packed, scales, stream);
}

kvq_status kvq_dequant_rot_inv_lambda(const uint8_t* packed, const float* scales, int64_t n_vec,
                                      int32_t d, int32_t group, const int8_t* signs,
                                      const float* lambda, kvq_rot rot, uint16_t* out,
                                      kvq_stream stream) {
  if (!lambda) return KVQ_ERR_NULL;
  return dequant_rot_inv(packed, scales, n_vec, d, group, signs, lambda, rot, out, stream);
}

kvq_status kvq_rot_quant_fwd_bits(const uint16_t* x, int64_t n_vec, int32_t d, int32_t group,
                                  int32_t bits, const int8_t* signs, kvq_rot rot, uint8_t* packed,
                                  float* scales, kvq_stream stream) {
  return rot_quant_fwd(x, n_vec, d, group, signs, nullptr, rot, packed, scales, stream, bits);
}

kvq_status kvq_dequant_rot_inv_bits(const uint8_t* packed, const float* scales, int64_t n_vec,
                                    int32_t d, int32_t group, int32_t bits, const int8_t* signs,
                                    kvq_rot rot, uint16_t* out, kvq_stream stream) {
  return dequant_rot_inv(packed, scales, n_vec, d, group, signs, nullptr, rot, out, stream, bits);
}

kvq_status kvq_decode_step(const uint16_t* x_new, uint8_t* packed, float* scales,
                           int64_t n_heads, int64_t cap, int64_t pos, int32_t d, int32_t group,
                           const int8_t* signs, kvq_rot rot, uint16_t* out, kvq_stream stream) {
  if (kvq_status s = check_shape(d, group, rot)) return s;
  if (n_heads < 0 || n_heads > kMaxRows || cap < 1 || cap > kMaxRows || pos < 0 || pos >= cap)
    return KVQ_ERR_BAD_SIZE;
  const int64_t ng = d / group;
  if (n_heads * cap > kMaxRows || n_heads * cap * ng > kMaxRows ||
      n_heads * (pos + 1) > kMaxRows)
    return KVQ_ERR_BAD_SIZE;
  if (!x_new || !packed || !scales || !signs || !out) return KVQ_ERR_NULL;
  if (!aligned(x_new, 16) || !aligned(packed, 16) || !aligned(scales, 4) || !aligned(out, 16))
    return KVQ_ERR_MISALIGNED;
  if (n_heads == 0) return KVQ_OK;
  DeviceInfo dev;
  if (kvq_status s = device_info(&dev)) return s;
  if (n_heads * (pos + 1) <= kvq::kWideMaxRows) {  // latency path: a warp per vector
    kvq::DecodeWideLaunch W{x_new, packed, scales, out, signs, n_heads, cap, pos, dev.sm_count,
                            reinterpret_cast<cudaStream_t>(stream)};
    cudaError_t e = d == 64    ? kvq::launch_decode_wide<64>(group, rot, W)
                    : d == 128 ? kvq::launch_decode_wide<128>(group, rot, W)
                               : kvq::launch_decode_wide<256>(group, rot, W);
    return from_cuda(e);
  }
  const uint64_t qp = uint64_t(d / 2), xp = uint64_t(2 * d);
  const uint64_t H = uint64_t(n_heads), CAP = uint64_t(cap), P = uint64_t(pos);
  CUtensorMap tmXn, tmQn, tmOn, tmQc, tmOc;
  bool ok = map_x(&tmXn, x_new, d, H, xp) &&
            map_q(&tmQn, packed + P * qp, d, H, CAP * qp) &&
            map_x(&tmOn, out + P * uint64_t(d), d, H, (P + 1) * xp);
  {
    const uint64_t dims[3] = {qp, CAP, H};
    const uint64_t strides[2] = {qp, CAP * qp};
    const uint32_t box[3] = {uint32_t(d / 2), uint32_t(vpw_of(d)), 1};
    ok = ok && make_map(&tmQc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, packed, dims, strides, box,
                        code_swizzle(d));
  }
  if (pos > 0) {
    const uint64_t dims[3] = {uint64_t(d), P, H};
    const uint64_t strides[2] = {xp, (P + 1) * xp};
    const uint32_t box[3] = {64, uint32_t(vpw_of(d)), 1};
    ok = ok && make_map(&tmOc, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, out, dims, strides, box,
                        CU_TENSOR_MAP_SWIZZLE_128B);
  } else {
    tmOc = tmOn;  // no cached rows: never used
  }
  if (!ok) return KVQ_ERR_CUDA;
  kvq::DecodeLaunch L{&tmXn,  &tmQn,   &tmOn, &tmQc, &tmOc,        signs,
                      scales, n_heads, cap,   pos,   dev.sm_count, reinterpret_cast<cudaStream_t>(stream)};
  cudaError_t e = d == 64    ? kvq::launch_decode<64>(group, rot, L)
                  : d == 128 ? kvq::launch_decode<128>(group, rot, L)
                             : kvq::launch_decode<256>(group, rot, L);
  return from_cuda(e);
}

kvq_status kvq_decode_step_windowed(const uint16_t* x_new, uint8_t* packed, float* scales,
                                    uint16_t* kv, int64_t n_heads, int64_t cap, int64_t pos,
                                    int32_t window, int32_t d, int32_t group, const int8_t* signs,
                                    kvq_rot rot, kvq_stream stream) {
  if (kvq_status s = check_shape(d, group, rot)) return s;
  if (n_heads < 0 || n_heads > kMaxRows || cap < 1 || cap > kMaxRows || pos < 0 || pos >= cap ||
      window < 1 || window > 4096)
    return KVQ_ERR_BAD_SIZE;
  const int64_t ng = d / group;
  if (n_heads * cap > kMaxRows || n_heads * cap * ng > kMaxRows ||
      n_heads * int64_t(window) > kMaxRows)
    return KVQ_ERR_BAD_SIZE;
  if (!x_new || !packed || !scales || !kv || !signs) return KVQ_ERR_NULL;
  if (!aligned(x_new, 16) || !aligned(packed, 16) || !aligned(scales, 4) || !aligned(kv, 16))
    return KVQ_ERR_MISALIGNED;
  if (n_heads == 0) return KVQ_OK;
  DeviceInfo dev;
  if (kvq_status s = device_info(&dev)) return s;
  kvq::WindowLaunch W{x_new, packed, scales, kv, signs, n_heads, cap, pos, window, dev.sm_count,
                      reinterpret_cast<cudaStream_t>(stream)};
  cudaError_t e = d == 64    ? kvq::launch_window<64>(group, rot, W)
                  : d == 128 ? kvq::launch_window<128>(group, rot, W)
                             : kvq::launch_window<256>(group, rot, W);
  return from_cuda(e);
}

kvq_status kvq_attend_decode(const uint16_t* q, const uint8_t* k_packed, const float* k_scales,
                             const uint8_t* v_packed, const float* v_scales, int64_t n_kv_heads,
                             int32_t n_q, int64_t cap, int64_t len, int32_t d, int32_t group,
                             const int8_t* signs, kvq_rot rot, float sm_scale, uint16_t* out,
                             kvq_stream stream) {
  if (kvq_status s = check_shape(d, group, rot)) return s;
  if (n_kv_heads < 0 || n_kv_heads > 65535 || n_q < 1 || n_q > 8 || cap < 1 || cap > kMaxRows ||
      len < 1 || len > cap || !std::isfinite(sm_scale))
    return KVQ_ERR_BAD_SIZE;
  const int64_t ng = d / group;
  if (n_kv_heads * cap * ng > kMaxRows || n_kv_heads * cap > kMaxRows) return KVQ_ERR_BAD_SIZE;
  if (!q || !k_packed || !k_scales || !v_packed || !v_scales || !signs || !out)
    return KVQ_ERR_NULL;
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(k_packed, 16) || !aligned(v_packed, 16) ||
      !aligned(k_scales, 4) || !aligned(v_scales, 4))
    return KVQ_ERR_MISALIGNED;
  if (n_kv_heads == 0) return KVQ_OK;
  DeviceInfo dev;
  if (kvq_status s = device_info(&dev)) return s;
  kvq::AttnLaunch A{q,   k_packed, k_scales, v_packed,     v_scales,
                    out, signs,    n_kv_heads, cap,        len,
                    n_q, sm_scale, dev.sm_count, reinterpret_cast<cudaStream_t>(stream)};
  cudaError_t e = d == 64    ? kvq::launch_attn<64>(group, rot, A)
                  : d == 128 ? kvq::launch_attn<128>(group, rot, A)
                             : kvq::launch_attn<256>(group, rot, A);
  return from_cuda(e);
}

const char* kvq_status_string(kvq_status s) {
  switch (s) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_NULL: return "a required pointer is NULL";
    case KVQ_ERR_BAD_DIM: return "d must be 64, 128 or 256";
    case KVQ_ERR_BAD_GROUP: return "group must be 32, 64, 128 or 256 and not larger than d";
    case KVQ_ERR_MISALIGNED: return "a pointer is not 16-byte aligned";
    case KVQ_ERR_BAD_ROT: return "rot must be KVQ_ROT_SRFT or KVQ_ROT_SRHT";
    case KVQ_ERR_CUDA: return "CUDA runtime error while enqueueing";
    case KVQ_ERR_BAD_SIZE: return "count or position out of range";
    case KVQ_ERR_DEVICE_TIMEOUT: return "a kernel timed out waiting for its own copy";
    case KVQ_ERR_UNSUPPORTED_DEVICE: return "device is not compute capability 10.0 (sm_100a)";
    case KVQ_ERR_BAD_BITS: return "bits must be 3 (d >= 128), 4, 6 or 8";
  }
  return "unknown status";
}

kvq_status kvq_device_status(int32_t clear) {
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
  uint32_t v64 = 0, v128 = 0, v256 = 0;
  if (kvq::read_status<64>(&v64, clear != 0) != cudaSuccess ||
      kvq::read_status<128>(&v128, clear != 0) != cudaSuccess ||
      kvq::read_status<256>(&v256, clear != 0) != cudaSuccess) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
  return (v64 | v128 | v256) ? KVQ_ERR_DEVICE_TIMEOUT : KVQ_OK;
}

int32_t kvq_version(void) { return 100; }

}  // extern "C"
