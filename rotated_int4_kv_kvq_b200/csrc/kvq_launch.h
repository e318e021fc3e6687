// kvq_launch.h -- internal interface between the C-ABI front end (kvq_api.cu)
// and the per-d kernel translation units (kvq_d64.cu, kvq_d128.cu,
// kvq_d256.cu).  Not part of the public API.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kvq {

// Threads per vector and vectors per warp tile for each d (must match the
// kernels' DefaultTPV).
constexpr int tpv_of(int d) { return d >= 256 ? 2 : 1; }
constexpr int vpw_of(int d) { return 32 / tpv_of(d); }

struct FwdLaunch {
  const CUtensorMap* tmX;  // x      [n_vec][d] fp16, box {64, VPW}, swizzle 128B
  const CUtensorMap* tmQ;  // packed [n_vec][d/2] u8, box {d/2, VPW}, swizzle = pitch
  const int8_t* signs;
  const float* lambda;     // per-channel factors [d] or NULL
  int bits;                // code width (3, 4, 6, 8); tmQ row pitch d*bits/8
  float* scales;
  int64_t n_vec;
  int sm_count;
  cudaStream_t stream;
};

struct InvLaunch {
  const CUtensorMap* tmQ;  // packed, as above
  const CUtensorMap* tmS;  // scales as 1-D f32, box {VPW * d/g}
  const CUtensorMap* tmX;  // out, as x above
  const int8_t* signs;
  const float* lambda;     // per-channel factors [d] or NULL
  int bits;                // code width (3, 4, 6, 8)
  int64_t n_vec;
  int sm_count;
  cudaStream_t stream;
};

// Decode calls with at most this many rows (new tokens + cached rows) run
// the one-warp-per-vector kernel (latency); larger ones the tiled kernel.
#ifndef KVQ_WIDE_MAX_ROWS
#define KVQ_WIDE_MAX_ROWS (int64_t(1) << 16)
#endif
constexpr int64_t kWideMaxRows = KVQ_WIDE_MAX_ROWS;
// The one-warp-per-vector kernel maps rows with 32-bit reciprocal
// multiplies that are exact for at most 2^16 rows per call.
static_assert(kWideMaxRows <= (int64_t(1) << 16), "wide decode calls are limited to 2^16 rows");

struct DecodeWideLaunch {
  const uint16_t* x_new;
  uint8_t* packed;
  float* scales;
  uint16_t* out;
  const int8_t* signs;
  int64_t n_heads, cap, pos;
  int sm_count;
  cudaStream_t stream;
};

struct WindowLaunch {
  const uint16_t* x_new;  // [n_heads][d]
  uint8_t* packed;        // [n_heads][cap][d/2]
  float* scales;          // [n_heads][cap][d/g]
  uint16_t* kv;           // [n_heads][cap][d]
  const int8_t* signs;
  int64_t n_heads, cap, pos;
  int window;
  int sm_count;
  cudaStream_t stream;
};

struct AttnLaunch {
  const uint16_t* q;        // [n_kv][nq][d]
  const uint8_t* k_packed;  // [n_kv][cap][d/2]
  const float* k_scales;    // [n_kv][cap][d/g]
  const uint8_t* v_packed;
  const float* v_scales;
  uint16_t* out;            // [n_kv][nq][d]
  const int8_t* signs;
  int64_t n_kv, cap, len;
  int nq;
  float sm_scale;
  int sm_count;
  cudaStream_t stream;
};

struct DecodeLaunch {
  const CUtensorMap* tmXn;  // x_new [n_heads][d], box {64, VPW}
  const CUtensorMap* tmQn;  // packed row pos of every head, box {d/2, VPW}
  const CUtensorMap* tmOn;  // out row pos of every head, box {64, VPW}
  const CUtensorMap* tmQc;  // packed cache 3-D {d/2, cap, n_heads}, box {d/2, VPW, 1}
  const CUtensorMap* tmOc;  // out rows < pos 3-D {d, pos, n_heads}, box {64, VPW, 1}
  const int8_t* signs;
  float* scales;
  int64_t n_heads, cap, pos;
  int sm_count;
  cudaStream_t stream;
};

// Implemented once per d in the matching translation unit.
template <int D>
cudaError_t launch_fwd(int group, int rot, const FwdLaunch& L);
template <int D>
cudaError_t launch_inv(int group, int rot, const InvLaunch& L);
template <int D>
cudaError_t launch_decode(int group, int rot, const DecodeLaunch& L);
template <int D>
cudaError_t launch_decode_wide(int group, int rot, const DecodeWideLaunch& L);
template <int D>
cudaError_t launch_window(int group, int rot, const WindowLaunch& L);
// group is a runtime argument of the attention kernel.
template <int D>
cudaError_t launch_attn(int group, int rot, const AttnLaunch& L);
// Reads (and optionally clears) the device status word of that translation
// unit on the current device; the caller has synchronized the device.
template <int D>
cudaError_t read_status(uint32_t* value, bool clear);

}  // namespace kvq
