// kvq_inst.cuh -- host-side launchers for the kernels of one vector length d.
// Included by exactly one translation unit per d (kvq_d64.cu, ...), which
// explicitly instantiates launch_fwd<d>, launch_inv<d>, launch_decode<d> and
// read_status<d>.
#pragma once

#include <algorithm>
#include <mutex>
#include <utility>

#include "kvq_codec.cuh"
#include "kvq_attn.cuh"
#include "kvq_wide.cuh"
#include "kvq_launch.h"

namespace kvq {

// Status word of this translation unit's kernels, one per device context.
// Bit 0: a bounded wait on an asynchronous copy ran out.
static __device__ unsigned g_status;

// Per-(d, rotation, direction) launch tuning: pipeline depth (tiles in
// flight per warp), output tiles in flight, and the minimum resident blocks
// per SM the register allocation must allow.  Chosen from same-box sweeps on
// the B200 (the d = 256 SRFT inverse keeps a third block despite a small
// spill: it measured faster than two blocks without one).
#ifndef KVQ_INV_STAGES_64
#define KVQ_INV_STAGES_64 2
#endif
#ifndef KVQ_INV_STAGES_BIG
#define KVQ_INV_STAGES_BIG 2
#endif
#ifndef KVQ_SOUT_BIG
#define KVQ_SOUT_BIG 1
#endif
#ifndef KVQ_SOUT_64
#define KVQ_SOUT_64 2
#endif
// d = 64 SRFT 4-bit inverse with one scale per vector (g = 64): one output
// tile in flight measured faster (88% against 85% of the copy peak, same
// box); g = 32 measured slower (87% against 89%), SRHT the same.
#ifndef KVQ_INV_SOUT_64_G64
#define KVQ_INV_SOUT_64_G64 1
#endif
#ifndef KVQ_ATTN_MAX_CLUSTER
#define KVQ_ATTN_MAX_CLUSTER 16
#endif
// Decode attention with one scale per token (g = d) and at most 4 queries
// per KV head on the tensor cores (1) or on the FP32 pipes (0)...
#ifndef KVQ_ATTN_TC
#define KVQ_ATTN_TC 1
#endif
// ... and at d = g = 64 with one query per KV head (instead of the lane-pair
// kernel).
#ifndef KVQ_ATTN_TC_64
#define KVQ_ATTN_TC_64 0
#endif
#ifndef KVQ_ATTN_PAIR_TOKENS
#define KVQ_ATTN_PAIR_TOKENS 8
#endif
#ifndef KVQ_ATTN_ROWS_PER_WARP
#define KVQ_ATTN_ROWS_PER_WARP 4
#endif
#ifndef KVQ_FWD_MINB_64
#define KVQ_FWD_MINB_64 5
#endif
#ifndef KVQ_INV_MINB_64
#define KVQ_INV_MINB_64 4
#endif
#ifndef KVQ_MINB_128_SRFT
#define KVQ_MINB_128_SRFT 3
#endif
#ifndef KVQ_FWD_MINB_256_SRFT
#define KVQ_FWD_MINB_256_SRFT 3
#endif
#ifndef KVQ_INV_MINB_256_SRFT
#define KVQ_INV_MINB_256_SRFT 3
#endif

template <int D, int ROT>
struct Tuning {
  static constexpr int TPV = DefaultTPV<D>::value;
  static constexpr int FWD_STAGES = 2;
  static constexpr int INV_STAGES = D == 64 ? KVQ_INV_STAGES_64 : KVQ_INV_STAGES_BIG;
  static constexpr int S_OUT = D == 64 ? KVQ_SOUT_64 : KVQ_SOUT_BIG;
  static constexpr bool SRFT = ROT == kRotSRFT;
  template <int G, bool LAM, int BITS>
  static constexpr int INV_S_OUT =
      D == 64 && G == 64 && SRFT && !LAM && BITS == 4 ? KVQ_INV_SOUT_64_G64 : S_OUT;
  static constexpr int FWD_MINB =
      D == 64 ? (SRFT ? KVQ_FWD_MINB_64 : 4) : (D == 128 ? (SRFT ? KVQ_MINB_128_SRFT : 3)
                                        : (SRFT ? KVQ_FWD_MINB_256_SRFT : 3));
  static constexpr int INV_MINB =
      D == 64 ? KVQ_INV_MINB_64 : (D == 128 ? (SRFT ? KVQ_MINB_128_SRFT : 2)
                                        : (SRFT ? KVQ_INV_MINB_256_SRFT : 3));
};

namespace detail {

constexpr int kMaxDevices = 64;

inline cudaError_t current_device(int* dev) {
  cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return e;
  return (*dev >= 0 && *dev < kMaxDevices) ? cudaSuccess : cudaErrorInvalidDevice;
}

// Device address of g_status on the current device (looked up once).
inline cudaError_t status_ptr(unsigned** out) {
  static unsigned* ptrs[kMaxDevices];
  static std::mutex mu;
  int dev;
  cudaError_t e = current_device(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> g(mu);
  if (ptrs[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_status);
    if (e != cudaSuccess) return e;
    ptrs[dev] = static_cast<unsigned*>(p);
  }
  *out = ptrs[dev];
  return cudaSuccess;
}

// Opt the kernel into its dynamic shared memory and look up how many blocks
// fit on one SM, once per kernel and device.
template <auto Kern>
cudaError_t setup(int smem, int* occ_out) {
  static int occ[kMaxDevices];
  static std::mutex mu;
  int dev;
  cudaError_t e = current_device(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> g(mu);
  if (occ[dev] == 0) {
    e = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int b = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, Kern, kThreads, smem);
    if (e != cudaSuccess) return e;
    occ[dev] = std::max(b, 1);
  }
  *occ_out = occ[dev];
  return cudaSuccess;
}

// Launch attribute of the decode-path kernels: programmatic stream
// serialization, so that a kernel's blocks can be scheduled while the
// previous kernel of the stream drains (the kernels wait for it with
// griddepcontrol.wait before touching global memory).
inline void pdl_attribute(cudaLaunchAttribute& at) {
  at.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at.val.programmaticStreamSerializationAllowed = KVQ_PDL ? 1 : 0;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), int grid, int threads, int smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(grid), 1, 1);
  cfg.blockDim = dim3(unsigned(threads), 1, 1);
  cfg.dynamicSmemBytes = size_t(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  pdl_attribute(attr[0]);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  return e == cudaSuccess ? cudaGetLastError() : e;
}

inline int grid_for(int64_t n_tiles, int sm_count, int occ) {
  const int64_t want = (n_tiles + kWarps - 1) / kWarps;
  return int(std::max<int64_t>(1, std::min<int64_t>(want, int64_t(sm_count) * occ)));
}

template <int D, int G, int ROT, bool LAM, int BITS = 4>
cudaError_t fwd_run(const FwdLaunch& L) {
  using T = Tuning<D, ROT>;
  constexpr auto kern =
      kvq_fwd_kernel<D, G, ROT, T::TPV, T::FWD_STAGES, T::S_OUT, T::FWD_MINB, LAM, BITS>;
  constexpr int smem = fwd_smem_bytes<D, ROT, T::TPV, T::FWD_STAGES, T::S_OUT, BITS>();
  int occ;
  unsigned* st;
  cudaError_t e = setup<kern>(smem, &occ);
  if (e == cudaSuccess) e = status_ptr(&st);
  if (e != cudaSuccess) return e;
  constexpr int vpw = 32 / T::TPV;
  FwdArgs a{L.signs, L.lambda, L.scales, L.n_vec, (L.n_vec + vpw - 1) / vpw};
  kern<<<grid_for(a.n_tiles, L.sm_count, occ), kThreads, smem, L.stream>>>(*L.tmX, *L.tmQ, a, st);
  return cudaGetLastError();
}

template <int D, int G, int ROT>
cudaError_t fwd_one(const FwdLaunch& L) {
  if (L.bits != 4) {
    // other code widths: no lambda; rows of d*bits/8 bytes (3 bits needs d >= 128)
    if (L.bits == 8) return fwd_run<D, G, ROT, false, 8>(L);
    if (L.bits == 6) return fwd_run<D, G, ROT, false, 6>(L);
    if constexpr (D >= 128) {
      if (L.bits == 3) return fwd_run<D, G, ROT, false, 3>(L);
    }
    return cudaErrorInvalidValue;
  }
  return L.lambda ? fwd_run<D, G, ROT, true>(L) : fwd_run<D, G, ROT, false>(L);
}

template <int D, int G, int ROT, bool LAM, int BITS = 4>
cudaError_t inv_run(const InvLaunch& L) {
  using T = Tuning<D, ROT>;
  constexpr auto kern =
      kvq_inv_kernel<D, G, ROT, T::TPV, T::INV_STAGES, T::template INV_S_OUT<G, LAM, BITS>,
                     T::INV_MINB, LAM, BITS>;
  constexpr int smem =
      inv_smem_bytes<D, G, ROT, T::TPV, T::INV_STAGES, T::template INV_S_OUT<G, LAM, BITS>,
                     BITS>();
  int occ;
  unsigned* st;
  cudaError_t e = setup<kern>(smem, &occ);
  if (e == cudaSuccess) e = status_ptr(&st);
  if (e != cudaSuccess) return e;
  constexpr int vpw = 32 / T::TPV;
  InvArgs a{L.signs, L.lambda, L.n_vec, (L.n_vec + vpw - 1) / vpw};
  kern<<<grid_for(a.n_tiles, L.sm_count, occ), kThreads, smem, L.stream>>>(*L.tmQ, *L.tmS,
                                                                             *L.tmX, a, st);
  return cudaGetLastError();
}

template <int D, int G, int ROT>
cudaError_t inv_one(const InvLaunch& L) {
  if (L.bits != 4) {
    if (L.bits == 8) return inv_run<D, G, ROT, false, 8>(L);
    if (L.bits == 6) return inv_run<D, G, ROT, false, 6>(L);
    if constexpr (D >= 128) {
      if (L.bits == 3) return inv_run<D, G, ROT, false, 3>(L);
    }
    return cudaErrorInvalidValue;
  }
  return L.lambda ? inv_run<D, G, ROT, true>(L) : inv_run<D, G, ROT, false>(L);
}

template <int D, int G, int ROT>
cudaError_t decode_one(const DecodeLaunch& L) {
  using T = Tuning<D, ROT>;
  constexpr auto kern = kvq_decode_kernel<D, G, ROT, T::TPV, T::INV_STAGES, 1>;
  constexpr int smem = decode_smem_bytes<D, ROT, T::TPV, T::INV_STAGES>();
  int occ;
  unsigned* st;
  cudaError_t e = setup<kern>(smem, &occ);
  if (e == cudaSuccess) e = status_ptr(&st);
  if (e != cudaSuccess) return e;
  constexpr int vpw = 32 / T::TPV;
  DecodeArgs a;
  a.signs = L.signs;
  a.scales = L.scales;
  a.n_heads = L.n_heads;
  a.cap = L.cap;
  a.pos = L.pos;
  a.n_new_tiles = (L.n_heads + vpw - 1) / vpw;
  a.tok_tiles = (L.pos + vpw - 1) / vpw;
  a.n_tiles = a.n_new_tiles + L.n_heads * a.tok_tiles;
  return launch_pdl(kern, grid_for(a.n_tiles, L.sm_count, occ), kThreads, smem, L.stream,
                    *L.tmXn, *L.tmQn, *L.tmOn, *L.tmQc, *L.tmOc, a, st);
}

// Resident kWideThreads-thread blocks per SM of a one-warp-per-vector kernel
// (cached per device).
template <auto Kern>
cudaError_t wide_occupancy(int* occ_out) {
  static int occ[kMaxDevices];
  static std::mutex mu;
  int dev;
  cudaError_t e = current_device(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> g(mu);
  if (occ[dev] == 0) {
    int b = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, Kern, kWideThreads, 0);
    if (e != cudaSuccess) return e;
    occ[dev] = std::max(b, 1);
  }
  *occ_out = occ[dev];
  return cudaSuccess;
}

inline int wide_grid(int64_t rows, int sm_count, int occ) {
  const int64_t want = (rows + kWideThreads / 32 - 1) / (kWideThreads / 32);
  return int(std::max<int64_t>(1, std::min<int64_t>(want, int64_t(sm_count) * occ)));
}

template <int D, int G, int ROT>
cudaError_t decode_wide_one(const DecodeWideLaunch& L) {
  constexpr auto kern = kvq_decode_wide_kernel<D, G, ROT>;
  int occ;
  cudaError_t e = wide_occupancy<kern>(&occ);
  if (e != cudaSuccess) return e;
  DecodeWideArgs a{L.x_new, L.packed, L.scales, L.out, L.signs, L.n_heads, L.cap, L.pos,
                   wide_pos_recip(L.pos)};
  return launch_pdl(kern, wide_grid(L.n_heads * (L.pos + 1), L.sm_count, occ), kWideThreads, 0,
                    L.stream, a);
}

template <int D, int G, int ROT>
cudaError_t window_one(const WindowLaunch& L) {
  constexpr auto kern = kvq_window_wide_kernel<D, G, ROT>;
  int occ;
  cudaError_t e = wide_occupancy<kern>(&occ);
  if (e != cudaSuccess) return e;
  WindowArgs a{L.x_new, L.packed, L.scales, L.kv, L.signs, L.n_heads, L.cap, L.pos, L.window};
  const bool flush = (L.pos + 1) % L.window == 0;
  const int64_t rows = flush ? L.n_heads * L.window : L.n_heads;
  return launch_pdl(kern, wide_grid(rows, L.sm_count, occ), kWideThreads, 0, L.stream, a);
}

// Largest cluster (blocks per KV head) the attention kernel `Kern` may use on
// the current device: up to 16 where the device can co-schedule them, else 8
// (looked up once per kernel and device; also opts the kernel into its
// dynamic shared memory).
template <auto Kern>
cudaError_t attn_max_cluster(int smem, int* out) {
  static int maxc[kMaxDevices];
  static std::mutex mu;
  int dev;
  cudaError_t e = current_device(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> g(mu);
  if (maxc[dev] == 0) {
    e = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    static_assert(KVQ_ATTN_MAX_CLUSTER <= kAttnMaxCluster, "attention merge weights");
    int c = std::min(8, KVQ_ATTN_MAX_CLUSTER);
    if (cudaFuncSetAttribute(Kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
        cudaSuccess) {
      cudaLaunchConfig_t q = {};
      q.gridDim = dim3(16, 1, 1);
      q.blockDim = dim3(kAttnThreads, 1, 1);
      q.dynamicSmemBytes = smem;
      int best = 0;
      if (cudaOccupancyMaxPotentialClusterSize(&best, Kern, &q) == cudaSuccess && best >= 8)
        c = std::min(std::min(best, 16), KVQ_ATTN_MAX_CLUSTER);
    }
    cudaGetLastError();
    maxc[dev] = c;
  }
  *out = maxc[dev];
  return cudaSuccess;
}

// The largest cluster size c <= limit (c >= 1) for which `need` clusters of
// c blocks are co-resident on the device (one wave), per the occupancy
// calculator: a cluster must fit in one GPC, so the SMs alone do not decide
// (e.g. 8 clusters of 16 blocks on 148 SMs take two waves).  Answers are
// cached per device, kernel and size.
template <auto Kern, int THREADS = kAttnThreads>
cudaError_t attn_fit_cluster(int smem, int limit, int64_t need, int* out) {
  static int maxact[kMaxDevices][kAttnMaxCluster + 1];  // 0: not asked yet
  static std::mutex mu;
  int dev;
  cudaError_t e = current_device(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> g(mu);
  int c = std::max(1, std::min(limit, kAttnMaxCluster));
  for (; c > 1; --c) {
    if (maxact[dev][c] == 0) {
      cudaLaunchConfig_t q = {};
      q.gridDim = dim3(unsigned(c), 1, 1);
      q.blockDim = dim3(THREADS, 1, 1);
      q.dynamicSmemBytes = smem;
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = unsigned(c);
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      q.attrs = &attr;
      q.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, Kern, &q) != cudaSuccess) {
        cudaGetLastError();
        n = -1;  // not placeable: never chosen
      }
      maxact[dev][c] = n > 0 ? n : -1;
    }
    if (maxact[dev][c] >= need) break;
  }
  *out = c;
  return cudaSuccess;
}

// One cluster of `cl` blocks per KV head.
template <typename... KArgs>
cudaError_t attn_launch(void (*kern)(KArgs...), int cl, int smem, const AttnLaunch& L,
                        const AttnArgs& a, int64_t grid_y = 0) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(cl), unsigned(grid_y > 0 ? grid_y : L.n_kv), 1);
  cfg.blockDim = dim3(kAttnThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = L.stream;
  cudaLaunchAttribute attr[2];
  pdl_attribute(attr[0]);
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = unsigned(cl);
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cl > 1 ? 2 : 1;  // a one-block cluster needs no cluster launch
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a);
  return e == cudaSuccess ? cudaGetLastError() : e;
}

// d = 64 with one query per KV head: the lane-pair kernel, about
// KVQ_ATTN_PAIR_TOKENS tokens per pair and block, up to two blocks per SM.
template <int D, int ROT>
cudaError_t attn_pair(int group, const AttnLaunch& L) {
  constexpr auto kern = kvq_attn_pair_kernel<D, ROT>;
  constexpr int smem = attn_pair_smem_bytes<D>();
  int max_cluster;
  cudaError_t e = attn_max_cluster<kern>(smem, &max_cluster);
  if (e != cudaSuccess) return e;
  constexpr int64_t per_block = int64_t(kAttnThreads / 2) * KVQ_ATTN_PAIR_TOKENS;
  const int64_t by_len = (L.len + per_block - 1) / per_block;
  const int64_t by_sms = std::max<int64_t>(1, 2 * int64_t(L.sm_count) / std::max<int64_t>(1, L.n_kv));
  int cl = int(std::max<int64_t>(
      1, std::min<int64_t>(max_cluster, std::min<int64_t>(by_len, by_sms))));
  e = attn_fit_cluster<kern>(smem, cl, L.n_kv, &cl);
  if (e != cudaSuccess) return e;
  AttnArgs a{L.q, L.k_packed, L.k_scales, L.v_packed, L.v_scales, L.out, L.signs, L.cap, L.len,
             L.nq, group, L.sm_scale * float(Wide<D, ROT>::KAPPA_D) * kLog2e};
  return attn_launch(kern, cl, smem, L, a);
}

template <int D, int ROT, int NQ>
cudaError_t attn_nq(int group, const AttnLaunch& L) {
  constexpr auto kern = kvq_attn_kernel<D, ROT, NQ>;
  constexpr int smem = attn_smem_bytes<D, NQ>();
  int max_cluster;
  cudaError_t e = attn_max_cluster<kern>(smem, &max_cluster);
  if (e != cudaSuccess) return e;
  // blocks per KV head (one cluster): about KVQ_ATTN_ROWS_PER_WARP rows per
  // warp, and no more than the SMs left per head (one resident block per SM)
  constexpr int64_t per_block = int64_t(kAttnWarps) * KVQ_ATTN_ROWS_PER_WARP;
  const int64_t by_len = (L.len + per_block - 1) / per_block;
  const int64_t by_sms = std::max<int64_t>(1, L.sm_count / std::max<int64_t>(1, L.n_kv));
  int cl = int(std::max<int64_t>(
      1, std::min<int64_t>(max_cluster, std::min<int64_t>(by_len, by_sms))));
  e = attn_fit_cluster<kern>(smem, cl, L.n_kv, &cl);
  if (e != cudaSuccess) return e;
  AttnArgs a{L.q, L.k_packed, L.k_scales, L.v_packed, L.v_scales, L.out, L.signs, L.cap, L.len,
             L.nq, group, L.sm_scale * float(Wide<D, ROT>::KAPPA_D) * kLog2e};
  return attn_launch(kern, cl, smem, L, a);
}

// g = d with at most 8 queries per KV head: the tensor-core kernel, about 32
// tokens per warp and block, one resident block per SM.  Each grid row is a
// (KV head, group of 4 queries) pair; the two groups of a head run side by
// side, so the second one reads the head's codes mostly from L2.
template <int D, int ROT, bool QG>
cudaError_t attn_tc(const AttnLaunch& L) {
  constexpr auto kern = kvq_attn_tc_kernel<D, ROT, QG>;
  constexpr int smem = attn_tc_smem_bytes<D>();
  int max_cluster;
  cudaError_t e = attn_max_cluster<kern>(smem, &max_cluster);
  if (e != cudaSuccess) return e;
  const int qgroups = (L.nq + 3) / 4;
  const int64_t rows = L.n_kv * qgroups;
  constexpr int64_t per_block = int64_t(kAttnWarps) * 2 * kTcChunk;
  const int64_t by_len = (L.len + per_block - 1) / per_block;
  const int64_t by_sms = std::max<int64_t>(1, L.sm_count / std::max<int64_t>(1, rows));
  int cl = int(std::max<int64_t>(
      1, std::min<int64_t>(max_cluster, std::min<int64_t>(by_len, by_sms))));
  e = attn_fit_cluster<kern>(smem, cl, rows, &cl);
  if (e != cudaSuccess) return e;
  AttnArgs a{L.q,      L.k_packed, L.k_scales, L.v_packed,
             L.v_scales, L.out,    L.signs,    L.cap,
             L.len,    L.nq,       D,          L.sm_scale * float(Wide<D, ROT>::KAPPA_D) * kLog2e,
             qgroups};
  return attn_launch(kern, cl, smem, L, a, rows);
}

template <int D, int ROT>
cudaError_t attn_rot(int group, const AttnLaunch& L) {
  if constexpr (D == 64) {
    if (L.nq == 1 && !(KVQ_ATTN_TC_64 && group == 64)) return attn_pair<D, ROT>(group, L);
  }
  if (KVQ_ATTN_TC && group == D && L.nq <= 4) return attn_tc<D, ROT, false>(L);
  if (KVQ_ATTN_TC && group == D && L.n_kv <= 32767)  // grid rows <= 65535
    return attn_tc<D, ROT, true>(L);
  if (L.nq <= 1) return attn_nq<D, ROT, 1>(group, L);
  if (L.nq <= 2) return attn_nq<D, ROT, 2>(group, L);
  if (L.nq <= 4) return attn_nq<D, ROT, 4>(group, L);
  return attn_nq<D, ROT, 8>(group, L);
}

// Run Op<D, G, ROT>(launch) for the runtime (group, rot) pair.
template <int D, template <int, int, int> class Op, class L>
cudaError_t dispatch(int group, int rot, const L& l) {
  auto by_rot = [&](auto gc) -> cudaError_t {
    constexpr int G = decltype(gc)::value;
    if constexpr (G > D) {
      return cudaErrorInvalidValue;
    } else {
      return rot == kRotSRFT ? Op<D, G, kRotSRFT>::run(l) : Op<D, G, kRotSRHT>::run(l);
    }
  };
  switch (group) {
    case 32: return by_rot(std::integral_constant<int, 32>{});
    case 64: return by_rot(std::integral_constant<int, 64>{});
    case 128: return by_rot(std::integral_constant<int, 128>{});
    case 256: return by_rot(std::integral_constant<int, 256>{});
    default: return cudaErrorInvalidValue;
  }
}

template <int D, int G, int ROT>
struct FwdOp {
  static cudaError_t run(const FwdLaunch& l) { return fwd_one<D, G, ROT>(l); }
};
template <int D, int G, int ROT>
struct InvOp {
  static cudaError_t run(const InvLaunch& l) { return inv_one<D, G, ROT>(l); }
};
template <int D, int G, int ROT>
struct DecodeOp {
  static cudaError_t run(const DecodeLaunch& l) { return decode_one<D, G, ROT>(l); }
};
template <int D, int G, int ROT>
struct DecodeWideOp {
  static cudaError_t run(const DecodeWideLaunch& l) { return decode_wide_one<D, G, ROT>(l); }
};
template <int D, int G, int ROT>
struct WindowOp {
  static cudaError_t run(const WindowLaunch& l) { return window_one<D, G, ROT>(l); }
};

}  // namespace detail

template <int D>
cudaError_t launch_fwd(int group, int rot, const FwdLaunch& L) {
  return detail::dispatch<D, detail::FwdOp>(group, rot, L);
}

template <int D>
cudaError_t launch_inv(int group, int rot, const InvLaunch& L) {
  return detail::dispatch<D, detail::InvOp>(group, rot, L);
}

template <int D>
cudaError_t launch_decode(int group, int rot, const DecodeLaunch& L) {
  return detail::dispatch<D, detail::DecodeOp>(group, rot, L);
}

template <int D>
cudaError_t launch_decode_wide(int group, int rot, const DecodeWideLaunch& L) {
  return detail::dispatch<D, detail::DecodeWideOp>(group, rot, L);
}

template <int D>
cudaError_t launch_window(int group, int rot, const WindowLaunch& L) {
  return detail::dispatch<D, detail::WindowOp>(group, rot, L);
}

template <int D>
cudaError_t launch_attn(int group, int rot, const AttnLaunch& L) {
  return rot == kRotSRFT ? detail::attn_rot<D, kRotSRFT>(group, L)
                         : detail::attn_rot<D, kRotSRHT>(group, L);
}

template <int D>
cudaError_t read_status(uint32_t* value, bool clear) {
  unsigned v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_status, sizeof(v));
  if (e != cudaSuccess) return e;
  if (clear && v != 0) {
    const unsigned z = 0;
    e = cudaMemcpyToSymbol(g_status, &z, sizeof(z));
    if (e != cudaSuccess) return e;
  }
  *value = v;
  return cudaSuccess;
}

}  // namespace kvq
