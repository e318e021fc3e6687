// kvq_wide.cuh -- one warp per vector: the latency-oriented engine of the
// decode step.
//
// A decode call touches few vectors (the new token of each head plus the
// cached rows of a layer), so its time is the length of one vector's
// dependency chain, not bandwidth.  Here a whole warp works on one vector:
// lane l holds W = d/32 values and every step is a handful of instructions
// per lane plus five shuffle stages.
//
// SRHT: lane l holds x[W l .. W l + W); in-lane Walsh-Hadamard over the low
// index bits, then one shuffle butterfly per lane bit.  y stays in natural
// order.
//
// SRFT: z_n = u_{2n} + i u_{2n+1}, N = d/2 points, C = N/32 per lane, lane l
// holds z_{l + 32 n1} (n1 < C).  Four-step FFT: in-lane DFT_C over n1,
// twiddle W_N^{l k1}, then a 32-point decimation-in-frequency FFT across the
// lanes (shuffle with lane ^ b, b = 16 .. 1).  Lane l ends with
// Z_{k1 + C k2} for k2 = bitrev5(l), so it owns the C consecutive outputs
// X_k, k in [C k2, C k2 + C), i.e. the chunk y[W k2 .. W k2 + W) of the
// packed spectrum.  The real split pairs Z_k with Z_{N-k}: for k1 >= 1 the
// partner sits in lane l ^ 31, register C - k1; for k1 = 0 in lane
// bitrev5(-k2 mod 32), register 0.  Scaling: the unnormalized packed
// spectrum is Y = 2X (y = KAPPA Y), and the inverse takes Yin = KAPPA y_hat,
// KAPPA = 1/sqrt(2d) both ways.
#pragma once

#include "kvq_device.cuh"

namespace kvq {

constexpr float kSqrt2Wide = 1.41421356237309504880f;
// Blocks of 4 warps: a short call (a few hundred rows) spreads over more SMs
// with at most one warp per scheduler, which shortens each row's latency.
constexpr int kWideThreads = 128;

// exp(-2 pi i j / 256) for j < 256, rounded once from double.
struct Tw256 {
  float c[256];
  float s[256];
};

constexpr Tw256 make_tw256() {
  Tw256 t{};
  for (int j = 0; j < 256; ++j) {
    const CS v = cos_sin_2pi(j, 256);
    t.c[j] = float(v.c);
    t.s[j] = float(-v.s);
  }
  return t;
}

// Global memory, read through the read-only path: every lane looks up its own
// twiddle, which a constant-bank table would serialize 32 ways.
static __device__ const Tw256 kTw256 = make_tw256();

// exp(-2 pi i j / n) as an (re, im) pair; n divides 256.
__device__ __forceinline__ f2 tw_fwd(int j, int n) {
  const int k = (j % n) * (256 / n);
  return mk2(__ldg(&kTw256.c[k]), __ldg(&kTw256.s[k]));
}

__device__ __forceinline__ int bitrev5(int l) { return __brev(unsigned(l)) >> 27; }

// a * w (complex)
__device__ __forceinline__ f2 cmulw(f2 a, f2 w) {
  const float ar = lo2(a), ai = hi2(a), wr = lo2(w), wi = hi2(w);
  return mk2(fmaf(ar, wr, -(ai * wi)), fmaf(ar, wi, ai * wr));
}

// a * conj(w)
__device__ __forceinline__ f2 cmulwc(f2 a, f2 w) {
  const float ar = lo2(a), ai = hi2(a), wr = lo2(w), wi = hi2(w);
  return mk2(fmaf(ar, wr, ai * wi), fmaf(ai, wr, -(ar * wi)));
}

__device__ __forceinline__ f2 shfl_idx2(f2 a, int src) {
  return mk2(__shfl_sync(kFull, lo2(a), src), __shfl_sync(kFull, hi2(a), src));
}

template <int D, int ROT>
struct Wide {
  static constexpr int W = D / 32;  // reals per lane
  static constexpr int C = W / 2;   // complex points (or words) per lane
  static constexpr int N = D / 2;   // SRFT complex length
  static constexpr double KAPPA_D =
      ROT == kRotSRFT ? 1.0 / const_sqrt(2.0 * D) : 1.0 / const_sqrt(double(D));
  static constexpr float KAPPA = float(KAPPA_D);
  static constexpr float KAPPA7 = float(KAPPA_D / 7.0);
};

// Per-lane constants, computed once per warp.
template <int D, int ROT>
struct WideLane {
  using P = Wide<D, ROT>;
  int lane;
  int k2;                // chunk of y this lane owns (bitrev5(lane) for SRFT)
  uint32_t mask[P::C];   // fp16 sign masks of the lane's words
  f2 st[5];              // SRFT: DIF stage twiddles (b = 16 >> s), 1 on clear lanes
  f2 s2[P::C];           // SRFT: W_N^{lane k1}
  f2 post[P::C];         // SRFT: (cos, sin)(2 pi k / d) for k = k1 + C k2
  int src0;              // SRFT: lane holding the partner of k1 = 0

  __device__ __forceinline__ void init(const int8_t* signs, int l) {
    lane = l;
    k2 = ROT == kRotSRFT ? bitrev5(l) : l;
#pragma unroll
    for (int j = 0; j < P::C; ++j) {
      // SRFT: word l + 32 j; SRHT: word C l + j
      const int w = ROT == kRotSRFT ? l + 32 * j : P::C * l + j;
      mask[j] = (signs[2 * w] < 0 ? 0x00008000u : 0u) | (signs[2 * w + 1] < 0 ? 0x80000000u : 0u);
    }
    if constexpr (ROT == kRotSRFT) {
#pragma unroll
      for (int s = 0; s < 5; ++s) {
        const int b = 16 >> s;
        st[s] = (l & b) ? tw_fwd(l & (b - 1), 2 * b) : mk2(1.0f, 0.0f);
      }
#pragma unroll
      for (int k1 = 0; k1 < P::C; ++k1) {
        s2[k1] = tw_fwd(l * k1, P::N);
        const f2 t = tw_fwd(k1 + P::C * k2, D);
        post[k1] = mk2(lo2(t), -hi2(t));  // (cos, sin)
      }
      src0 = bitrev5((32 - k2) & 31);
    }
  }
};

// In-lane DFT of C points (forward sign for INV = false), natural order.
template <int C, bool INV>
__device__ __forceinline__ void dft_small(f2 (&z)[C]) {
  if constexpr (C == 2) {
    const f2 a = z[0], b = z[1];
    z[0] = add2(a, b);
    z[1] = sub2(a, b);
  } else if constexpr (C == 4) {
    const f2 t0 = add2(z[0], z[2]), t1 = sub2(z[0], z[2]);
    const f2 t2 = add2(z[1], z[3]), d = sub2(z[1], z[3]);
    // forward: t3 = -i d; inverse: +i d
    const f2 t3 = INV ? mk2(-hi2(d), lo2(d)) : mk2(hi2(d), -lo2(d));
    z[0] = add2(t0, t2);
    z[2] = sub2(t0, t2);
    z[1] = add2(t1, t3);
    z[3] = sub2(t1, t3);
  }
}

// Forward rotation: Y (the lane's W values of chunk k2, unnormalized,
// y = KAPPA * Y) from the lane's sign-flipped fp16 words.
template <int D, int ROT>
__device__ __forceinline__ void wide_rotate_fwd(const uint32_t (&xw)[Wide<D, ROT>::C],
                                                const WideLane<D, ROT>& L,
                                                float (&Y)[Wide<D, ROT>::W]) {
  using P = Wide<D, ROT>;
  if constexpr (ROT == kRotSRHT) {
    f2 v[P::C];
#pragma unroll
    for (int j = 0; j < P::C; ++j) {
      const float2 f = half2_bits_to_float2(xw[j]);
      v[j] = mk2(f.x, f.y);
    }
    fwht<P::C>(v);
#pragma unroll
    for (int b = 1; b < 32; b <<= 1) {
      const float sg = (L.lane & b) ? -1.0f : 1.0f;
      const f2 sg2 = mk2(sg, sg);
#pragma unroll
      for (int j = 0; j < P::C; ++j) v[j] = fma2(sg2, v[j], shfl_xor2(v[j], b));
    }
#pragma unroll
    for (int j = 0; j < P::C; ++j) {
      Y[2 * j] = lo2(v[j]);
      Y[2 * j + 1] = hi2(v[j]);
    }
  } else {
    f2 z[P::C];
#pragma unroll
    for (int j = 0; j < P::C; ++j) {
      const float2 f = half2_bits_to_float2(xw[j]);
      z[j] = mk2(f.x, f.y);
    }
    dft_small<P::C, false>(z);
#pragma unroll
    for (int k1 = 1; k1 < P::C; ++k1) z[k1] = cmulw(z[k1], L.s2[k1]);
#pragma unroll
    for (int s = 0; s < 5; ++s) {
      const int b = 16 >> s;
      const float sg = (L.lane & b) ? -1.0f : 1.0f;
      const f2 sg2 = mk2(sg, sg);
#pragma unroll
      for (int k1 = 0; k1 < P::C; ++k1)
        z[k1] = cmulw(fma2(sg2, z[k1], shfl_xor2(z[k1], b)), L.st[s]);
    }
    // real split: X'_k = S + W_d^k (-i T), S = A + conj B', T = A - conj B'
    f2 part[P::C];
    part[0] = shfl_idx2(z[0], L.src0);
#pragma unroll
    for (int k1 = 1; k1 < P::C; ++k1) part[k1] = shfl_xor2(z[P::C - k1], 31);
#pragma unroll
    for (int k1 = 0; k1 < P::C; ++k1) {
      const f2 p1 = add2(z[k1], part[k1]);  // (Sr, Ti)
      const f2 p2 = sub2(z[k1], part[k1]);  // (Tr, Si)
      const float sr = lo2(p1), ti = hi2(p1), tr = lo2(p2), si = hi2(p2);
      const float c = lo2(L.post[k1]), s = hi2(L.post[k1]);
      const float wr = fmaf(c, ti, -(s * tr)), wi = -fmaf(c, tr, s * ti);
      Y[2 * k1] = sr + wr;
      Y[2 * k1 + 1] = si + wi;
    }
    if (L.lane == 0) {  // k = 0: sqrt2 X_0 and sqrt2 X_{N} (both real)
      const float a = lo2(z[0]), b = hi2(z[0]);
      Y[0] = kSqrt2Wide * (a + b);
      Y[1] = kSqrt2Wide * (a - b);
    }
  }
}

// Inverse rotation: the lane's fp16 words (before the sign flip) of
// u = R^T y_hat from Yin = KAPPA * y_hat (the lane's chunk k2).
template <int D, int ROT>
__device__ __forceinline__ void wide_rotate_inv(const float (&Y)[Wide<D, ROT>::W],
                                                const WideLane<D, ROT>& L,
                                                uint32_t (&xw)[Wide<D, ROT>::C]) {
  using P = Wide<D, ROT>;
  if constexpr (ROT == kRotSRHT) {
    f2 v[P::C];
#pragma unroll
    for (int j = 0; j < P::C; ++j) v[j] = mk2(Y[2 * j], Y[2 * j + 1]);
#pragma unroll
    for (int b = 1; b < 32; b <<= 1) {
      const float sg = (L.lane & b) ? -1.0f : 1.0f;
      const f2 sg2 = mk2(sg, sg);
#pragma unroll
      for (int j = 0; j < P::C; ++j) v[j] = fma2(sg2, v[j], shfl_xor2(v[j], b));
    }
    fwht<P::C>(v);
#pragma unroll
    for (int j = 0; j < P::C; ++j) xw[j] = float2_to_half2_bits(lo2(v[j]), hi2(v[j]));
  } else {
    f2 x[P::C];
#pragma unroll
    for (int k1 = 0; k1 < P::C; ++k1) x[k1] = mk2(Y[2 * k1], Y[2 * k1 + 1]);
    f2 part[P::C];
    part[0] = shfl_idx2(x[0], L.src0);
#pragma unroll
    for (int k1 = 1; k1 < P::C; ++k1) part[k1] = shfl_xor2(x[P::C - k1], 31);
    f2 z[P::C];
#pragma unroll
    for (int k1 = 0; k1 < P::C; ++k1) {
      // Q_k = S + i W_d^{-k} D, S = A + conj B', D = A - conj B'
      const f2 p1 = add2(x[k1], part[k1]);  // (Sr, Di)
      const f2 p2 = sub2(x[k1], part[k1]);  // (Dr, Si)
      const float sr = lo2(p1), di = hi2(p1), dr = lo2(p2), si = hi2(p2);
      const float c = lo2(L.post[k1]), s = hi2(L.post[k1]);
      const float vr = fmaf(c, dr, -(s * di)), vi = fmaf(c, di, s * dr);
      z[k1] = mk2(sr - vi, si + vr);
    }
    if (L.lane == 0) {
      const float a = Y[0], b = Y[1];
      z[0] = mk2(kSqrt2Wide * (a + b), kSqrt2Wide * (a - b));
    }
    // inverse 32-point DFT across lanes: decimation in time on the
    // bit-reversed lane order, conjugate twiddles
#pragma unroll
    for (int s = 4; s >= 0; --s) {
      const int b = 16 >> s;
      const float sg = (L.lane & b) ? -1.0f : 1.0f;
      const f2 sg2 = mk2(sg, sg);
#pragma unroll
      for (int k1 = 0; k1 < P::C; ++k1) {
        const f2 v = cmulwc(z[k1], L.st[s]);
        z[k1] = fma2(sg2, v, shfl_xor2(v, b));
      }
    }
#pragma unroll
    for (int k1 = 1; k1 < P::C; ++k1) z[k1] = cmulwc(z[k1], L.s2[k1]);
    dft_small<P::C, true>(z);
#pragma unroll
    for (int j = 0; j < P::C; ++j) xw[j] = float2_to_half2_bits(lo2(z[j]), hi2(z[j]));
  }
}

// ------------------------------------------------------ decode kernel ---

struct DecodeWideArgs {
  const uint16_t* x_new;  // [n_heads][d]
  uint8_t* packed;        // [n_heads][cap][d/2]
  float* scales;          // [n_heads][cap][d/g]
  uint16_t* out;          // [n_heads][pos+1][d]
  const int8_t* signs;
  int64_t n_heads, cap, pos;
  uint32_t pos_recip;     // ceil(2^32 / pos) for pos >= 2 (wide_pos_recip)
};

// The multiplier that divides a cached-row index n < 2^16 by pos exactly:
// n / pos = umulhi(n, ceil(2^32 / pos)) for 2 <= pos <= 2^16 (checked for
// every such pos and n).  Computed once per call on the host.
inline uint32_t wide_pos_recip(int64_t pos) {
  return pos > 1 ? uint32_t(0xFFFFFFFFull / uint64_t(pos)) + 1u : 0u;
}

// Loads through the read-only path unless RO is false (rows this kernel
// also writes).
template <bool RO, class T>
__device__ __forceinline__ T wide_ld(const T* p) {
  if constexpr (RO) {
    return __ldg(p);
  } else {
    return *p;
  }
}

template <int D, int ROT, bool RO = true>
__device__ __forceinline__ void wide_load_words(const uint16_t* row, const WideLane<D, ROT>& L,
                                                uint32_t (&xw)[Wide<D, ROT>::C]) {
  using P = Wide<D, ROT>;
  const uint32_t* w = reinterpret_cast<const uint32_t*>(row);
  if constexpr (ROT == kRotSRFT) {
#pragma unroll
    for (int j = 0; j < P::C; ++j) xw[j] = wide_ld<RO>(w + L.lane + 32 * j) ^ L.mask[j];
  } else if constexpr (P::C == 4) {
    const uint4 v = wide_ld<RO>(reinterpret_cast<const uint4*>(w) + L.lane);
    xw[0] = v.x ^ L.mask[0];
    xw[1] = v.y ^ L.mask[1];
    xw[2] = v.z ^ L.mask[2];
    xw[3] = v.w ^ L.mask[3];
  } else if constexpr (P::C == 2) {
    const uint2 v = wide_ld<RO>(reinterpret_cast<const uint2*>(w) + L.lane);
    xw[0] = v.x ^ L.mask[0];
    xw[1] = v.y ^ L.mask[1];
  } else {
    xw[0] = wide_ld<RO>(w + L.lane) ^ L.mask[0];
  }
}

template <int D, int ROT>
__device__ __forceinline__ void wide_store_words(uint16_t* row, const WideLane<D, ROT>& L,
                                                 const uint32_t (&xw)[Wide<D, ROT>::C]) {
  using P = Wide<D, ROT>;
  uint32_t* w = reinterpret_cast<uint32_t*>(row);
  if constexpr (ROT == kRotSRFT) {
#pragma unroll
    for (int j = 0; j < P::C; ++j) w[L.lane + 32 * j] = xw[j] ^ L.mask[j];
  } else if constexpr (P::C == 4) {
    reinterpret_cast<uint4*>(w)[L.lane] =
        make_uint4(xw[0] ^ L.mask[0], xw[1] ^ L.mask[1], xw[2] ^ L.mask[2], xw[3] ^ L.mask[3]);
  } else if constexpr (P::C == 2) {
    reinterpret_cast<uint2*>(w)[L.lane] = make_uint2(xw[0] ^ L.mask[0], xw[1] ^ L.mask[1]);
  } else {
    w[L.lane] = xw[0] ^ L.mask[0];
  }
}

// Group max over the lanes of one scale group (chunk k2 = lane for SRHT,
// bitrev5(lane) for SRFT: consecutive chunks are low lane bits, resp. high).
template <int D, int G, int ROT>
__device__ __forceinline__ float wide_group_max(float m) {
  constexpr int GL = G / Wide<D, ROT>::W;  // lanes per group
  if constexpr (ROT == kRotSRHT) {
#pragma unroll
    for (int b = 1; b < GL; b <<= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, b));
  } else {
#pragma unroll
    for (int b = 16, i = 1; i < GL; b >>= 1, i <<= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, b));
  }
  return m;
}

// Code bytes of the lane's chunk of one row.
template <int D, int ROT>
__device__ __forceinline__ void wide_store_code(uint8_t* qrow, const WideLane<D, ROT>& L,
                                                uint32_t code) {
  constexpr int QB = Wide<D, ROT>::W / 2;
  if constexpr (QB == 4) {
    reinterpret_cast<uint32_t*>(qrow)[L.k2] = code;
  } else if constexpr (QB == 2) {
    reinterpret_cast<uint16_t*>(qrow)[L.k2] = uint16_t(code);
  } else {
    qrow[L.k2] = uint8_t(code);
  }
}

template <int D, int ROT>
__device__ __forceinline__ uint32_t wide_load_code(const uint8_t* qrow, const WideLane<D, ROT>& L) {
  constexpr int QB = Wide<D, ROT>::W / 2;
  if constexpr (QB == 4) {
    return __ldg(reinterpret_cast<const uint32_t*>(qrow) + L.k2);
  } else if constexpr (QB == 2) {
    return __ldg(reinterpret_cast<const uint16_t*>(qrow) + L.k2);
  } else {
    return __ldg(qrow + L.k2);
  }
}

// Forward step on one fp16 row (steps a1-a5): writes the row's codes and
// scales, returns this lane's code bytes and its group's scale.
template <int D, int G, int ROT, bool RO = true>
__device__ __forceinline__ void wide_quantize_row(const uint16_t* src, uint8_t* qrow, float* srow,
                                                  const WideLane<D, ROT>& L, uint32_t& code,
                                                  float& s) {
  using P = Wide<D, ROT>;
  constexpr int GL = G / P::W;  // lanes (chunks) per group
  uint32_t xw[P::C];
  wide_load_words<D, ROT, RO>(src, L, xw);
  float Y[P::W];
  wide_rotate_fwd<D, ROT>(xw, L, Y);
  float m = fabsf(Y[0]);
#pragma unroll
  for (int j = 1; j < P::W; ++j) m = fmaxf(m, fabsf(Y[j]));
  m = wide_group_max<D, G, ROT>(m);
  const float inv = m > 0.0f ? __fdiv_rn(7.0f, m) : 0.0f;
  s = m * P::KAPPA7;
  uint32_t f[8];
#pragma unroll
  for (int j = 0; j < 8; ++j)
    f[j] = j < P::W ? __float_as_uint(__fmaf_rn(Y[j], inv, kRoundMagic))
                    : __float_as_uint(kRoundMagic);
  code = pack8(f);
  wide_store_code<D, ROT>(qrow, L, code);
  if (L.k2 % GL == 0) srow[L.k2 / GL] = s;
}

// Inverse step on one row (steps a6-a7) from the lane's code bytes and
// scale; writes the fp16 row.
template <int D, int ROT>
__device__ __forceinline__ void wide_dequant_row(uint32_t code, float s, uint16_t* dst,
                                                 const WideLane<D, ROT>& L) {
  using P = Wide<D, ROT>;
  const f2 magic = mk2(kUnpackMagic, kUnpackMagic);
  float Y[P::W];
  {
    f2 q[4];
    unpack8(code, q);
    const float sk = s * P::KAPPA;
    const f2 sk2 = mk2(sk, sk);
#pragma unroll
    for (int j = 0; j < P::C; ++j) {
      const f2 v = mul2(sub2(q[j], magic), sk2);
      Y[2 * j] = lo2(v);
      Y[2 * j + 1] = hi2(v);
    }
  }
  uint32_t xo[P::C];
  wide_rotate_inv<D, ROT>(Y, L, xo);
  wide_store_words<D, ROT>(dst, L, xo);
}

template <int D, int G, int ROT>
__global__ void __launch_bounds__(kWideThreads) kvq_decode_wide_kernel(const DecodeWideArgs a) {
  constexpr int NG = D / G;
  constexpr int GL = G / Wide<D, ROT>::W;  // lanes (chunks) per group
  const int lane = threadIdx.x & 31;
  pdl_wait();  // no global access before the previous kernel completes
  WideLane<D, ROT> L;
  L.init(a.signs, lane);
  const int64_t gw = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = (int64_t(gridDim.x) * blockDim.x) >> 5;
  const int64_t total = a.n_heads * (a.pos + 1);
  // item -> (head, row): the new token of every head first, then cached rows.
  // This kernel runs calls of at most 2^16 rows, so the cached-row index n
  // and pos fit 16 bits and n / pos is one multiply by the host's
  // reciprocal (wide_pos_recip) instead of a 64-bit division per row.
  const uint32_t P = uint32_t(a.pos);
  auto where = [&](int64_t it, int64_t& head, int64_t& row) {
    const bool fresh = it < a.n_heads;
    const uint32_t n = uint32_t(it - a.n_heads);
    const uint32_t q = P > 1u ? __umulhi(n, a.pos_recip) : n;
    head = fresh ? it : int64_t(q);
    row = fresh ? a.pos : int64_t(n - q * P);
    return fresh;
  };
  // the codes and scale of a cached row are loaded one item ahead, so their
  // latency overlaps the previous row's transform
  uint32_t code_next = 0;
  float s_next = 0.0f;
  auto prefetch = [&](int64_t it) {
    int64_t head, row;
    if (it < total && !where(it, head, row)) {
      const int64_t r = head * a.cap + row;
      code_next = wide_load_code<D, ROT>(a.packed + r * (D / 2), L);
      s_next = __ldg(a.scales + r * NG + L.k2 / GL);
    }
  };
  prefetch(gw);
  for (int64_t it = gw; it < total; it += nw) {
    int64_t head, row;
    const bool fresh = where(it, head, row);
    uint32_t code = code_next;  // this lane's W codes
    float s = s_next;           // scale of this lane's group
    prefetch(it + nw);
    if (fresh) {
      uint8_t* qrow = a.packed + (head * a.cap + row) * (D / 2);
      float* srow = a.scales + (head * a.cap + row) * NG;
      wide_quantize_row<D, G, ROT>(a.x_new + head * D, qrow, srow, L, code, s);
    }
    wide_dequant_row<D, ROT>(code, s, a.out + (head * (a.pos + 1) + row) * D, L);
  }
  pdl_release();
}

// ------------------------------------------- windowed decode (prefix cache) ---

struct WindowArgs {
  const uint16_t* x_new;  // [n_heads][d]
  uint8_t* packed;        // [n_heads][cap][d/2]
  float* scales;          // [n_heads][cap][d/g]
  uint16_t* kv;           // [n_heads][cap][d], persistent attention view
  const int8_t* signs;
  int64_t n_heads, cap, pos;
  int window;
};

// Decode step with a dequantized-prefix cache and an fp16 tail ([P1]
// "Before you celebrate...", second condition): row pos of kv receives the
// new token exactly; when that completes a window of `window` rows, the
// window's rows are quantized into the int4 cache and kv keeps their
// dequantized values, so rows of completed windows read as dequantized and
// the rest of the prefix is never recomputed.
template <int D, int G, int ROT>
__global__ void __launch_bounds__(kWideThreads) kvq_window_wide_kernel(const WindowArgs a) {
  constexpr int NG = D / G;
  const int lane = threadIdx.x & 31;
  const int64_t gw = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = (int64_t(gridDim.x) * blockDim.x) >> 5;
  const bool flush = (a.pos + 1) % a.window == 0;
  pdl_wait();  // no global access before the previous kernel completes
  if (!flush) {  // copy the new rows into the tail
    for (int64_t h = gw; h < a.n_heads; h += nw) {
      const uint4* src = reinterpret_cast<const uint4*>(a.x_new + h * D);
      uint4* dst = reinterpret_cast<uint4*>(a.kv + (h * a.cap + a.pos) * D);
      for (int c = lane; c < D / 8; c += 32) dst[c] = __ldg(src + c);
    }
    pdl_release();
    return;
  }
  WideLane<D, ROT> L;
  L.init(a.signs, lane);
  const int64_t first = a.pos + 1 - a.window;
  const int64_t total = a.n_heads * a.window;
  for (int64_t it = gw; it < total; it += nw) {
    const int64_t head = it / a.window;
    const int64_t row = first + it % a.window;
    const uint16_t* src = row == a.pos ? a.x_new + head * D : a.kv + (head * a.cap + row) * D;
    uint8_t* qrow = a.packed + (head * a.cap + row) * (D / 2);
    float* srow = a.scales + (head * a.cap + row) * NG;
    uint32_t code;
    float s;
    wide_quantize_row<D, G, ROT, false>(src, qrow, srow, L, code, s);
    __syncwarp();  // every lane has read the source row before it is overwritten
    wide_dequant_row<D, ROT>(code, s, a.kv + (head * a.cap + row) * D, L);
  }
  pdl_release();
}

}  // namespace kvq
