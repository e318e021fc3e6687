// kvq_codec.cuh -- fused forward / inverse / decode-step kernels of libkvq.
//
// Design (sm_100a, HBM-bound codec, no tensor cores):
//  * Persistent grid, 4 warps per CTA, each warp an independent pipeline over
//    "warp tiles" of VPW consecutive vectors (VPW = 32 / TPV, TPV = threads
//    per vector).  Lane 0 of the warp issues TMA tensor copies
//    (cp.async.bulk.tensor) of whole tiles into shared memory several tiles
//    ahead, completing on per-stage mbarriers; all lanes wait (bounded).
//  * The fp16 tile is staged with 128-byte swizzle and the code tile with the
//    swizzle matching its row pitch, so each thread reads its own vector
//    with conflict-free 128-bit shared loads.
//  * Each thread holds its vector (or half of it) in registers and runs the
//    whole step there: sign flip, rotation (FFT / FWHT, plus one exchange
//    stage through warp shuffles when TPV = 2), absmax, round, pack.
//  * Results are written to a shared tile and stored by TMA (bulk groups);
//    scales are written directly with coalesced vector stores.
//
// Forward ("Fusing four steps into two kernels is not enough": rotate plus
// quantize in one kernel) and inverse (dequantize plus inverse rotate) each
// read their input once and write their output once.
#pragma once

#include "kvq_device.cuh"

namespace kvq {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;

template <int D_, int ROT_, int TPV_>
struct Cfg {
  static constexpr int D = D_;
  static constexpr int ROT = ROT_;
  static constexpr int TPV = TPV_;
  static constexpr int VPW = 32 / TPV;     // vectors per warp tile
  static constexpr int E = D / TPV;        // reals per thread
  static constexpr int NW = E / 2;         // fp16-pair words per thread
  static constexpr int NQ = E / 8;         // packed-code words per thread
  static constexpr int XTILE = VPW * D * 2;  // fp16 tile bytes
  static constexpr int QTILE = VPW * D / 2;  // code tile bytes
  static constexpr int SLAB = VPW * 128;   // one 64-column fp16 slab
  static constexpr int QP = D / 2;         // code row pitch in bytes
  // y = KAPPA * (unnormalized transform of u): SRFT 1/sqrt(2d), SRHT 1/sqrt(d)
  static constexpr double KAPPA_D =
      ROT == kRotSRFT ? 1.0 / const_sqrt(2.0 * D) : 1.0 / const_sqrt(double(D));
  static constexpr float KAPPA = float(KAPPA_D);
  static constexpr float KAPPA7 = float(KAPPA_D / 7.0);
  static_assert(D % 64 == 0 && (TPV == 1 || TPV == 2), "shape");
};

template <int D>
struct DefaultTPV {
  static constexpr int value = D >= 256 ? 2 : 1;
};

// Word (fp16 pair) of the vector held in slot j of thread t.
template <class C>
__host__ __device__ constexpr int word_of(int t, int j) {
  return (C::ROT == kRotSRFT && C::TPV == 2) ? 2 * j + t : t * C::NW + j;
}

template <class C>
__device__ __forceinline__ uint32_t sign_mask_word(const int8_t* signs, int w) {
  return (signs[2 * w] < 0 ? 0x00008000u : 0u) | (signs[2 * w + 1] < 0 ? 0x80000000u : 0u);
}

// ------------------------------------------------ shared-memory tile I/O ---

// Swizzled byte offset of 16-byte chunk `cc` (0..7) of a 128-byte row.
__device__ __forceinline__ uint32_t sw128(int row, int cc) {
  return uint32_t(row * 128 + ((cc ^ (row & 7)) << 4));
}

// Swizzled byte offset of 16-byte chunk `c` of a code row of pitch P bytes
// (TMA swizzle mode 32B / 64B / 128B for P = 32 / 64 / 128).
template <int P>
__device__ __forceinline__ uint32_t swq(int row, int c) {
  return uint32_t(row * P + ((c ^ (((row * P) >> 7) & (P / 16 - 1))) << 4));
}

template <class C>
__device__ __forceinline__ void load_x(uint32_t tile, int row, int t, uint32_t mask,
                                       uint32_t (&xw)[C::NW]) {
  if constexpr (C::TPV == 1 || C::ROT == kRotSRHT) {
#pragma unroll
    for (int c = 0; c < C::NW / 4; ++c) {
      const int gc = t * (C::NW / 4) + c;  // chunk of the row
      const uint4 v = lds128(tile + (gc / 8) * C::SLAB + sw128(row, gc % 8));
      const uint4 m = lds128(mask + c * 16);
      xw[4 * c + 0] = v.x ^ m.x;
      xw[4 * c + 1] = v.y ^ m.y;
      xw[4 * c + 2] = v.z ^ m.z;
      xw[4 * c + 3] = v.w ^ m.w;
    }
  } else {  // SRFT, TPV = 2: thread t holds the words 2j + t
#pragma unroll
    for (int jj = 0; jj < C::NW / 4; ++jj) {
      const uint4 m = lds128(mask + jj * 16);
      const uint32_t mm[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int j = 4 * jj + r;
        const int cc = (j % 16) / 2;
        const uint32_t a = tile + (j / 16) * C::SLAB + sw128(row, cc) + (2 * (j % 2) + t) * 4;
        xw[j] = lds32(a) ^ mm[r];
      }
    }
  }
}

template <class C>
__device__ __forceinline__ void store_x(uint32_t tile, int row, int t, uint32_t mask,
                                        const uint32_t (&xw)[C::NW]) {
  if constexpr (C::TPV == 1 || C::ROT == kRotSRHT) {
#pragma unroll
    for (int c = 0; c < C::NW / 4; ++c) {
      const int gc = t * (C::NW / 4) + c;
      const uint4 m = lds128(mask + c * 16);
      sts128(tile + (gc / 8) * C::SLAB + sw128(row, gc % 8), xw[4 * c] ^ m.x,
             xw[4 * c + 1] ^ m.y, xw[4 * c + 2] ^ m.z, xw[4 * c + 3] ^ m.w);
    }
  } else {
#pragma unroll
    for (int jj = 0; jj < C::NW / 4; ++jj) {
      const uint4 m = lds128(mask + jj * 16);
      const uint32_t mm[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int j = 4 * jj + r;
        const int cc = (j % 16) / 2;
        const uint32_t a = tile + (j / 16) * C::SLAB + sw128(row, cc) + (2 * (j % 2) + t) * 4;
        sts32(a, xw[j] ^ mm[r]);
      }
    }
  }
}

template <class C>
__device__ __forceinline__ void load_codes(uint32_t tile, int row, int t, uint32_t (&qw)[C::NQ]) {
#pragma unroll
  for (int c = 0; c < C::NQ / 4; ++c) {
    const uint4 v = lds128(tile + swq<C::QP>(row, t * (C::NQ / 4) + c));
    qw[4 * c] = v.x;
    qw[4 * c + 1] = v.y;
    qw[4 * c + 2] = v.z;
    qw[4 * c + 3] = v.w;
  }
}

template <class C>
__device__ __forceinline__ void store_codes(uint32_t tile, int row, int t,
                                            const uint32_t (&qw)[C::NQ]) {
#pragma unroll
  for (int c = 0; c < C::NQ / 4; ++c)
    sts128(tile + swq<C::QP>(row, t * (C::NQ / 4) + c), qw[4 * c], qw[4 * c + 1], qw[4 * c + 2],
           qw[4 * c + 3]);
}

// ------------------------------------------------------ forward rotation ---

// Y (this thread's E consecutive rotated coordinates, unnormalized: the true
// y is KAPPA * Y) from the sign-flipped fp16 words.
template <class C>
__device__ __forceinline__ void rotate_fwd(const uint32_t (&xw)[C::NW], int t, float (&Y)[C::E]) {
  if constexpr (C::ROT == kRotSRHT) {
#pragma unroll
    for (int j = 0; j < C::NW; ++j) {
      const float2 f = half2_bits_to_float2(xw[j]);
      Y[2 * j] = f.x;
      Y[2 * j + 1] = f.y;
    }
    fwht<C::E>(Y);
    if constexpr (C::TPV == 2) {  // H_d = [[H, H], [H, -H]] across the pair
      const float sg = t ? -1.0f : 1.0f;
#pragma unroll
      for (int i = 0; i < C::E; ++i) {
        const float p = __shfl_xor_sync(kFull, Y[i], 1);
        Y[i] = fmaf(sg, Y[i], p);
      }
    }
  } else if constexpr (C::TPV == 1) {
    // z_n = u_{2n} + i u_{2n+1}; Z = FFT_{d/2}(z); X_k from (Z_k, Z_{d/2-k}).
    constexpr int N = C::D / 2;
    constexpr int LN = ilog2(N);
    float zr[N], zi[N];
#pragma unroll
    for (int j = 0; j < N; ++j) {
      const float2 f = half2_bits_to_float2(xw[j]);
      zr[j] = f.x;
      zi[j] = f.y;
    }
    fft_dif<N, false>(zr, zi);
    constexpr float R2 = 1.41421356237309504880f;
    Y[0] = R2 * (zr[0] + zi[0]);  // sqrt2 * X_0
    Y[1] = R2 * (zr[0] - zi[0]);  // sqrt2 * X_{d/2}
    static_for<1, N / 2>([&](auto kk) {
      constexpr int k = decltype(kk)::value;
      constexpr int sa = bitrev(k, LN), sb = bitrev(N - k, LN);
      const float ar = zr[sa], ai = zi[sa], br = zr[sb], bi = -zi[sb];  // B = conj Z_{N-k}
      const float sr = ar + br, si = ai + bi, tr = ar - br, ti = ai - bi;
      // 2X_k = S + W^k (-i T), 2X_{N-k} = conj(S - W^k (-i T)), W = exp(-2 pi i / d)
      constexpr float c = tw_cos(k, C::D), s = tw_sin(k, C::D);
      const float pr = ti, pi = -tr;
      const float wr = fmaf(c, pr, s * pi), wi = fmaf(c, pi, -(s * pr));
      Y[2 * k] = sr + wr;
      Y[2 * k + 1] = si + wi;
      Y[2 * (N - k)] = sr - wr;
      Y[2 * (N - k) + 1] = wi - si;
    });
    constexpr int sm = bitrev(N / 2, LN);
    Y[N] = 2.0f * zr[sm];  // 2X_{d/4} = 2 conj Z_{d/4}
    Y[N + 1] = -2.0f * zi[sm];
  } else {
    // TPV = 2.  Thread t holds z_{2m+t} (m < M = d/4): in-thread FFT_M, then
    // the last decimation-in-time stage across the pair gives thread t the
    // outputs Z_{k + t M}; X_k for those k uses the partner's Z_{d/2-k}.
    constexpr int M = C::D / 4;
    constexpr int N = C::D / 2;
    constexpr int LM = ilog2(M);
    float zr[M], zi[M];
#pragma unroll
    for (int j = 0; j < M; ++j) {
      const float2 f = half2_bits_to_float2(xw[j]);
      zr[j] = f.x;
      zi[j] = f.y;
    }
    fft_dif<M, false>(zr, zi);
    const float sg = t ? -1.0f : 1.0f;
    static_for<0, M>([&](auto kk) {
      constexpr int k = decltype(kk)::value;
      constexpr int sl = bitrev(k, LM);
      float r = zr[sl], i = zi[sl];
      if constexpr (k != 0) {
        float wr, wi;
        twiddle<N, k, false>(r, i, wr, wi);
        r = t ? wr : r;
        i = t ? wi : i;
      }
      const float pr = __shfl_xor_sync(kFull, r, 1);
      const float pi = __shfl_xor_sync(kFull, i, 1);
      zr[sl] = fmaf(sg, r, pr);  // t=0: F0 + W F1; t=1: F0 - W F1
      zi[sl] = fmaf(sg, i, pi);
    });
    constexpr float R2 = 1.41421356237309504880f;
    {
      const float a = zr[0], b = zi[0];
      Y[0] = t ? 2.0f * a : R2 * (a + b);  // t=1 holds Z_{d/4}: 2 conj Z_{d/4}
      Y[1] = t ? -2.0f * b : R2 * (a - b);
    }
    static_for<1, M>([&](auto kk) {
      constexpr int k = decltype(kk)::value;
      constexpr int sa = bitrev(k, LM), sb = bitrev(M - k, LM);
      const float ar = zr[sa], ai = zi[sa];
      const float br = __shfl_xor_sync(kFull, zr[sb], 1);
      const float bi = -__shfl_xor_sync(kFull, zi[sb], 1);
      const float sr = ar + br, si = ai + bi;
      const float ur = br - ar, ui = bi - ai;  // U = -T
      // thread 0: P = -i T = (-ui, ur); thread 1: W^{M} = -i folds in, P = -T = U
      const float pr = t ? ur : -ui;
      const float pi = t ? ui : ur;
      constexpr float c = tw_cos(k, C::D), s = tw_sin(k, C::D);
      const float wr = fmaf(c, pr, s * pi), wi = fmaf(c, pi, -(s * pr));
      Y[2 * k] = sr + wr;
      Y[2 * k + 1] = si + wi;
    });
  }
}

// ------------------------------------------------------ inverse rotation ---

// Thread's fp16 words of u = R^T y_hat.  The input is pre-scaled,
// Yin = KAPPA * y_hat, so that the unnormalized inverse transform (the exact
// inverse of rotate_fwd's unnormalized map up to the factor 1/KAPPA^2) yields
// u itself.
template <class C>
__device__ __forceinline__ void rotate_inv(float (&Y)[C::E], int t, uint32_t (&xw)[C::NW]) {
  if constexpr (C::ROT == kRotSRHT) {
    if constexpr (C::TPV == 2) {
      const float sg = t ? -1.0f : 1.0f;
#pragma unroll
      for (int i = 0; i < C::E; ++i) {
        const float p = __shfl_xor_sync(kFull, Y[i], 1);
        Y[i] = fmaf(sg, Y[i], p);
      }
    }
    fwht<C::E>(Y);
#pragma unroll
    for (int j = 0; j < C::NW; ++j) xw[j] = float2_to_half2_bits(Y[2 * j], Y[2 * j + 1]);
  } else if constexpr (C::TPV == 1) {
    constexpr int N = C::D / 2;
    constexpr int LN = ilog2(N);
    constexpr float R2 = 1.41421356237309504880f;
    float zr[N], zi[N];
    // Q_k = (A + B) + i W^{-k} (A - B), A = X'_k, B = conj X'_{N-k}
    zr[0] = R2 * (Y[0] + Y[1]);
    zi[0] = R2 * (Y[0] - Y[1]);
    static_for<1, N / 2>([&](auto kk) {
      constexpr int k = decltype(kk)::value;
      const float ar = Y[2 * k], ai = Y[2 * k + 1];
      const float br = Y[2 * (N - k)], bi = -Y[2 * (N - k) + 1];
      const float sr = ar + br, si = ai + bi, dr = ar - br, di = ai - bi;
      constexpr float c = tw_cos(k, C::D), s = tw_sin(k, C::D);
      const float vr = fmaf(c, dr, -(s * di)), vi = fmaf(c, di, s * dr);  // W^{-k} D
      zr[k] = sr - vi;  // Q_k = S + i V
      zi[k] = si + vr;
      zr[N - k] = sr + vi;  // Q_{N-k} = conj(S - i V)
      zi[N - k] = vr - si;
    });
    zr[N / 2] = 2.0f * Y[N];
    zi[N / 2] = -2.0f * Y[N + 1];
    fft_dif<N, true>(zr, zi);
    static_for<0, N>([&](auto nn) {
      constexpr int n = decltype(nn)::value;
      constexpr int sl = bitrev(n, LN);
      xw[n] = float2_to_half2_bits(zr[sl], zi[sl]);
    });
  } else {
    constexpr int M = C::D / 4;
    constexpr int N = C::D / 2;
    constexpr int LM = ilog2(M);
    constexpr float R2 = 1.41421356237309504880f;
    float zr[M], zi[M];
    {
      const float a = Y[0], b = Y[1];
      zr[0] = t ? 2.0f * a : R2 * (a + b);
      zi[0] = t ? -2.0f * b : R2 * (a - b);
    }
    static_for<1, M>([&](auto kk) {
      constexpr int k = decltype(kk)::value;
      const float ar = Y[2 * k], ai = Y[2 * k + 1];
      const float br = __shfl_xor_sync(kFull, Y[2 * (M - k)], 1);
      const float bi = -__shfl_xor_sync(kFull, Y[2 * (M - k) + 1], 1);
      const float sr = ar + br, si = ai + bi, dr = ar - br, di = ai - bi;
      constexpr float c = tw_cos(k, C::D), s = tw_sin(k, C::D);
      const float vr = fmaf(c, dr, -(s * di)), vi = fmaf(c, di, s * dr);
      // thread 0: Q = S + i V; thread 1: W^{-M} = +i folds in, Q = S - V
      zr[k] = sr - (t ? vr : vi);
      zi[k] = si + (t ? -vi : vr);
    });
    // Inverse of the cross-pair stage: thread 0 keeps E_k = Q_k + Q_{k+M},
    // thread 1 keeps O_k = (Q_k - Q_{k+M}) W_{d/2}^{-k}.
    const float sg = t ? -1.0f : 1.0f;
    static_for<0, M>([&](auto kk) {
      constexpr int k = decltype(kk)::value;
      const float pr = __shfl_xor_sync(kFull, zr[k], 1);
      const float pi = __shfl_xor_sync(kFull, zi[k], 1);
      float r = fmaf(sg, zr[k], pr), i = fmaf(sg, zi[k], pi);
      if constexpr (k != 0) {
        float wr, wi;
        twiddle<N, k, true>(r, i, wr, wi);
        r = t ? wr : r;
        i = t ? wi : i;
      }
      zr[k] = r;
      zi[k] = i;
    });
    fft_dif<M, true>(zr, zi);
    static_for<0, M>([&](auto mm) {
      constexpr int m = decltype(mm)::value;
      constexpr int sl = bitrev(m, LM);
      xw[m] = float2_to_half2_bits(zr[sl], zi[sl]);
    });
  }
}

// ------------------------------------------------------ quantize / pack ---

template <class C, int G>
struct Groups {
  static constexpr int GL = G <= C::E ? G : C::E;  // group length in this thread
  static constexpr int NL = C::E / GL;             // groups (scales) per thread
  static constexpr bool SHARED = G > C::E;         // one group over the pair
  static constexpr int NG = C::D / G;              // scales per vector
  static_assert(GL % 8 == 0, "group");
};

template <class C, int G>
__device__ __forceinline__ void quantize(const float (&Y)[C::E], uint32_t (&qw)[C::NQ],
                                         float (&sc)[Groups<C, G>::NL]) {
  using Gr = Groups<C, G>;
#pragma unroll
  for (int g = 0; g < Gr::NL; ++g) {
    float m = absmax<Gr::GL>(&Y[g * Gr::GL]);
    if constexpr (Gr::SHARED) m = fmaxf(m, __shfl_xor_sync(kFull, m, 1));
    const float inv = m > 0.0f ? __fdiv_rn(7.0f, m) : 0.0f;
    sc[g] = m * C::KAPPA7;
#pragma unroll
    for (int w = 0; w < Gr::GL / 8; ++w) {
      uint32_t f[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        f[i] = __float_as_uint(__fmaf_rn(Y[g * Gr::GL + 8 * w + i], inv, kRoundMagic));
      qw[(g * Gr::GL) / 8 + w] = pack8(f);
    }
  }
}

// Yin = q * (s * KAPPA), ready for the unnormalized inverse transform.
template <class C, int G>
__device__ __forceinline__ void dequantize(const uint32_t (&qw)[C::NQ],
                                           const float (&sc)[Groups<C, G>::NL],
                                           float (&Y)[C::E]) {
  using Gr = Groups<C, G>;
#pragma unroll
  for (int g = 0; g < Gr::NL; ++g) {
    const float sk = sc[g] * C::KAPPA;
#pragma unroll
    for (int w = 0; w < Gr::GL / 8; ++w) {
      float q[8];
      unpack8(qw[(g * Gr::GL) / 8 + w], q);
#pragma unroll
      for (int i = 0; i < 8; ++i) Y[g * Gr::GL + 8 * w + i] = q[i] * sk;
    }
  }
}

// ------------------------------------------------------------- kernels ---

struct FwdArgs {
  const int8_t* signs;
  float* scales;
  int64_t n_vec;
  int64_t n_tiles;
};

struct InvArgs {
  const int8_t* signs;
  int64_t n_vec;
  int64_t n_tiles;
};

struct DecodeArgs {
  const int8_t* signs;
  float* scales;  // [n_heads][cap][d/g]
  int64_t n_heads;
  int64_t cap;
  int64_t pos;
  int64_t n_new_tiles;  // ceil(n_heads / VPW)
  int64_t tok_tiles;    // ceil(pos / VPW)
  int64_t n_tiles;      // n_new_tiles + n_heads * tok_tiles
};

template <class C>
__device__ __forceinline__ void fill_sign_masks(const int8_t* signs, uint32_t* s_mask) {
  for (int i = threadIdx.x; i < C::D / 2; i += blockDim.x) {
    const int t = i / C::NW, j = i % C::NW;
    s_mask[i] = sign_mask_word<C>(signs, word_of<C>(t, j));
  }
}

template <class C, int G>
__device__ __forceinline__ void store_scales_global(float* scales, int64_t vrow, int t,
                                                    const float (&sc)[Groups<C, G>::NL]) {
  using Gr = Groups<C, G>;
  if constexpr (Gr::SHARED) {
    if (t == 0) scales[vrow * Gr::NG] = sc[0];
  } else {
    float* p = scales + vrow * Gr::NG + t * Gr::NL;
    if constexpr (Gr::NL == 1) {
      p[0] = sc[0];
    } else if constexpr (Gr::NL == 2) {
      *reinterpret_cast<float2*>(p) = make_float2(sc[0], sc[1]);
    } else {
#pragma unroll
      for (int i = 0; i < Gr::NL; i += 4)
        *reinterpret_cast<float4*>(p + i) = make_float4(sc[i], sc[i + 1], sc[i + 2], sc[i + 3]);
    }
  }
}

template <class C, int G>
__device__ __forceinline__ void load_scales_smem(uint32_t sbuf, int row, int t,
                                                 float (&sc)[Groups<C, G>::NL]) {
  using Gr = Groups<C, G>;
  const uint32_t a = sbuf + uint32_t(row * Gr::NG + (Gr::SHARED ? 0 : t * Gr::NL)) * 4u;
#pragma unroll
  for (int i = 0; i < Gr::NL; ++i) sc[i] = __uint_as_float(lds32(a + 4 * i));
}

template <int S>
struct Stages {
  static constexpr int value = S;
};

// Per-warp ring bookkeeping: which tiles have a load in flight.
struct Ring {
  int64_t issued;    // loads issued (tiles of this warp, in order)
  int64_t consumed;  // tiles waited for
};

// After a timed-out wait: wait (bounded) for the loads still in flight so
// that no copy lands in shared memory after the block exits, then record.
template <int S_IN>
__device__ __noinline__ void drain_and_fail(uint32_t bars, const Ring& r, unsigned* status) {
  for (int64_t k = r.consumed; k < r.issued; ++k)
    (void)mbar_wait_bounded(bars + 8u * uint32_t(k % S_IN), uint32_t((k / S_IN) & 1));
  atomicOr(status, 1u);
}

template <int D, int G, int ROT, int TPV, int S_IN>
__global__ void __launch_bounds__(kThreads, 1)
    kvq_fwd_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmQ,
                   const FwdArgs a, unsigned* status) {
  using C = Cfg<D, ROT, TPV>;
  using Gr = Groups<C, G>;
  constexpr int S_OUT = 2;
  constexpr int WARP_BYTES = S_IN * C::XTILE + S_OUT * C::QTILE;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars_sm[kWarps][S_IN];
  __shared__ __align__(16) uint32_t s_mask[C::D / 2];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = C::TPV == 2 ? (lane & 1) : 0;
  const int row = C::TPV == 2 ? (lane >> 1) : lane;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t xbuf = base + uint32_t(warp * WARP_BYTES);
  const uint32_t qbuf = xbuf + uint32_t(S_IN * C::XTILE);
  const uint32_t bars = smem_u32(&bars_sm[warp][0]);

  fill_sign_masks<C>(a.signs, s_mask);
  if (lane == 0) {
    for (int s = 0; s < S_IN; ++s) mbar_init(bars + 8u * s, 1);
    fence_mbar_init();
  }
  if (threadIdx.x == 0) {
    prefetch_tensormap(&tmX);
    prefetch_tensormap(&tmQ);
  }
  __syncthreads();
  const uint32_t mask = smem_u32(s_mask) + uint32_t(t * C::NW * 4);

  const int64_t gw = int64_t(blockIdx.x) * kWarps + warp;
  const int64_t nw = int64_t(gridDim.x) * kWarps;
  Ring ring{0, 0};
  auto issue = [&](int64_t tile) {  // lane 0 only
    const int s = int(ring.issued % S_IN);
    const uint32_t bar = bars + 8u * s;
    const uint32_t dst = xbuf + uint32_t(s * C::XTILE);
    mbar_arrive_expect_tx(bar, C::XTILE);
#pragma unroll
    for (int j = 0; j < C::D / 64; ++j)
      tma_load_2d(dst + j * C::SLAB, &tmX, bar, 64 * j, int(tile * C::VPW));
    ++ring.issued;
  };
  if (lane == 0)
    for (int s = 0; s < S_IN && gw + s * nw < a.n_tiles; ++s) issue(gw + s * nw);

  bool failed = false;
  for (int64_t tile = gw; tile < a.n_tiles; tile += nw) {
    const int s = int(ring.consumed % S_IN);
    const bool ok = mbar_wait_bounded(bars + 8u * s, uint32_t((ring.consumed / S_IN) & 1));
    if (!__all_sync(kFull, ok)) {
      failed = true;
      break;
    }
    ++ring.consumed;
    uint32_t xw[C::NW];
    load_x<C>(xbuf + uint32_t(s * C::XTILE), row, t, mask, xw);
    __syncwarp();
    if (lane == 0) {
      const int64_t nt = tile + int64_t(S_IN) * nw;
      if (nt < a.n_tiles) {
        fence_proxy_async_smem();
        issue(nt);
      }
    }
    float Y[C::E];
    rotate_fwd<C>(xw, t, Y);
    uint32_t qw[C::NQ];
    float sc[Gr::NL];
    quantize<C, G>(Y, qw, sc);

    const int o = int((ring.consumed - 1) % S_OUT);
    if (lane == 0) bulk_wait_read<S_OUT - 1>();
    __syncwarp();
    const uint32_t qdst = qbuf + uint32_t(o * C::QTILE);
    store_codes<C>(qdst, row, t, qw);
    const int64_t vrow = tile * C::VPW + row;
    if (vrow < a.n_vec) store_scales_global<C, G>(a.scales, vrow, t, sc);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(&tmQ, qdst, 0, int(tile * C::VPW));
      bulk_commit();
    }
  }
  if (lane == 0) {
    bulk_wait_all();
    if (failed) drain_and_fail<S_IN>(bars, ring, status);
  }
}

template <int D, int G, int ROT, int TPV, int S_IN>
__global__ void __launch_bounds__(kThreads, 1)
    kvq_inv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmS,
                   const __grid_constant__ CUtensorMap tmX, const InvArgs a, unsigned* status) {
  using C = Cfg<D, ROT, TPV>;
  using Gr = Groups<C, G>;
  constexpr int S_OUT = 2;
  constexpr int STILE = C::VPW * Gr::NG * 4;
  constexpr int STAGE = C::QTILE + ((STILE + 1023) / 1024) * 1024;
  constexpr int WARP_BYTES = S_IN * STAGE + S_OUT * C::XTILE;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars_sm[kWarps][S_IN];
  __shared__ __align__(16) uint32_t s_mask[C::D / 2];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = C::TPV == 2 ? (lane & 1) : 0;
  const int row = C::TPV == 2 ? (lane >> 1) : lane;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t ibuf = base + uint32_t(warp * WARP_BYTES);
  const uint32_t xbuf = ibuf + uint32_t(S_IN * STAGE);
  const uint32_t bars = smem_u32(&bars_sm[warp][0]);

  fill_sign_masks<C>(a.signs, s_mask);
  if (lane == 0) {
    for (int s = 0; s < S_IN; ++s) mbar_init(bars + 8u * s, 1);
    fence_mbar_init();
  }
  if (threadIdx.x == 0) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmS);
    prefetch_tensormap(&tmX);
  }
  __syncthreads();
  const uint32_t mask = smem_u32(s_mask) + uint32_t(t * C::NW * 4);

  const int64_t gw = int64_t(blockIdx.x) * kWarps + warp;
  const int64_t nw = int64_t(gridDim.x) * kWarps;
  Ring ring{0, 0};
  auto issue = [&](int64_t tile) {
    const int s = int(ring.issued % S_IN);
    const uint32_t bar = bars + 8u * s;
    const uint32_t dst = ibuf + uint32_t(s * STAGE);
    mbar_arrive_expect_tx(bar, C::QTILE + STILE);
    tma_load_2d(dst, &tmQ, bar, 0, int(tile * C::VPW));
    tma_load_1d(dst + C::QTILE, &tmS, bar, int(tile * C::VPW * Gr::NG));
    ++ring.issued;
  };
  if (lane == 0)
    for (int s = 0; s < S_IN && gw + s * nw < a.n_tiles; ++s) issue(gw + s * nw);

  bool failed = false;
  for (int64_t tile = gw; tile < a.n_tiles; tile += nw) {
    const int s = int(ring.consumed % S_IN);
    const bool ok = mbar_wait_bounded(bars + 8u * s, uint32_t((ring.consumed / S_IN) & 1));
    if (!__all_sync(kFull, ok)) {
      failed = true;
      break;
    }
    ++ring.consumed;
    const uint32_t src = ibuf + uint32_t(s * STAGE);
    uint32_t qw[C::NQ];
    float sc[Gr::NL];
    load_codes<C>(src, row, t, qw);
    load_scales_smem<C, G>(src + C::QTILE, row, t, sc);
    __syncwarp();
    if (lane == 0) {
      const int64_t nt = tile + int64_t(S_IN) * nw;
      if (nt < a.n_tiles) {
        fence_proxy_async_smem();
        issue(nt);
      }
    }
    float Y[C::E];
    dequantize<C, G>(qw, sc, Y);
    uint32_t xw[C::NW];
    rotate_inv<C>(Y, t, xw);

    const int o = int((ring.consumed - 1) % S_OUT);
    if (lane == 0) bulk_wait_read<S_OUT - 1>();
    __syncwarp();
    const uint32_t xdst = xbuf + uint32_t(o * C::XTILE);
    store_x<C>(xdst, row, t, mask, xw);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
#pragma unroll
      for (int j = 0; j < C::D / 64; ++j)
        tma_store_2d(&tmX, xdst + j * C::SLAB, 64 * j, int(tile * C::VPW));
      bulk_commit();
    }
  }
  if (lane == 0) {
    bulk_wait_all();
    if (failed) drain_and_fail<S_IN>(bars, ring, status);
  }
}

// Decode step: tiles [0, n_new_tiles) quantize the new token of VPW heads
// (forward step), write its codes/scales into cache row `pos`, and write
// its dequantized output row from registers; the remaining tiles run the
// inverse step over cache rows [0, pos) of one head each.
template <int D, int G, int ROT, int TPV, int S_IN>
__global__ void __launch_bounds__(kThreads, 1)
    kvq_decode_kernel(const __grid_constant__ CUtensorMap tmXn,  // x_new [n_heads][d]
                      const __grid_constant__ CUtensorMap tmQn,  // packed row pos, per head
                      const __grid_constant__ CUtensorMap tmOn,  // out row pos, per head
                      const __grid_constant__ CUtensorMap tmQc,  // packed cache, 3-D
                      const __grid_constant__ CUtensorMap tmOc,  // out rows < pos, 3-D
                      const DecodeArgs a, unsigned* status) {
  using C = Cfg<D, ROT, TPV>;
  using Gr = Groups<C, G>;
  constexpr int S_OUT = 2;
  constexpr int STAGE = C::QTILE;
  constexpr int WARP_BYTES = S_IN * STAGE + S_OUT * C::XTILE;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars_sm[kWarps][S_IN + 1];
  __shared__ __align__(16) uint32_t s_mask[C::D / 2];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = C::TPV == 2 ? (lane & 1) : 0;
  const int row = C::TPV == 2 ? (lane >> 1) : lane;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t ibuf = base + uint32_t(warp * WARP_BYTES);
  const uint32_t xbuf = ibuf + uint32_t(S_IN * STAGE);
  const uint32_t bars = smem_u32(&bars_sm[warp][0]);
  const uint32_t bar_new = bars + 8u * S_IN;

  fill_sign_masks<C>(a.signs, s_mask);
  if (lane == 0) {
    for (int s = 0; s <= S_IN; ++s) mbar_init(bars + 8u * s, 1);
    fence_mbar_init();
  }
  __syncthreads();
  const uint32_t mask = smem_u32(s_mask) + uint32_t(t * C::NW * 4);
  const int64_t gw = int64_t(blockIdx.x) * kWarps + warp;
  const int64_t nw = int64_t(gridDim.x) * kWarps;

  // ---- new tokens: one synchronous tile at a time (few heads per call) ----
  uint32_t new_phase = 0;
  bool failed = false;
  for (int64_t nt = gw; nt < a.n_new_tiles; nt += nw) {
    const uint32_t xin = xbuf, xout = xbuf + C::XTILE, qout = ibuf;
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_new, C::XTILE);
#pragma unroll
      for (int j = 0; j < C::D / 64; ++j)
        tma_load_2d(xin + j * C::SLAB, &tmXn, bar_new, 64 * j, int(nt * C::VPW));
    }
    const bool ok = mbar_wait_bounded(bar_new, new_phase);
    if (!__all_sync(kFull, ok)) {
      if (lane == 0) {
        (void)mbar_wait_bounded(bar_new, new_phase);
        atomicOr(status, 1u);
      }
      return;
    }
    new_phase ^= 1u;
    uint32_t xw[C::NW];
    load_x<C>(xin, row, t, mask, xw);
    float Y[C::E];
    rotate_fwd<C>(xw, t, Y);
    uint32_t qw[C::NQ];
    float sc[Gr::NL];
    quantize<C, G>(Y, qw, sc);
    store_codes<C>(qout, row, t, qw);
    const int64_t h = nt * C::VPW + row;
    if (h < a.n_heads) {
      float* p = a.scales + (h * a.cap + a.pos) * Gr::NG;
      if constexpr (Gr::SHARED) {
        if (t == 0) p[0] = sc[0];
      } else {
#pragma unroll
        for (int i = 0; i < Gr::NL; ++i) p[t * Gr::NL + i] = sc[i];
      }
    }
    dequantize<C, G>(qw, sc, Y);
    rotate_inv<C>(Y, t, xw);
    store_x<C>(xout, row, t, mask, xw);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(&tmQn, qout, 0, int(nt * C::VPW));
#pragma unroll
      for (int j = 0; j < C::D / 64; ++j)
        tma_store_2d(&tmOn, xout + j * C::SLAB, 64 * j, int(nt * C::VPW));
      bulk_commit();
      bulk_wait_read<0>();
    }
    __syncwarp();
  }

  // ---- cached rows [0, pos): pipelined inverse step ----
  // Codes arrive by TMA; scales (a row of the scales cache is d/g floats,
  // so a cache row need not start on the 16 bytes a TMA copy needs) are read
  // with plain loads, issued before the wait on the codes.
  const int64_t n_inv = a.n_tiles - a.n_new_tiles;
  int64_t first = gw - a.n_new_tiles;  // this warp's first inverse tile
  if (first < 0) first += ((-first + nw - 1) / nw) * nw;
  Ring ring{0, 0};
  auto coords = [&](int64_t i, int& head, int& tok) {
    head = int(i / a.tok_tiles);
    tok = int((i % a.tok_tiles) * C::VPW);
  };
  auto issue = [&](int64_t i) {
    int head, tok;
    coords(i, head, tok);
    const int s = int(ring.issued % S_IN);
    const uint32_t bar = bars + 8u * s;
    mbar_arrive_expect_tx(bar, C::QTILE);
    tma_load_3d(ibuf + uint32_t(s * STAGE), &tmQc, bar, 0, tok, head);
    ++ring.issued;
  };
  if (lane == 0)
    for (int s = 0; s < S_IN && first + s * nw < n_inv; ++s) issue(first + s * nw);
  for (int64_t i = first; i < n_inv; i += nw) {
    float sc[Gr::NL];
    {
      int head, tok;
      coords(i, head, tok);
      const int64_t r = int64_t(tok) + row;
      const float* p = a.scales + (int64_t(head) * a.cap + r) * Gr::NG +
                       (Gr::SHARED ? 0 : t * Gr::NL);
#pragma unroll
      for (int k = 0; k < Gr::NL; ++k) sc[k] = r < a.pos ? __ldg(p + k) : 0.0f;
    }
    const int s = int(ring.consumed % S_IN);
    const bool ok = mbar_wait_bounded(bars + 8u * s, uint32_t((ring.consumed / S_IN) & 1));
    if (!__all_sync(kFull, ok)) {
      failed = true;
      break;
    }
    ++ring.consumed;
    const uint32_t src = ibuf + uint32_t(s * STAGE);
    uint32_t qw[C::NQ];
    load_codes<C>(src, row, t, qw);
    __syncwarp();
    if (lane == 0) {
      const int64_t ni = i + int64_t(S_IN) * nw;
      if (ni < n_inv) {
        fence_proxy_async_smem();
        issue(ni);
      }
    }
    float Y[C::E];
    dequantize<C, G>(qw, sc, Y);
    uint32_t xw[C::NW];
    rotate_inv<C>(Y, t, xw);
    const int o = int((ring.consumed - 1) % S_OUT);
    if (lane == 0) bulk_wait_read<S_OUT - 1>();
    __syncwarp();
    const uint32_t xdst = xbuf + uint32_t(o * C::XTILE);
    store_x<C>(xdst, row, t, mask, xw);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      int head, tok;
      coords(i, head, tok);
#pragma unroll
      for (int j = 0; j < C::D / 64; ++j) tma_store_3d(&tmOc, xdst + j * C::SLAB, 64 * j, tok, head);
      bulk_commit();
    }
  }
  if (lane == 0) {
    bulk_wait_all();
    if (failed) drain_and_fail<S_IN>(bars, ring, status);
  }
}

// Dynamic shared memory each kernel needs (plus 1 KiB alignment slack).
template <int D, int ROT, int TPV, int S_IN>
constexpr int fwd_smem_bytes() {
  using C = Cfg<D, ROT, TPV>;
  return kWarps * (S_IN * C::XTILE + 2 * C::QTILE) + 1024;
}

template <int D, int ROT, int TPV, int S_IN>
constexpr int decode_smem_bytes() {
  using C = Cfg<D, ROT, TPV>;
  return kWarps * (S_IN * C::QTILE + 2 * C::XTILE) + 1024;
}

template <int D, int G, int ROT, int TPV, int S_IN>
constexpr int inv_smem_bytes() {
  using C = Cfg<D, ROT, TPV>;
  constexpr int STILE = C::VPW * (D / G) * 4;
  constexpr int STAGE = C::QTILE + ((STILE + 1023) / 1024) * 1024;
  return kWarps * (S_IN * STAGE + 2 * C::XTILE) + 1024;
}

}  // namespace kvq
