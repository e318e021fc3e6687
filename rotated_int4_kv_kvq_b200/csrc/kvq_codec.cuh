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
#include "kvq_rfft.cuh"

// Inverse of the one-thread SRFT: 1 = generated c2r codelet, 0 = half-length
// complex FFT with the real pre-split.
#ifndef KVQ_INV_CODELET
#define KVQ_INV_CODELET 0
#endif

namespace kvq {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;

// Where a thread's E local rotated coordinates sit in the vector's y:
//  kLayFull    (one thread per vector): local i is y[i].
//  kLayHalf    (SRHT, thread pair):     thread t holds y[t*E + i].
//  kLayQuarter (SRFT, thread pair):     local half h (E/2 values) of thread t is
//           quarter qd = h ? 3 - 2t : 2t of y, i.e. thread 0 holds quarters
//           0 and 3 and thread 1 quarters 2 and 1.  This is where the pair
//           split of the real FFT leaves each output (see rotate_fwd), and it
//           makes every (X_k, X_{N-k}) pair but one local to a thread.
constexpr int kLayFull = 0, kLayHalf = 1, kLayQuarter = 2;

template <int D_, int ROT_, int TPV_>
struct Cfg {
  static constexpr int D = D_;
  static constexpr int ROT = ROT_;
  static constexpr int TPV = TPV_;
  static constexpr int VPW = 32 / TPV;     // vectors per warp tile
  static constexpr int E = D / TPV;        // reals per thread
  static constexpr int P = E / 2;          // float pairs per thread
  static constexpr int NW = E / 2;         // fp16-pair words per thread
  static constexpr int NQ = E / 8;         // packed-code words per thread
  static constexpr int XTILE = VPW * D * 2;  // fp16 tile bytes
  static constexpr int QTILE = VPW * D / 2;  // code tile bytes
  static constexpr int SLAB = VPW * 128;   // one 64-column fp16 slab
  static constexpr int QP = D / 2;         // code row pitch in bytes
  static constexpr int LAYOUT = TPV == 1 ? kLayFull : (ROT == kRotSRFT ? kLayQuarter : kLayHalf);
  // y = KAPPA_FWD * Y (Y: rotate_fwd's unnormalized output) and the inverse
  // takes Yin = KAPPA_INV * y_hat.  One-thread SRFT (generated real-FFT
  // codelets, Y = packed rfft with X_0, X_{d/2} over sqrt2): sqrt(2/d) and
  // 1/sqrt(2d).  Thread-pair SRFT (Y = 2X packing): 1/sqrt(2d) both ways.
  // SRHT: 1/sqrt(d) both ways.
  static constexpr bool CODELET = ROT == kRotSRFT && TPV == 1;
  static constexpr bool INV_CODELET = KVQ_INV_CODELET != 0;
  static constexpr double KAPPA_FWD_D =
      ROT == kRotSRHT ? 1.0 / const_sqrt(double(D))
                      : (CODELET ? const_sqrt(2.0 / D) : 1.0 / const_sqrt(2.0 * D));
  static constexpr double KAPPA_INV_D =
      ROT == kRotSRHT ? 1.0 / const_sqrt(double(D)) : 1.0 / const_sqrt(2.0 * D);
  static constexpr float KAPPA_INV = float(KAPPA_INV_D);
  static constexpr float KAPPA7 = float(KAPPA_FWD_D / 7.0);
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

// Quarter of y holding local half h of thread t (kLayQuarter layout).
__device__ __forceinline__ int quarter_of(int t, int h) { return h ? 3 - 2 * t : 2 * t; }

// y index of local coordinate i of thread t.
template <class C>
__device__ __forceinline__ int global_y(int t, int i) {
  if constexpr (C::LAYOUT == kLayFull) {
    return i;
  } else if constexpr (C::LAYOUT == kLayHalf) {
    return t * C::E + i;
  } else {
    return quarter_of(t, i / (C::E / 2)) * (C::D / 4) + i % (C::E / 2);
  }
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

// 16-byte code chunk of the row holding local code chunk lc of thread t.
template <class C>
__device__ __forceinline__ int code_chunk(int t, int lc) {
  return global_y<C>(t, 32 * lc) / 32;
}

template <class C>
__device__ __forceinline__ void load_codes(uint32_t tile, int row, int t, uint32_t (&qw)[C::NQ]) {
#pragma unroll
  for (int c = 0; c < C::NQ / 4; ++c) {
    const uint4 v = lds128(tile + swq<C::QP>(row, code_chunk<C>(t, c)));
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
    sts128(tile + swq<C::QP>(row, code_chunk<C>(t, c)), qw[4 * c], qw[4 * c + 1], qw[4 * c + 2],
           qw[4 * c + 3]);
}

// ------------------------------------------------------ forward rotation ---

constexpr float kSqrt2 = 1.41421356237309504880f;

// Y: this thread's E rotated coordinates as P pairs (local order of the
// layout), unnormalized: the true y is KAPPA * Y.  Input: sign-flipped fp16
// words.
template <class C>
__device__ __forceinline__ void rotate_fwd(const uint32_t (&xw)[C::NW], int t, f2 (&Y)[C::P]) {
  if constexpr (C::ROT == kRotSRHT) {
#pragma unroll
    for (int j = 0; j < C::NW; ++j) {
      const float2 f = half2_bits_to_float2(xw[j]);
      Y[j] = mk2(f.x, f.y);
    }
    fwht<C::P>(Y);
    if constexpr (C::TPV == 2) {  // H_d = [[H, H], [H, -H]] across the pair
      const float sg = t ? -1.0f : 1.0f;
      const f2 sg2 = mk2(sg, sg);
#pragma unroll
      for (int i = 0; i < C::P; ++i) Y[i] = fma2(sg2, Y[i], shfl_xor2(Y[i], 1));
    }
  } else if constexpr (C::TPV == 1) {
    // Real-input split-radix codelet: Y = packed rfft of u.
    float u[C::D], y[C::D];
#pragma unroll
    for (int j = 0; j < C::NW; ++j) {
      const float2 f = half2_bits_to_float2(xw[j]);
      u[2 * j] = f.x;
      u[2 * j + 1] = f.y;
    }
    RFFT<C::D>::fwd(u, y);
#pragma unroll
    for (int k = 0; k < C::P; ++k) Y[k] = mk2(y[2 * k], y[2 * k + 1]);
  } else {
    // Thread pair, d/2 = N complex points, M = N/2 per thread, Q = M/2.
    // Thread t holds z_{2m+t}: in-thread FFT_M gives F_t(k); thread 1 turns
    // F_1(k) into G(k) = W_N^k F_1(k); one exchange gives, per slot k,
    //   k <  Q: thread 0 Z_k = F0 + G,        thread 1 Z_{k+M} = F0 - G,
    //   k >= Q: thread 0 Z_{k+M} = F0 - G,    thread 1 Z_k = F0 + G,
    // so that both threads pair slot k with slot M - k for the real split
    // (only the pair (Q, Q) straddles the threads).
    constexpr int M = C::D / 4;
    constexpr int N = C::D / 2;
    constexpr int Q = M / 2;
    constexpr int LM = ilog2(M);
    f2 z[M];
#pragma unroll
    for (int j = 0; j < M; ++j) {
      const float2 f = half2_bits_to_float2(xw[j]);
      z[j] = mk2(f.x, f.y);
    }
    fft_dif<M, false>(z);
    const float sg = t ? -1.0f : 1.0f;
    const f2 sgA = mk2(sg, sg), sgB = mk2(-sg, -sg);
    static_for<0, M>([&](auto kk) {
      constexpr int k = decltype(kk)::value;
      constexpr int sl = bitrev(k, LM);
      f2 own = z[sl];
      if constexpr (k != 0) {
        if (t) own = twiddle<N, k, false>(own);
      }
      const f2 p = shfl_xor2(own, 1);
      z[sl] = (k < Q) ? fma2(sgA, own, p) : fma2(sgB, p, own);
    });
    {  // slot 0: thread 0 Z_0 -> sqrt2 X_0, sqrt2 X_{d/2}; thread 1 Z_M -> 2 conj Z_M
      const float a = lo2(z[0]), b = hi2(z[0]);
      Y[0] = t ? mk2(2.0f * a, -2.0f * b) : mk2(kSqrt2 * (a + b), kSqrt2 * (a - b));
    }
    static_for<1, Q>([&](auto kk) {
      constexpr int k = decltype(kk)::value;
      const f2 p1 = add2(z[bitrev(k, LM)], z[bitrev(M - k, LM)]);
      const f2 p2 = sub2(z[bitrev(k, LM)], z[bitrev(M - k, LM)]);
      const float sr = lo2(p1), ti = hi2(p1), tr = lo2(p2), si = hi2(p2);
      // thread 0: W_d^k (-i T); thread 1 holds Z_{k+M}: W_d^{k+M} = -i W_d^k,
      // so it applies W_d^k to (-T).
      const float pr = t ? -tr : ti, pi = t ? -ti : -tr;
      constexpr float c = tw_cos(k, C::D), s = tw_sin(k, C::D);
      const float wr = fmaf(c, pr, s * pi), wi = fmaf(c, pi, -(s * pr));
      Y[k] = mk2(sr + wr, si + wi);
      Y[M - k] = mk2(sr - wr, wi - si);
    });
    {  // slot Q: partner across the pair; thread 0 makes X_{Q+M}, thread 1 X_Q
      const f2 own = z[bitrev(Q, LM)];
      const f2 other = shfl_xor2(own, 1);
      const f2 p1 = add2(own, other), p2 = sub2(own, other);
      const float sr = lo2(p1), ti = hi2(p1), tr = lo2(p2), si = hi2(p2);
      const float pr = t ? ti : -tr, pi = t ? -tr : -ti;
      constexpr float c = tw_cos(Q, C::D), s = tw_sin(Q, C::D);
      const float wr = fmaf(c, pr, s * pi), wi = fmaf(c, pi, -(s * pr));
      Y[Q] = mk2(sr + wr, si + wi);
    }
  }
}

// ------------------------------------------------------ inverse rotation ---

// Thread's fp16 words of u = R^T y_hat.  The input is pre-scaled,
// Yin = KAPPA * y_hat, so that the unnormalized inverse transform (the exact
// inverse of rotate_fwd's unnormalized map up to the factor 1/KAPPA^2) yields
// u itself.
template <class C>
__device__ __forceinline__ void rotate_inv(f2 (&Y)[C::P], int t, uint32_t (&xw)[C::NW]) {
  if constexpr (C::ROT == kRotSRHT) {
    if constexpr (C::TPV == 2) {
      const float sg = t ? -1.0f : 1.0f;
      const f2 sg2 = mk2(sg, sg);
#pragma unroll
      for (int i = 0; i < C::P; ++i) Y[i] = fma2(sg2, Y[i], shfl_xor2(Y[i], 1));
    }
    fwht<C::P>(Y);
#pragma unroll
    for (int j = 0; j < C::NW; ++j) xw[j] = float2_to_half2_bits(lo2(Y[j]), hi2(Y[j]));
  } else if constexpr (C::TPV == 1 && C::INV_CODELET) {
    float y[C::D], u[C::D];
#pragma unroll
    for (int k = 0; k < C::P; ++k) {
      y[2 * k] = lo2(Y[k]);
      y[2 * k + 1] = hi2(Y[k]);
    }
    RFFT<C::D>::inv(y, u);
#pragma unroll
    for (int n = 0; n < C::NW; ++n) xw[n] = float2_to_half2_bits(u[2 * n], u[2 * n + 1]);
  } else if constexpr (C::TPV == 1) {
    // Half-length complex inverse FFT after the real pre-split.
    constexpr int N = C::D / 2;
    constexpr int LN = ilog2(N);
    f2 z[N];
    {
      const float a = lo2(Y[0]), b = hi2(Y[0]);
      z[0] = mk2(kSqrt2 * (a + b), kSqrt2 * (a - b));
    }
    // Q_k = (A + B) + i W^{-k} (A - B), A = X'_k, B = conj X'_{N-k}
    static_for<1, N / 2>([&](auto kk) {
      constexpr int k = decltype(kk)::value;
      const f2 p1 = add2(Y[k], Y[N - k]);  // (Sr, Di) with B = conj Y[N-k]
      const f2 p2 = sub2(Y[k], Y[N - k]);  // (Dr, Si)
      const float sr = lo2(p1), di = hi2(p1), dr = lo2(p2), si = hi2(p2);
      constexpr float c = tw_cos(k, C::D), s = tw_sin(k, C::D);
      const float vr = fmaf(c, dr, -(s * di)), vi = fmaf(c, di, s * dr);  // W^{-k} D
      z[k] = mk2(sr - vi, si + vr);      // S + i V
      z[N - k] = mk2(sr + vi, vr - si);  // conj(S - i V)
    });
    z[N / 2] = mk2(2.0f * lo2(Y[N / 2]), -2.0f * hi2(Y[N / 2]));
    fft_dif<N, true>(z);
    static_for<0, N>([&](auto nn) {
      constexpr int n = decltype(nn)::value;
      const f2 v = z[bitrev(n, LN)];
      xw[n] = float2_to_half2_bits(lo2(v), hi2(v));
    });
  } else {
    constexpr int M = C::D / 4;
    constexpr int N = C::D / 2;
    constexpr int Q = M / 2;
    constexpr int LM = ilog2(M);
    f2 z[M];
    {
      const float a = lo2(Y[0]), b = hi2(Y[0]);
      z[0] = t ? mk2(2.0f * a, -2.0f * b) : mk2(kSqrt2 * (a + b), kSqrt2 * (a - b));
    }
    static_for<1, Q>([&](auto kk) {
      constexpr int k = decltype(kk)::value;
      const f2 p1 = add2(Y[k], Y[M - k]);
      const f2 p2 = sub2(Y[k], Y[M - k]);
      const float sr = lo2(p1), di = hi2(p1), dr = lo2(p2), si = hi2(p2);
      constexpr float c = tw_cos(k, C::D), s = tw_sin(k, C::D);
      const float vr = fmaf(c, dr, -(s * di)), vi = fmaf(c, di, s * dr);  // W_d^{-k} D
      // thread 0: Q_k = S + i V, Q_{N-k} = conj(S - i V); thread 1 holds
      // X'_{k+M}: W_d^{-(k+M)} = i W_d^{-k}, so Q = S - V, conj(S + V).
      z[k] = t ? mk2(sr - vr, si - vi) : mk2(sr - vi, si + vr);
      z[M - k] = t ? mk2(sr + vr, -(si + vi)) : mk2(sr + vi, vr - si);
    });
    {  // slot Q: thread 0 holds X'_{Q+M}, thread 1 X'_Q; partner across
      const f2 other = shfl_xor2(Y[Q], 1);
      const f2 p1 = add2(Y[Q], other), p2 = sub2(Y[Q], other);
      const float sr = lo2(p1), di = hi2(p1), dr = lo2(p2), si = hi2(p2);
      constexpr float c = tw_cos(Q, C::D), s = tw_sin(Q, C::D);
      const float vr = fmaf(c, dr, -(s * di)), vi = fmaf(c, di, s * dr);
      z[Q] = t ? mk2(sr - vi, si + vr) : mk2(sr - vr, si - vi);
    }
    // Inverse of the pair exchange: thread 0 forms E_k = Q_k + Q_{k+M},
    // thread 1 O_k = (Q_k - Q_{k+M}) W_N^{-k}.
    const float sg = t ? -1.0f : 1.0f;
    const f2 sgA = mk2(sg, sg);
    static_for<0, M>([&](auto kk) {
      constexpr int k = decltype(kk)::value;
      const f2 own = z[k];
      const f2 p = shfl_xor2(own, 1);
      f2 r = (k < Q) ? fma2(sgA, own, p) : fma2(sgA, p, own);
      if constexpr (k != 0) {
        if (t) r = twiddle<N, k, true>(r);
      }
      z[k] = r;
    });
    fft_dif<M, true>(z);
    static_for<0, M>([&](auto mm) {
      constexpr int m = decltype(mm)::value;
      const f2 v = z[bitrev(m, LM)];
      xw[m] = float2_to_half2_bits(lo2(v), hi2(v));
    });
  }
}

// ------------------------------------------------------ quantize / pack ---

constexpr int kXNone = 0, kXShared = 1, kXCrossHalf = 2, kXAll = 3;

template <class C, int G>
struct Groups {
  static constexpr int GL =
      C::LAYOUT == kLayQuarter ? (G <= C::E / 2 ? G : C::E / 2) : (G <= C::E ? G : C::E);
  static constexpr int NL = C::E / GL;  // local groups (scales) per thread
  static constexpr int NG = C::D / G;   // scales per vector
  static constexpr int X = C::LAYOUT == kLayFull    ? kXNone
                           : C::LAYOUT == kLayHalf  ? (G > C::E ? kXShared : kXNone)
                           : (G <= C::E / 2 ? kXNone : (G == C::D / 2 ? kXCrossHalf : kXAll));
  static_assert(GL % 16 == 0, "group");
};

// Scale index within the vector of local group lg of thread t.
template <class C, int G>
__device__ __forceinline__ int global_group(int t, int lg) {
  using Gr = Groups<C, G>;
  if constexpr (Gr::X == kXNone) return global_y<C>(t, lg * Gr::GL) / G;
  if constexpr (Gr::X == kXCrossHalf) return quarter_of(t, lg) / 2;
  return 0;
}

// Whether thread t stores the scale of local group lg.
template <class C, int G>
__device__ __forceinline__ bool writes_scale(int t, int lg) {
  using Gr = Groups<C, G>;
  if constexpr (Gr::X == kXNone) return true;
  if constexpr (Gr::X == kXAll) return t == 0 && lg == 0;
  return t == 0;
}

template <class C, int G>
__device__ __forceinline__ void quantize(const f2 (&Y)[C::P], uint32_t (&qw)[C::NQ],
                                         float (&sc)[Groups<C, G>::NL]) {
  using Gr = Groups<C, G>;
  constexpr int GP = Gr::GL / 2;  // pairs per local group
  float m[Gr::NL];
#pragma unroll
  for (int g = 0; g < Gr::NL; ++g) m[g] = absmax2<GP>(&Y[g * GP]);
  if constexpr (Gr::X == kXShared) {
    m[0] = fmaxf(m[0], __shfl_xor_sync(kFull, m[0], 1));
  } else if constexpr (Gr::X == kXCrossHalf) {
    const float o0 = __shfl_xor_sync(kFull, m[0], 1), o1 = __shfl_xor_sync(kFull, m[1], 1);
    m[0] = fmaxf(m[0], o1);
    m[1] = fmaxf(m[1], o0);
  } else if constexpr (Gr::X == kXAll) {
    float a = fmaxf(m[0], m[1]);
    a = fmaxf(a, __shfl_xor_sync(kFull, a, 1));
    m[0] = a;
    m[1] = a;
  }
  const f2 magic = mk2(kRoundMagic, kRoundMagic);
#pragma unroll
  for (int g = 0; g < Gr::NL; ++g) {
    const float inv = m[g] > 0.0f ? __fdiv_rn(7.0f, m[g]) : 0.0f;
    sc[g] = m[g] * C::KAPPA7;
    const f2 inv2 = mk2(inv, inv);
#pragma unroll
    for (int w = 0; w < GP / 4; ++w) {
      uint32_t f[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const f2 v = Y[g * GP + 4 * w + i];
        if constexpr (C::CODELET) {  // scalar outputs: no re-pairing moves
          f[2 * i] = __float_as_uint(__fmaf_rn(lo2(v), inv, kRoundMagic));
          f[2 * i + 1] = __float_as_uint(__fmaf_rn(hi2(v), inv, kRoundMagic));
        } else {
          const f2 r = fma2(v, inv2, magic);
          f[2 * i] = __float_as_uint(lo2(r));
          f[2 * i + 1] = __float_as_uint(hi2(r));
        }
      }
      qw[(g * GP) / 4 + w] = pack8(f);
    }
  }
}

// Yin = q * (s * KAPPA), ready for the unnormalized inverse transform.
template <class C, int G>
__device__ __forceinline__ void dequantize(const uint32_t (&qw)[C::NQ],
                                           const float (&sc)[Groups<C, G>::NL],
                                           f2 (&Y)[C::P]) {
  using Gr = Groups<C, G>;
  constexpr int GP = Gr::GL / 2;
  const f2 magic = mk2(kUnpackMagic, kUnpackMagic);
#pragma unroll
  for (int g = 0; g < Gr::NL; ++g) {
    const float sk = sc[g] * C::KAPPA_INV;
    const f2 sk2 = mk2(sk, sk);
#pragma unroll
    for (int w = 0; w < GP / 4; ++w) {
      f2 q[4];
      unpack8(qw[(g * GP) / 4 + w], q);
#pragma unroll
      for (int i = 0; i < 4; ++i) Y[g * GP + 4 * w + i] = mul2(sub2(q[i], magic), sk2);
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
  float* row = scales + vrow * Gr::NG;
  if constexpr (Gr::X == kXNone) {
    // runs of R consecutive scales (two runs per thread in the quarter layout)
    constexpr int R = C::LAYOUT == kLayQuarter ? Gr::NL / 2 : Gr::NL;
#pragma unroll
    for (int r = 0; r < Gr::NL / R; ++r) {
      float* p = row + global_group<C, G>(t, r * R);
      if constexpr (R == 1) {
        p[0] = sc[r];
      } else if constexpr (R == 2) {
        *reinterpret_cast<float2*>(p) = make_float2(sc[2 * r], sc[2 * r + 1]);
      } else {
#pragma unroll
        for (int i = 0; i < R; i += 4)
          *reinterpret_cast<float4*>(p + i) =
              make_float4(sc[r * R + i], sc[r * R + i + 1], sc[r * R + i + 2], sc[r * R + i + 3]);
      }
    }
  } else {
#pragma unroll
    for (int lg = 0; lg < Gr::NL; ++lg)
      if (writes_scale<C, G>(t, lg)) row[global_group<C, G>(t, lg)] = sc[lg];
  }
}

template <class C, int G>
__device__ __forceinline__ void load_scales_smem(uint32_t sbuf, int row, int t,
                                                 float (&sc)[Groups<C, G>::NL]) {
  using Gr = Groups<C, G>;
  const uint32_t a = sbuf + uint32_t(row * Gr::NG) * 4u;
#pragma unroll
  for (int lg = 0; lg < Gr::NL; ++lg)
    sc[lg] = __uint_as_float(lds32(a + 4u * uint32_t(global_group<C, G>(t, lg))));
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

template <int D, int G, int ROT, int TPV, int S_IN, int S_OUT, int MINB>
__global__ void __launch_bounds__(kThreads, MINB)
    kvq_fwd_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmQ,
                   const FwdArgs a, unsigned* status) {
  using C = Cfg<D, ROT, TPV>;
  using Gr = Groups<C, G>;
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
    f2 Y[C::P];
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

template <int D, int G, int ROT, int TPV, int S_IN, int S_OUT, int MINB>
__global__ void __launch_bounds__(kThreads, MINB)
    kvq_inv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmS,
                   const __grid_constant__ CUtensorMap tmX, const InvArgs a, unsigned* status) {
  using C = Cfg<D, ROT, TPV>;
  using Gr = Groups<C, G>;
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
    f2 Y[C::P];
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
template <int D, int G, int ROT, int TPV, int S_IN, int MINB>
__global__ void __launch_bounds__(kThreads, MINB)
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
    f2 Y[C::P];
    rotate_fwd<C>(xw, t, Y);
    uint32_t qw[C::NQ];
    float sc[Gr::NL];
    quantize<C, G>(Y, qw, sc);
    store_codes<C>(qout, row, t, qw);
    const int64_t h = nt * C::VPW + row;
    if (h < a.n_heads) {
      float* p = a.scales + (h * a.cap + a.pos) * Gr::NG;
#pragma unroll
      for (int lg = 0; lg < Gr::NL; ++lg)
        if (writes_scale<C, G>(t, lg)) p[global_group<C, G>(t, lg)] = sc[lg];
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
      const float* p = a.scales + (int64_t(head) * a.cap + r) * Gr::NG;
#pragma unroll
      for (int k = 0; k < Gr::NL; ++k)
        sc[k] = r < a.pos ? __ldg(p + global_group<C, G>(t, k)) : 0.0f;
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
    f2 Y[C::P];
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
template <int D, int ROT, int TPV, int S_IN, int S_OUT>
constexpr int fwd_smem_bytes() {
  using C = Cfg<D, ROT, TPV>;
  return kWarps * (S_IN * C::XTILE + S_OUT * C::QTILE) + 1024;
}

template <int D, int ROT, int TPV, int S_IN>
constexpr int decode_smem_bytes() {
  using C = Cfg<D, ROT, TPV>;
  return kWarps * (S_IN * C::QTILE + 2 * C::XTILE) + 1024;
}

template <int D, int G, int ROT, int TPV, int S_IN, int S_OUT>
constexpr int inv_smem_bytes() {
  using C = Cfg<D, ROT, TPV>;
  constexpr int STILE = C::VPW * (D / G) * 4;
  constexpr int STAGE = C::QTILE + ((STILE + 1023) / 1024) * 1024;
  return kWarps * (S_IN * STAGE + S_OUT * C::XTILE) + 1024;
}

}  // namespace kvq
