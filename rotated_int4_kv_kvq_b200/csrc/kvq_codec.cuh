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
//    stage through warp shuffles when TPV = 2), absmax, round, pack.  The
//    forward flips and widens each fp16 input with one mixed-precision
//    multiply-add by an fp16 +-1 (the inverse XORs the fp16 sign bits of its
//    output words, or folds the signs into its lambda factors).
//  * SRFT: an fp16 word is an (even, odd) sample pair, so one generated
//    two-lane real-FFT codelet in packed fp32x2 transforms both parity halves
//    at once (half the issue slots of a scalar codelet) and a radix-2 join
//    in scalar fp32 completes the spectrum; the inverse mirrors it.
//  * Results are written to a shared tile and stored by TMA (bulk groups);
//    scales are written directly with coalesced vector stores.
//
// Forward ("Fusing four steps into two kernels is not enough": rotate plus
// quantize in one kernel) and inverse (dequantize plus inverse rotate) each
// read their input once and write their output once.
#pragma once

#include "kvq_device.cuh"
#include "kvq_rfft.cuh"

namespace kvq {

// Test builds only: the forward kernel arms the mbarrier of this input tile
// but issues no copy for it, so the wait on it runs out (with nothing in
// flight) and the time-out path is exercised.  -1 (every product build):
// every tile is loaded.
#ifndef KVQ_TEST_SKIP_TILE
#define KVQ_TEST_SKIP_TILE (-1)
#endif

// Round the SRFT join outputs with packed f32x2 multiply-adds (1) or one
// scalar multiply-add per value (0).
#ifndef KVQ_SRFT_QFMA2
#define KVQ_SRFT_QFMA2 1
#endif
// Warp barriers between batches of 8 lambda factor loads in the inverse (1)
// or none (0).
#ifndef KVQ_LAM_FENCE
#define KVQ_LAM_FENCE 1
#endif
// Flip and widen the fp16 inputs with one mixed-precision multiply-add per
// sample (1), or XOR the sign bits and widen (0).
#ifndef KVQ_MIXED_CVT
#define KVQ_MIXED_CVT 1
#endif

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;

// Where a thread's E local rotated coordinates sit in the vector's y:
//  kLayFull    (one thread per vector): local i is y[i].
//  kLayHadamard (SRHT, thread pair):    local half h (E/2 values) of thread
//           t is quarter 2h + t of y: thread 0 holds quarters 0 and 2,
//           thread 1 quarters 1 and 3 (see rotate_fwd).
//  kLayQuarter (SRFT, thread pair):     local half h (E/2 values) of thread t is
//           quarter qd = h ? 3 - 2t : 2t of y, i.e. thread 0 holds quarters
//           0 and 3 and thread 1 quarters 2 and 1.  This is where the pair
//           join of the two half-length real FFTs leaves each output (see
//           pair_join_fwd); both halves are in natural y order.
constexpr int kLayFull = 0, kLayHadamard = 1, kLayQuarter = 2;

template <int D_, int ROT_, int TPV_, int BITS_ = 4>
struct Cfg {
  static constexpr int D = D_;
  static constexpr int ROT = ROT_;
  static constexpr int TPV = TPV_;
  static constexpr int BITS = BITS_;       // code width
  static constexpr int VPW = 32 / TPV;     // vectors per warp tile
  static constexpr int E = D / TPV;        // reals per thread
  static constexpr int P = E / 2;          // float pairs per thread
  static constexpr int NW = E / 2;         // fp16-pair words per thread
  static constexpr int NQ = E * BITS / 32;  // packed-code words per thread
  static constexpr int XTILE = VPW * D * 2;  // fp16 tile bytes
  static constexpr int QTILE = VPW * D * BITS / 8;  // code tile bytes
  // shared-memory stride of a code tile: whole KiB, so that the swizzled
  // tiles placed after it keep the 1024-byte alignment TMA swizzling needs
  static constexpr int QSTRIDE = (QTILE + 1023) / 1024 * 1024;
  static constexpr int SLAB = VPW * 128;   // one 64-column fp16 slab
  static constexpr int QP = D * BITS / 8;  // code row pitch in bytes
  static constexpr int QMAX = (1 << (BITS - 1)) - 1;
  // Code tiles of other widths move as NSLAB swizzled slabs of SW bytes per
  // row (SW = 128, 64 or 32 dividing the row; 0: one unswizzled box of QP),
  // so that rows starting on the same bank do not collide.  4-bit tiles are
  // one box of QP bytes swizzled by their own pitch.
  static constexpr int SW = BITS == 4 ? QP
                            : (QP % 128 == 0 ? 128 : (QP % 64 == 0 ? 64 : (QP % 32 == 0 ? 32 : 0)));
  static constexpr int NSLAB = SW ? QP / SW : 1;
  static constexpr int QSLAB = VPW * (SW ? SW : QP);  // bytes of one slab
  static constexpr int LAYOUT = TPV == 1 ? kLayFull : (ROT == kRotSRFT ? kLayQuarter : kLayHadamard);
  // y = KAPPA_FWD * Y (Y: rotate_fwd's unnormalized output) and the inverse
  // takes Yin = KAPPA_INV * y_hat.  SRFT (Y = packed rfft with X_0, X_{d/2}
  // over sqrt2, from the generated real-FFT codelets, joined across the pair
  // at d = 256; the inverse codelet is the forward one's transpose, half the
  // unnormalized inverse DFT): sqrt(2/d) both ways.  SRHT: 1/sqrt(d) both
  // ways.
  static constexpr bool CODELET = ROT == kRotSRFT && TPV == 1;
  // Thread-pair SRFT: each thread runs a d/2-point real FFT on the even
  // (thread 0) or odd (thread 1) samples; one half-volume exchange joins them.
  static constexpr bool PAIR_RFFT = ROT == kRotSRFT && TPV == 2;
  static constexpr double KAPPA_FWD_D =
      ROT == kRotSRHT ? 1.0 / const_sqrt(double(D)) : const_sqrt(2.0 / D);
  static constexpr double KAPPA_INV_D =
      ROT == kRotSRHT ? 1.0 / const_sqrt(double(D)) : const_sqrt(2.0 / D);
  static constexpr float KAPPA_INV = float(KAPPA_INV_D);
  static constexpr float KAPPA7 = float(KAPPA_FWD_D / QMAX);  // stored scale = m * KAPPA7
  static_assert(D % 64 == 0 && (TPV == 1 || TPV == 2), "shape");
  static_assert(BITS == 3 || BITS == 4 || BITS == 6 || BITS == 8, "code width");
  static_assert(BITS == 4 || QP % 16 == 0, "code rows must be whole 16-byte chunks");
};

template <int D>
struct DefaultTPV {
  static constexpr int value = D >= 256 ? 2 : 1;
};


// Quarter of y holding local half h of thread t (kLayQuarter layout).
__device__ __forceinline__ int quarter_of(int t, int h) { return h ? 3 - 2 * t : 2 * t; }

// y index of local coordinate i of thread t.
template <class C>
__device__ __forceinline__ int global_y(int t, int i) {
  if constexpr (C::LAYOUT == kLayFull) {
    return i;
  } else if constexpr (C::LAYOUT == kLayHadamard) {
    return (2 * (i / (C::E / 2)) + t) * (C::D / 4) + i % (C::E / 2);
  } else {
    return quarter_of(t, i / (C::E / 2)) * (C::D / 4) + i % (C::E / 2);
  }
}

// fp16 sign bits to XOR into word w = (x_{2w}, x_{2w+1}).
__device__ __forceinline__ uint32_t sign_mask_word(const int8_t* signs, int w) {
  return (signs[2 * w] < 0 ? 0x00008000u : 0u) | (signs[2 * w + 1] < 0 ? 0x80000000u : 0u);
}

// Sign mask of word j of thread t as load_x hands it out.  Thread-pair SRFT:
// thread t holds v_m = u_{2m+t} (-1)^{t m}, word j = (v_{2j}, v_{2j+1}); the
// modulation (-1)^m of thread 1 moves its spectrum by d/4 bins.  Otherwise
// thread t holds words t*NW + j; thread-pair SRHT: thread 1's second half
// negated (a sign pattern on the input of a Walsh-Hadamard transform is a
// permutation of its output, see rotate_fwd).
template <class C>
__device__ __forceinline__ uint32_t load_mask_word(const int8_t* signs, int t, int j) {
  if constexpr (C::PAIR_RFFT) {
    const bool lo = signs[4 * j + t] < 0;
    const bool hi = (signs[4 * j + 2 + t] < 0) != (t == 1);
    return (lo ? 0x00008000u : 0u) | (hi ? 0x80000000u : 0u);
  } else {
    uint32_t m = sign_mask_word(signs, t * C::NW + j);
    if (C::ROT == kRotSRHT && C::TPV == 2 && t == 1 && j >= C::NW / 2) m ^= 0x80008000u;
    return m;
  }
}

// Sign mask of word j of thread t as store_x receives it (words t*NW + j),
// including the polarity of the inverse two-lane codelet's outputs.
// Thread-pair SRFT: the odd samples of every odd word arrive negated (see
// rotate_inv).
template <class C>
__device__ __forceinline__ uint32_t store_mask_word(const int8_t* signs, int t, int j) {
  uint32_t m = sign_mask_word(signs, t * C::NW + j);
  // thread-pair SRHT: thread 1's second half arrives negated (rotate_inv)
  if (C::ROT == kRotSRHT && C::TPV == 2 && t == 1 && j >= C::NW / 2) m ^= 0x80008000u;
  if constexpr (C::ROT == kRotSRFT) {
    constexpr uint64_t neg = RFFT2<C::E / 2>::INV_NEG;  // inverse codelet polarity
    if constexpr (C::TPV == 1) {
      if ((neg >> j) & 1u) m ^= 0x80008000u;
    } else {
      // word j = 2i + b holds half b of P_i (own) and of P_{i+NR/4}
      // (partner); thread 1 puts the partner's half first
      const int i = j / 2;
      const bool own = (neg >> i) & 1u, other = (neg >> (i + C::NW / 2)) & 1u;
      const bool lo = t ? other : own, hi = t ? own : other;
      m ^= (lo ? 0x00008000u : 0u) | (hi ? 0x80000000u : 0u);
      if (j & 1) m ^= 0x80000000u;
    }
  }
  return m;
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

// Sign-flipped fp16 word w (samples (lo, hi)) widened to an f32 pair.  With
// KVQ_MIXED_CVT the sign table entry m holds fp16 +-1 pairs and one
// mixed-precision multiply-add per sample flips and widens it; otherwise m
// holds sign-bit masks XOR-ed into the word before a plain widening.
__device__ __forceinline__ f2 signed_pair(uint32_t w, uint32_t m) {
#if KVQ_MIXED_CVT
  return half2_times_signs(w, m);
#else
  const float2 f = half2_bits_to_float2(w ^ m);
  return mk2(f.x, f.y);
#endif
}

// Thread t's words of the row, sign-flipped and widened to f32 pairs.
template <class C>
__device__ __forceinline__ void load_x(uint32_t tile, int row, int t, uint32_t mask,
                                       f2 (&u)[C::NW]) {
  if constexpr (!C::PAIR_RFFT) {
#pragma unroll
    for (int c = 0; c < C::NW / 4; ++c) {
      const int gc = t * (C::NW / 4) + c;  // chunk of the row
      const uint4 v = lds128(tile + (gc / 8) * C::SLAB + sw128(row, gc % 8));
      const uint4 m = lds128(mask + c * 16);
      u[4 * c + 0] = signed_pair(v.x, m.x);
      u[4 * c + 1] = signed_pair(v.y, m.y);
      u[4 * c + 2] = signed_pair(v.z, m.z);
      u[4 * c + 3] = signed_pair(v.w, m.w);
    }
  } else {
    // Both threads of the pair read the whole row; thread t keeps fp16 half
    // t of every word, two words per result: (u_{4j+t}, u_{4j+2+t}).
    const uint32_t sel = t ? 0x7632u : 0x5410u;
#pragma unroll
    for (int c = 0; c < C::D / 16; ++c) {
      const uint4 m = lds128(mask + c * 16);
      const uint4 v0 = lds128(tile + ((2 * c) / 8) * C::SLAB + sw128(row, (2 * c) % 8));
      const uint4 v1 = lds128(tile + ((2 * c + 1) / 8) * C::SLAB + sw128(row, (2 * c + 1) % 8));
      u[4 * c + 0] = signed_pair(__byte_perm(v0.x, v0.y, sel), m.x);
      u[4 * c + 1] = signed_pair(__byte_perm(v0.z, v0.w, sel), m.y);
      u[4 * c + 2] = signed_pair(__byte_perm(v1.x, v1.y, sel), m.z);
      u[4 * c + 3] = signed_pair(__byte_perm(v1.z, v1.w, sel), m.w);
    }
  }
}

// Thread t's words of the output row into the swizzled tile, XOR-ed with
// the store-side sign masks (MASK), or as they are (the lambda path has
// applied the signs in fp32 already).
template <class C, bool MASK = true>
__device__ __forceinline__ void store_x(uint32_t tile, int row, int t, uint32_t mask,
                                        const uint32_t (&xw)[C::NW]) {
#pragma unroll
  for (int c = 0; c < C::NW / 4; ++c) {
    const int gc = t * (C::NW / 4) + c;
    uint4 m = make_uint4(0u, 0u, 0u, 0u);
    if constexpr (MASK) m = lds128(mask + c * 16);
    sts128(tile + (gc / 8) * C::SLAB + sw128(row, gc % 8), xw[4 * c] ^ m.x,
           xw[4 * c + 1] ^ m.y, xw[4 * c + 2] ^ m.z, xw[4 * c + 3] ^ m.w);
  }
}

// 16-byte code chunk of the row holding local code chunk lc of thread t.
template <class C>
__device__ __forceinline__ int code_chunk(int t, int lc) {
  return global_y<C>(t, 32 * lc) / 32;
}

// Codes of the thread's runs of 32 consecutive y coordinates: 4-bit tiles
// are swizzled 16-byte chunks; other widths are plain rows of QP bytes, a run
// of 32 codes being BITS whole words.
template <class C>
__device__ __forceinline__ uint32_t run_byte(int t, int run) {
  return uint32_t(global_y<C>(t, 32 * run) * C::BITS / 8);
}

// Shared address of byte `o` (a multiple of 4) of `row` in a code tile of
// another width.
template <class C>
__device__ __forceinline__ uint32_t code_word(uint32_t tile, int row, uint32_t o) {
  if constexpr (C::SW == 0) {
    return tile + uint32_t(row * C::QP) + o;
  } else {
    const uint32_t s = o / C::SW, b = o % C::SW;
    return tile + s * uint32_t(C::QSLAB) + swq<C::SW>(row, int(b / 16)) + (b % 16);
  }
}

template <class C>
__device__ __forceinline__ void load_codes(uint32_t tile, int row, int t, uint32_t (&qw)[C::NQ]) {
  if constexpr (C::BITS == 4) {
#pragma unroll
    for (int c = 0; c < C::NQ / 4; ++c) {
      const uint4 v = lds128(tile + swq<C::QP>(row, code_chunk<C>(t, c)));
      qw[4 * c] = v.x;
      qw[4 * c + 1] = v.y;
      qw[4 * c + 2] = v.z;
      qw[4 * c + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int r = 0; r < C::E / 32; ++r)
#pragma unroll
      for (int k = 0; k < C::BITS; ++k)
        qw[r * C::BITS + k] = lds32(code_word<C>(tile, row, run_byte<C>(t, r) + 4u * k));
  }
}

template <class C>
__device__ __forceinline__ void store_codes(uint32_t tile, int row, int t,
                                            const uint32_t (&qw)[C::NQ]) {
  if constexpr (C::BITS == 4) {
#pragma unroll
    for (int c = 0; c < C::NQ / 4; ++c)
      sts128(tile + swq<C::QP>(row, code_chunk<C>(t, c)), qw[4 * c], qw[4 * c + 1],
             qw[4 * c + 2], qw[4 * c + 3]);
  } else {
#pragma unroll
    for (int r = 0; r < C::E / 32; ++r)
#pragma unroll
      for (int k = 0; k < C::BITS; ++k)
        sts32(code_word<C>(tile, row, run_byte<C>(t, r) + 4u * k), qw[r * C::BITS + k]);
  }
}

// ------------------------------------------------------ forward rotation ---

constexpr float kSqrt2 = 1.41421356237309504880f;

// Sign of output j of a two-lane codelet (bit j of its polarity mask).
template <uint64_t NEG, int J>
__device__ __forceinline__ constexpr float lane_sign() {
  return ((NEG >> J) & 1u) ? -1.0f : 1.0f;
}

// W_N^K (x + i y) = m (hr + i hi) in the tangent form: with c = cos, s =
// sin of 2 pi K / N and K <= N / 8, m = c and (hr, hi) = (x + t y, y - t x),
// t = s / c; above, m = s and t = c / s.  The caller folds m into the adds
// that follow (fused multiply-adds), so a twiddle costs two operations
// instead of four.
template <int K, int N>
__device__ __forceinline__ void twiddle_tan(float x, float y, float& m, float& hr, float& hi) {
  if constexpr (8 * K <= N) {
    constexpr float t = float(cos_sin_2pi(K, N).s / cos_sin_2pi(K, N).c);
    m = tw_cos(K, N);
    hr = fmaf(t, y, x);
    hi = fmaf(-t, x, y);
  } else {
    constexpr float t = float(cos_sin_2pi(K, N).c / cos_sin_2pi(K, N).s);
    m = tw_sin(K, N);
    hr = fmaf(t, x, y);
    hi = fmaf(t, y, -x);
  }
}

// In-thread radix-2 join.  y2 is RFFT2<N/2>::fwd of the words of an N-point
// real sequence, i.e. the packed spectra E (lane x: even samples) and O
// (lane y: odd samples); Y receives the packed N-point rfft in the codelet
// packing: Y[0] = (X_0, X_{N/2}) / sqrt2, Y[N/4] = X_{N/4}, and
// X_k = E_k + W_N^k O_k, X_{N/2-k} = conj(E_k - W_N^k O_k) in Y[k],
// Y[N/2-k].
// TAN selects the tangent-form twiddle (twiddle_tan); the plain form
// (FMUL + FFMA per product, then the adds) measured faster in the d = 128
// kernel only.
template <int N, bool TAN = true>
__device__ __forceinline__ void join_lanes_fwd(const f2 (&y2)[N / 2], f2 (&Y)[N / 2]) {
  constexpr uint64_t NEG = RFFT2<N / 2>::FWD_NEG;
  {
    const float e0 = lane_sign<NEG, 0>() * lo2(y2[0]), o0 = lane_sign<NEG, 0>() * hi2(y2[0]);
    Y[0] = mk2(e0 + o0, e0 - o0);
    const float eq = lane_sign<NEG, 1>() * lo2(y2[1]), oq = lane_sign<NEG, 1>() * hi2(y2[1]);
    Y[N / 4] = mk2(kSqrt2 * eq, -kSqrt2 * oq);  // E - i O at bin N/4
  }
  static_for<1, N / 4>([&](auto kk) {
    constexpr int k = decltype(kk)::value;
    constexpr float sr = lane_sign<NEG, 2 * k>(), si = lane_sign<NEG, 2 * k + 1>();
    const float er = sr * lo2(y2[2 * k]), orr = sr * hi2(y2[2 * k]);
    const float ei = si * lo2(y2[2 * k + 1]), oi = si * hi2(y2[2 * k + 1]);
    if constexpr (TAN) {
      float m, hr, hi;  // W_N^k O_k = m (hr, hi)
      twiddle_tan<k, N>(orr, oi, m, hr, hi);
      Y[k] = mk2(fmaf(m, hr, er), fmaf(m, hi, ei));
      Y[N / 2 - k] = mk2(fmaf(-m, hr, er), fmaf(m, hi, -ei));
    } else {
      constexpr float c = tw_cos(k, N), s = tw_sin(k, N);
      const float gr = fmaf(c, orr, s * oi), gi = fmaf(c, oi, -(s * orr));  // W_N^k O_k
      Y[k] = mk2(er + gr, ei + gi);
      Y[N / 2 - k] = mk2(er - gr, gi - ei);
    }
  });
}

// Thread-pair join of the two half-length real FFTs (d = 2*NR points).
// On entry y holds this thread's packed NR-point rfft (codelet packing):
// thread 0 the spectrum E of the even samples, thread 1 the spectrum
// V_k = O_{k+NR/2} = conj(O_{NR/2-k}) of its modulated odd samples.  The
// radix-2 step X_k = E_k + W_d^k O_k, X_{NR-k} = conj(E_k - W_d^k O_k) needs
// one value from the partner per output pair: in step a both threads keep
// slot a and send slot NR/2 - a.  Thread 0 then forms X_a and X_{NR-a},
// thread 1 X_{NR/2+a} and X_{NR/2-a} (with W_d^{NR/2-a} O_{NR/2-a} =
// -i conj(W_d^a V_a)), written to slots a (first quarter of its y) and
// NR/2 - a (second quarter) of Y.
template <class C>
__device__ __forceinline__ void pair_join_fwd(const f2 (&y)[C::D / 4], int t, f2 (&Y)[C::P]) {
  constexpr int H = C::D / 4;  // slots per thread
  const bool odd = t != 0;
  {  // a = 0: slot 0 is (Re, Re) of bins 0 and NR/2
    const float own = lo2(y[0]);
    const float r = __shfl_xor_sync(kFull, hi2(y[0]), 1);
    // thread 0: (X_0, X_d/2)/sqrt2 = (E_0 + O_0, E_0 - O_0)/sqrt2;
    // thread 1: X_{d/4} = E_{d/4} - i O_{d/4}
    Y[0] = odd ? mk2(kSqrt2 * r, -kSqrt2 * own) : mk2(own + r, own - r);
  }
  static_for<1, H / 2 + 1>([&](auto aa) {
    constexpr int a = decltype(aa)::value;
    const float ox = lo2(y[a]), oy = hi2(y[a]);
    const float rx = __shfl_xor_sync(kFull, lo2(y[H - a]), 1);
    const float ry = __shfl_xor_sync(kFull, hi2(y[H - a]), 1);
    // thread 0 twiddles conj(received) = O_a, thread 1 its own V_a times
    // -i (W_d^{NR/2+a} = -i W_d^a), i.e. (Im V_a, -Re V_a): the same twiddle
    // code then gives both threads their q / m
    const float tx = odd ? oy : rx, ty = -(odd ? ox : ry);
    const float px = odd ? rx : ox, py = odd ? -ry : oy;  // E (thread 1: conj E)
    float m, qx, qy;  // q = W_d^a t = m (qx, qy)
    twiddle_tan<a, C::D>(tx, ty, m, qx, qy);
    if constexpr (a < H / 2) Y[a] = mk2(fmaf(m, qx, px), fmaf(m, qy, py));
    Y[H - a] = mk2(fmaf(-m, qx, px), fmaf(m, qy, -py));
  });
}

// Y: this thread's E rotated coordinates as P pairs (local order of the
// layout), unnormalized: the true y is KAPPA * Y.  Input: the sign-flipped
// samples of load_x (consumed).
// With LAM, the values are multiplied by the load-side lambda pairs at
// `lam` (shared memory) first.
template <class C, bool LAM = false>
__device__ __forceinline__ void rotate_fwd(f2 (&u)[C::NW], int t, f2 (&Y)[C::P],
                                           uint32_t lam = 0) {
  if constexpr (LAM) {
#pragma unroll
    for (int j = 0; j < C::NW; ++j) u[j] = mul2(u[j], lds_f2(lam + 8u * j));
  }
  if constexpr (C::ROT == kRotSRHT) {
#pragma unroll
    for (int j = 0; j < C::NW; ++j) Y[j] = u[j];
    fwht<C::P>(Y);
    if constexpr (C::TPV == 2) {
      // H_d = [[H, H], [H, -H]] across the pair, exchanging half the data.
      // Thread 1's input carries the sign (-1)^{bit log2(E/2) of n} (its load
      // mask), and a Walsh-Hadamard transform turns that sign pattern into
      // the index shift k -> k ^ E/2 of its output: its first P/2 pairs hold
      // outputs E/2..E-1, the rest 0..E/2-1.  Both threads send pairs
      // P/2..P-1 and keep 0..P/2-1, so each holds (H x_lo)_k and (H x_hi)_k
      // for its quarter of k (thread 0: k < E/2) and forms y_k = lo + hi,
      // y_{k+d/2} = lo - hi; thread 1's difference is hi - lo, negated
      // (quantize takes it back).
      constexpr int H = C::P / 2;
#pragma unroll
      for (int i = 0; i < H; ++i) {
        const f2 own = Y[i], r = shfl_xor2(Y[H + i], 1);
        Y[i] = add2(own, r);
        Y[H + i] = sub2(own, r);
      }
    }
  } else {
    // Each word is (even, odd) sample: one two-lane codelet transforms both
    // parity halves of this thread's E samples, the join makes their rfft.
    f2 y2[C::NW];
    RFFT2<C::E / 2>::fwd(u, y2);
    if constexpr (C::TPV == 1) {
      join_lanes_fwd<C::E, C::D != 128>(y2, Y);
    } else {
      f2 yt[C::P];
      join_lanes_fwd<C::E>(y2, yt);
      pair_join_fwd<C>(yt, t, Y);
    }
  }
}

// ------------------------------------------------------ inverse rotation ---

// Inverse of join_lanes_fwd: from the packed N-point spectrum Y build the
// two-lane input of RFFT2<N/2>::inv, z = (E'', O'') with
// E''_k = X_k + conj X_{N/2-k} and O''_k = W_N^{-k} (X_k - conj X_{N/2-k}),
// so that lane x of the inverse is the unnormalized N-point inverse at the
// even samples and lane y at the odd samples.
template <int N>
__device__ __forceinline__ void split_lanes_inv(const f2 (&Y)[N / 2], f2 (&z)[N / 2]) {
  {
    const float a = lo2(Y[0]), b = hi2(Y[0]);
    z[0] = mk2(a + b, a - b);
    z[1] = mk2(kSqrt2 * lo2(Y[N / 4]), -kSqrt2 * hi2(Y[N / 4]));
  }
  static_for<1, N / 4>([&](auto kk) {
    constexpr int k = decltype(kk)::value;
    const float xr = lo2(Y[k]), xi = hi2(Y[k]);
    const float mr = lo2(Y[N / 2 - k]), mi = hi2(Y[N / 2 - k]);
    const float dr = xr - mr, di = xi + mi;
    constexpr float c = tw_cos(k, N), s = tw_sin(k, N);
    z[2 * k] = mk2(xr + mr, fmaf(c, dr, -(s * di)));
    z[2 * k + 1] = mk2(xi - mi, fmaf(c, di, s * dr));
  });
}

// Inverse of pair_join_fwd, up to a factor 2 folded into KAPPA_INV: from the
// two quarters of y_hat this thread holds, rebuild its half-length spectrum
// (thread 0: E; thread 1: V, additionally multiplied by (-1)^k so that its
// inverse FFT comes out rotated by NR/2 samples, see rotate_inv).  In step a
// both threads form S = h0 + conj(h1) and D = h0 - conj(h1) from their pair
// (h0, h1); thread 0 keeps E_a = S and sends conj(O_a) = W_d^a conj(D),
// thread 1 keeps i conj(W_d^a conj(D)) and sends conj(S) = E_{NR/2-a}.
template <class C>
__device__ __forceinline__ void pair_join_inv(const f2 (&Y)[C::P], int t, f2 (&Z)[C::D / 4]) {
  constexpr int H = C::D / 4;
  const bool odd = t != 0;
  {  // a = 0
    const float hx = lo2(Y[0]), hy = hi2(Y[0]);
    const float keep = odd ? -kSqrt2 * hy : hx + hy;
    const float send = odd ? kSqrt2 * hx : hx - hy;
    Z[0] = mk2(keep, __shfl_xor_sync(kFull, send, 1));
  }
  static_for<1, H / 2 + 1>([&](auto aa) {
    constexpr int a = decltype(aa)::value;
    const float h1x = lo2(Y[H - a]), h1y = hi2(Y[H - a]);
    float h0x, h0y;
    if constexpr (a < H / 2) {
      h0x = lo2(Y[a]);
      h0y = hi2(Y[a]);
    } else {  // the pair of slot NR/4 straddles the threads
      h0x = __shfl_xor_sync(kFull, h1x, 1);
      h0y = __shfl_xor_sync(kFull, h1y, 1);
    }
    const float sx = h0x + h1x, sy = h0y - h1y;
    const float dx = h0x - h1x, dy = h0y + h1y;
    constexpr float sg = (a & 1) ? -1.0f : 1.0f;  // (-1)^a, thread 1's rotation
    constexpr float c = sg * tw_cos(a, C::D), s = sg * tw_sin(a, C::D);
    const float mx = fmaf(c, dx, -(s * dy)), my = -fmaf(c, dy, s * dx);
    const float kx = odd ? my : sx, ky = odd ? mx : sy;
    if constexpr (a < H / 2) {
      const float ex = odd ? sx : mx, ey = odd ? -sy : my;
      Z[H - a] = mk2(__shfl_xor_sync(kFull, ex, 1), __shfl_xor_sync(kFull, ey, 1));
    }
    Z[a] = mk2(kx, ky);
  });
}

// Thread's fp16 words of u = R^T y_hat.  The input is pre-scaled,
// Yin = KAPPA * y_hat, so that the unnormalized inverse transform (the exact
// inverse of rotate_fwd's unnormalized map up to the factor 1/KAPPA^2) yields
// u itself.  Words of a two-lane codelet output that carry polarity -1 are
// corrected by the store-side sign mask.
// With LAM, the values are multiplied by the store-side factor pairs at
// `lam` (shared memory: sign / lambda, see fill_lambda) before the fp16
// rounding, and the store path applies no sign mask.
template <class C, bool LAM = false>
__device__ __forceinline__ void rotate_inv(f2 (&Y)[C::P], int t, uint32_t (&xw)[C::NW],
                                           uint32_t lam = 0) {
  auto scaled = [&](f2 v, int j) {
    if constexpr (LAM) v = mul2(v, lds_f2(lam + 8u * j));
    return float2_to_half2_bits(lo2(v), hi2(v));
  };
  // With LAM, a warp barrier after every 8 converted words: shared-memory
  // loads are not moved across it, so at most 8 lambda pairs are live at a
  // time (loaded all at once, they pushed the register demand into spills).
  auto fence = [&](int j) {
    if constexpr (LAM && KVQ_LAM_FENCE) {
      if (j % 8 == 7) __syncwarp();
    }
  };
  if constexpr (C::ROT == kRotSRHT) {
    if constexpr (C::TPV == 2) {
      // Inverse of rotate_fwd's pair step: from a = y_k, b = y_{k+d/2} of
      // this thread's quarter of k, thread 0 keeps the sums a + b and sends
      // the differences a - b, thread 1 the other way round; thread 0 then
      // holds y_lo + y_hi in order, thread 1 y_lo - y_hi with its halves
      // swapped, whose transform carries the sign (-1)^{bit log2(E/2) of m}
      // (taken back by its store mask).
      constexpr int H = C::P / 2;
      const float sg = t ? -1.0f : 1.0f;
      const f2 sg2 = mk2(sg, sg), nsg2 = mk2(-sg, -sg);
#pragma unroll
      for (int i = 0; i < H; ++i) {
        const f2 a = Y[i], b = Y[H + i];
        Y[i] = fma2(sg2, b, a);
        Y[H + i] = shfl_xor2(fma2(nsg2, b, a), 1);
      }
    }
    fwht<C::P>(Y);
#pragma unroll
    for (int j = 0; j < C::NW; ++j) {
      xw[j] = scaled(Y[j], j);
      fence(j);
    }
  } else {
    f2 z[C::NW], x2[C::NW];
    if constexpr (C::TPV == 1) {
      split_lanes_inv<C::E>(Y, z);
    } else {
      f2 zt[C::D / 4];
      pair_join_inv<C>(Y, t, zt);
      split_lanes_inv<C::E>(zt, z);
    }
    RFFT2<C::E / 2>::inv(z, x2);
    if constexpr (C::TPV == 1) {
#pragma unroll
      for (int n = 0; n < C::NW; ++n) {
        xw[n] = scaled(x2[n], n);
        fence(n);
      }
    } else {
      // Thread 0 holds the even samples e_m, thread 1 r_m = (-1)^m o_{m+NR/2}
      // (o: odd samples), as fp16 pairs P_i = (s_{2i}, s_{2i+1}).  Both keep
      // P_i and send P_{i+NR/4} (i < NR/4); thread t assembles words
      // t*NR/2 + 2i, 2i + 1 of x; the odd word's odd sample arrives negated
      // (fixed by the sign mask).
      const uint32_t se = t ? 0x1054u : 0x5410u, so = t ? 0x3276u : 0x7632u;
#pragma unroll
      for (int i = 0; i < C::NW / 2; ++i) {
        const uint32_t own = scaled(x2[i], i);
        const uint32_t r = __shfl_xor_sync(kFull, scaled(x2[i + C::NW / 2], i + C::NW / 2), 1);
        fence(2 * i + 1);
        xw[2 * i] = __byte_perm(own, r, se);
        xw[2 * i + 1] = __byte_perm(own, r, so);
      }
    }
  }
}

// ------------------------------------------------------ quantize / pack ---

// How a group's absmax is formed: kXNone within the thread, kXCrossHalf
// local half h of one thread with local half 1 - h of the other, kXPaired
// local half h of both threads, kXAll the whole vector over the pair.
constexpr int kXNone = 0, kXCrossHalf = 1, kXPaired = 2, kXAll = 3;

template <class C, int G>
struct Groups {
  static constexpr int GL =
      C::LAYOUT == kLayFull ? (G <= C::E ? G : C::E) : (G <= C::E / 2 ? G : C::E / 2);
  static constexpr int NL = C::E / GL;  // local groups (scales) per thread
  static constexpr int NG = C::D / G;   // scales per vector
  static constexpr int X =
      C::LAYOUT == kLayFull
          ? kXNone
          : (G <= C::E / 2 ? kXNone
                           : (G == C::D / 2 ? (C::LAYOUT == kLayQuarter ? kXCrossHalf : kXPaired)
                                            : kXAll));
  static_assert(GL % 16 == 0, "group");
};

// Scale index within the vector of local group lg of thread t.
template <class C, int G>
__device__ __forceinline__ int global_group(int t, int lg) {
  using Gr = Groups<C, G>;
  if constexpr (Gr::X == kXNone) return global_y<C>(t, lg * Gr::GL) / G;
  if constexpr (Gr::X == kXCrossHalf) return quarter_of(t, lg) / 2;
  if constexpr (Gr::X == kXPaired) return lg;
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

// Codes and scales of thread t's values Y.  Thread-pair SRHT: thread 1's
// second local half holds -y (rotate_fwd), quantized with the sign taken
// back.
template <class C, int G>
__device__ __forceinline__ void quantize(const f2 (&Y)[C::P], uint32_t (&qw)[C::NQ],
                                         float (&sc)[Groups<C, G>::NL], int t) {
  using Gr = Groups<C, G>;
  constexpr int GP = Gr::GL / 2;  // pairs per local group
  float m[Gr::NL];
#pragma unroll
  for (int g = 0; g < Gr::NL; ++g) m[g] = absmax2<GP>(&Y[g * GP]);
  if constexpr (Gr::X == kXPaired) {
#pragma unroll
    for (int g = 0; g < Gr::NL; ++g) m[g] = fmaxf(m[g], __shfl_xor_sync(kFull, m[g], 1));
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
    float inv = m[g] > 0.0f ? __fdiv_rn(float(C::QMAX), m[g]) : 0.0f;
    if constexpr (C::LAYOUT == kLayHadamard) {
      if (t == 1 && g >= Gr::NL / 2) inv = -inv;
    }
    sc[g] = m[g] * C::KAPPA7;
    const f2 inv2 = mk2(inv, inv);
    if constexpr (C::BITS != 4) {
      // runs of 32 codes -> BITS words of a little-endian bitstream
#pragma unroll
      for (int r = 0; r < GP / 16; ++r) {
        uint32_t f[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const f2 v = Y[g * GP + 16 * r + i];
          f[2 * i] = __float_as_uint(__fmaf_rn(lo2(v), inv, kRoundMagic));
          f[2 * i + 1] = __float_as_uint(__fmaf_rn(hi2(v), inv, kRoundMagic));
        }
        uint32_t w[C::BITS];
        packb<C::BITS>(f, w);
#pragma unroll
        for (int k = 0; k < C::BITS; ++k) qw[((g * GP) / 16 + r) * C::BITS + k] = w[k];
      }
      continue;
    }
#pragma unroll
    for (int w = 0; w < GP / 4; ++w) {
      uint32_t f[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const f2 v = Y[g * GP + 4 * w + i];
        if constexpr (C::ROT == kRotSRFT && !KVQ_SRFT_QFMA2) {  // scalar join outputs
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
    if constexpr (C::BITS != 4) {
#pragma unroll
      for (int r = 0; r < GP / 16; ++r) {
        uint32_t w[C::BITS];
#pragma unroll
        for (int k = 0; k < C::BITS; ++k) w[k] = qw[((g * GP) / 16 + r) * C::BITS + k];
        float q[32];
        unpackb<C::BITS>(w, q);
#pragma unroll
        for (int i = 0; i < 16; ++i) Y[g * GP + 16 * r + i] = mul2(mk2(q[2 * i], q[2 * i + 1]), sk2);
      }
      continue;
    }
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
  const float* lambda;  // per-channel factors (LAM kernels only)
  float* scales;
  int64_t n_vec;
  int64_t n_tiles;
};

struct InvArgs {
  const int8_t* signs;
  const float* lambda;  // per-channel factors (LAM kernels only)
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

// Per-channel factor (lambda) of the fp32 values a thread holds, as pairs in
// the order of its words: load side (word j of load_x) and store side (the
// pairs rotate_inv converts to fp16 itself).  Thread-pair SRFT: thread t's
// load word j holds channels (4j + t, 4j + 2 + t); on the store side thread
// 0 converts e_m = x_{2m} and thread 1 r_m = +-x_{2((m + NR/2) mod NR) + 1}.
template <class C>
__device__ __forceinline__ void lambda_channels(int t, int j, bool store, int& c0, int& c1) {
  if constexpr (C::PAIR_RFFT) {
    if (!store) {
      c0 = 4 * j + t;
      c1 = 4 * j + 2 + t;
    } else if (t == 0) {
      c0 = 4 * j;
      c1 = 4 * j + 2;
    } else {
      constexpr int NR = C::E;
      c0 = 2 * ((2 * j + NR / 2) % NR) + 1;
      c1 = 2 * ((2 * j + 1 + NR / 2) % NR) + 1;
    }
  } else {
    c0 = 2 * (t * C::NW + j);
    c1 = c0 + 1;
  }
}

// Store-side factor of lane l (0: low, 1: high sample) of pair p that thread
// role tp converts to fp16 in rotate_inv: the sign the store mask would
// apply to that sample (D and the inverse codelet's output polarity) over
// lambda of its channel.  Thread-pair SRFT: pairs p < NW/2 stay with the
// thread and land in words 2p + l of its half of the row (low half for
// thread 0, high half for thread 1); pairs p >= NW/2 go to the partner as
// its words 2(p - NW/2) + l (high half for thread 0, low half for thread 1).
template <class C>
__device__ __forceinline__ float store_factor(const int8_t* signs, const float* lambda, int tp,
                                              int p, int l) {
  int t = tp, w = p, h = l;
  if constexpr (C::PAIR_RFFT) {
    const bool own = p < C::NW / 2;
    t = own ? tp : 1 - tp;
    w = 2 * (own ? p : p - C::NW / 2) + l;
    h = own ? (t == 0 ? 0 : 1) : (t == 0 ? 1 : 0);
  }
  const uint32_t m = store_mask_word<C>(signs, t, w);
  const bool neg = (m >> (h ? 31 : 15)) & 1u;
  const float inv = 1.0f / lambda[2 * (t * C::NW + w) + h];
  return neg ? -inv : inv;
}

// s_lam[0, d/2): lambda pairs of the load side, s_lam[d/2, d): the
// store-side factor pairs (sign / lambda, see store_factor), NW pairs per
// thread role t.  With lambda the store path applies the signs through these
// factors in fp32 and skips the fp16 sign-bit XOR.
template <class C>
__device__ __forceinline__ void fill_lambda(const int8_t* signs, const float* lambda, f2* s_lam) {
  for (int i = threadIdx.x; i < C::D / 2; i += blockDim.x) {
    const int t = i / C::NW, j = i % C::NW;
    int c0, c1;
    lambda_channels<C>(t, j, false, c0, c1);
    s_lam[i] = mk2(lambda[c0], lambda[c1]);
    s_lam[C::D / 2 + i] = mk2(store_factor<C>(signs, lambda, t, j, 0),
                              store_factor<C>(signs, lambda, t, j, 1));
  }
}

// s_mask[0, d/2): load-side masks, s_mask[d/2, d): store-side masks, each
// as NW words per thread role t.
template <class C>
__device__ __forceinline__ void fill_sign_masks(const int8_t* signs, uint32_t* s_mask) {
  for (int i = threadIdx.x; i < C::D / 2; i += blockDim.x) {
    const int t = i / C::NW, j = i % C::NW;
    // load side: sign-bit masks, or fp16 +-1 pairs for the mixed-precision
    // flip (0x3C00 = 1.0, 0xBC00 = -1.0)
    s_mask[i] = load_mask_word<C>(signs, t, j) ^ (KVQ_MIXED_CVT ? 0x3C003C00u : 0u);
    s_mask[C::D / 2 + i] = store_mask_word<C>(signs, t, j);
  }
}

template <class C, int G>
__device__ __forceinline__ void store_scales_global(float* scales, int64_t vrow, int t,
                                                    const float (&sc)[Groups<C, G>::NL]) {
  using Gr = Groups<C, G>;
  float* row = scales + vrow * Gr::NG;
  if constexpr (Gr::X == kXNone) {
    // runs of R consecutive scales (two runs per thread in the pair layouts)
    constexpr int R = C::LAYOUT == kLayFull ? Gr::NL : Gr::NL / 2;
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

template <int D, int G, int ROT, int TPV, int S_IN, int S_OUT, int MINB, bool LAM = false,
          int BITS = 4>
__global__ void __launch_bounds__(kThreads, MINB)
    kvq_fwd_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmQ,
                   const FwdArgs a, unsigned* status) {
  using C = Cfg<D, ROT, TPV, BITS>;
  using Gr = Groups<C, G>;
  constexpr int WARP_BYTES = S_IN * C::XTILE + S_OUT * C::QSTRIDE;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars_sm[kWarps][S_IN];
  __shared__ __align__(16) uint32_t s_mask[C::D];
  __shared__ __align__(16) f2 s_lam[LAM ? C::D : 1];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = C::TPV == 2 ? (lane & 1) : 0;
  const int row = C::TPV == 2 ? (lane >> 1) : lane;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t xbuf = base + uint32_t(warp * WARP_BYTES);
  const uint32_t qbuf = xbuf + uint32_t(S_IN * C::XTILE);
  const uint32_t bars = smem_u32(&bars_sm[warp][0]);

  fill_sign_masks<C>(a.signs, s_mask);
  if constexpr (LAM) fill_lambda<C>(a.signs, a.lambda, s_lam);
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
  const uint32_t lam = smem_u32(s_lam) + uint32_t(t * C::NW * 8);

  const int64_t gw = int64_t(blockIdx.x) * kWarps + warp;
  const int64_t nw = int64_t(gridDim.x) * kWarps;
  Ring ring{0, 0};
  auto issue = [&](int64_t tile) {  // lane 0 only
    const int s = int(ring.issued % S_IN);
    const uint32_t bar = bars + 8u * s;
    const uint32_t dst = xbuf + uint32_t(s * C::XTILE);
    mbar_arrive_expect_tx(bar, C::XTILE);
    if (KVQ_TEST_SKIP_TILE < 0 || tile != KVQ_TEST_SKIP_TILE) {
#pragma unroll
      for (int j = 0; j < C::D / 64; ++j)
        tma_load_2d(dst + j * C::SLAB, &tmX, bar, 64 * j, int(tile * C::VPW));
    }
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
    f2 u[C::NW];
    load_x<C>(xbuf + uint32_t(s * C::XTILE), row, t, mask, u);
    __syncwarp();
    if (lane == 0) {
      const int64_t nt = tile + int64_t(S_IN) * nw;
      if (nt < a.n_tiles) {
        fence_proxy_async_smem();
        issue(nt);
      }
    }
    f2 Y[C::P];
    rotate_fwd<C, LAM>(u, t, Y, lam);
    uint32_t qw[C::NQ];
    float sc[Gr::NL];
    quantize<C, G>(Y, qw, sc, t);

    const int o = int((ring.consumed - 1) % S_OUT);
    if (lane == 0) bulk_wait_read<S_OUT - 1>();
    __syncwarp();
    const uint32_t qdst = qbuf + uint32_t(o * C::QSTRIDE);
    store_codes<C>(qdst, row, t, qw);
    const int64_t vrow = tile * C::VPW + row;
    if (vrow < a.n_vec) store_scales_global<C, G>(a.scales, vrow, t, sc);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
#pragma unroll
      for (int sl = 0; sl < C::NSLAB; ++sl)
        tma_store_2d(&tmQ, qdst + uint32_t(sl * C::QSLAB), sl * C::SW, int(tile * C::VPW));
      bulk_commit();
    }
  }
  if (lane == 0) {
    bulk_wait_all();
    if (failed) drain_and_fail<S_IN>(bars, ring, status);
  }
}

template <int D, int G, int ROT, int TPV, int S_IN, int S_OUT, int MINB, bool LAM = false,
          int BITS = 4>
__global__ void __launch_bounds__(kThreads, MINB)
    kvq_inv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmS,
                   const __grid_constant__ CUtensorMap tmX, const InvArgs a, unsigned* status) {
  using C = Cfg<D, ROT, TPV, BITS>;
  using Gr = Groups<C, G>;
  constexpr int STILE = C::VPW * Gr::NG * 4;
  constexpr int STAGE = C::QSTRIDE + ((STILE + 1023) / 1024) * 1024;
  constexpr int WARP_BYTES = S_IN * STAGE + S_OUT * C::XTILE;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars_sm[kWarps][S_IN];
  __shared__ __align__(16) uint32_t s_mask[C::D];
  __shared__ __align__(16) f2 s_lam[LAM ? C::D : 1];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = C::TPV == 2 ? (lane & 1) : 0;
  const int row = C::TPV == 2 ? (lane >> 1) : lane;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t ibuf = base + uint32_t(warp * WARP_BYTES);
  const uint32_t xbuf = ibuf + uint32_t(S_IN * STAGE);
  const uint32_t bars = smem_u32(&bars_sm[warp][0]);

  fill_sign_masks<C>(a.signs, s_mask);
  if constexpr (LAM) fill_lambda<C>(a.signs, a.lambda, s_lam);
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
  const uint32_t mask_st = smem_u32(s_mask) + uint32_t((C::D / 2 + t * C::NW) * 4);
  const uint32_t lam_st = smem_u32(s_lam) + uint32_t((C::D / 2 + t * C::NW) * 8);

  const int64_t gw = int64_t(blockIdx.x) * kWarps + warp;
  const int64_t nw = int64_t(gridDim.x) * kWarps;
  Ring ring{0, 0};
  auto issue = [&](int64_t tile) {
    const int s = int(ring.issued % S_IN);
    const uint32_t bar = bars + 8u * s;
    const uint32_t dst = ibuf + uint32_t(s * STAGE);
    mbar_arrive_expect_tx(bar, C::QTILE + STILE);
#pragma unroll
    for (int sl = 0; sl < C::NSLAB; ++sl)
      tma_load_2d(dst + uint32_t(sl * C::QSLAB), &tmQ, bar, sl * C::SW, int(tile * C::VPW));
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
    rotate_inv<C, LAM>(Y, t, xw, lam_st);

    const int o = int((ring.consumed - 1) % S_OUT);
    if (lane == 0) bulk_wait_read<S_OUT - 1>();
    __syncwarp();
    const uint32_t xdst = xbuf + uint32_t(o * C::XTILE);
    store_x<C, !LAM>(xdst, row, t, mask_st, xw);
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
  __shared__ __align__(16) uint32_t s_mask[C::D];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = C::TPV == 2 ? (lane & 1) : 0;
  const int row = C::TPV == 2 ? (lane >> 1) : lane;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t ibuf = base + uint32_t(warp * WARP_BYTES);
  const uint32_t xbuf = ibuf + uint32_t(S_IN * STAGE);
  const uint32_t bars = smem_u32(&bars_sm[warp][0]);
  const uint32_t bar_new = bars + 8u * S_IN;

  pdl_wait();  // no global access before the previous kernel completes
  fill_sign_masks<C>(a.signs, s_mask);
  if (lane == 0) {
    for (int s = 0; s <= S_IN; ++s) mbar_init(bars + 8u * s, 1);
    fence_mbar_init();
  }
  __syncthreads();
  const uint32_t mask = smem_u32(s_mask) + uint32_t(t * C::NW * 4);
  const uint32_t mask_st = mask + uint32_t(C::D / 2 * 4);
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
    f2 u[C::NW];
    load_x<C>(xin, row, t, mask, u);
    f2 Y[C::P];
    rotate_fwd<C>(u, t, Y);
    uint32_t qw[C::NQ];
    float sc[Gr::NL];
    quantize<C, G>(Y, qw, sc, t);
    store_codes<C>(qout, row, t, qw);
    const int64_t h = nt * C::VPW + row;
    if (h < a.n_heads) {
      float* p = a.scales + (h * a.cap + a.pos) * Gr::NG;
#pragma unroll
      for (int lg = 0; lg < Gr::NL; ++lg)
        if (writes_scale<C, G>(t, lg)) p[global_group<C, G>(t, lg)] = sc[lg];
    }
    dequantize<C, G>(qw, sc, Y);
    uint32_t xw[C::NW];
    rotate_inv<C>(Y, t, xw);
    store_x<C>(xout, row, t, mask_st, xw);
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
    store_x<C>(xdst, row, t, mask_st, xw);
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
  pdl_release();
  if (lane == 0) {
    bulk_wait_all();
    if (failed) drain_and_fail<S_IN>(bars, ring, status);
  }
}

// Dynamic shared memory each kernel needs (plus 1 KiB alignment slack).
template <int D, int ROT, int TPV, int S_IN, int S_OUT, int BITS = 4>
constexpr int fwd_smem_bytes() {
  using C = Cfg<D, ROT, TPV, BITS>;
  return kWarps * (S_IN * C::XTILE + S_OUT * C::QSTRIDE) + 1024;
}

template <int D, int ROT, int TPV, int S_IN>
constexpr int decode_smem_bytes() {
  using C = Cfg<D, ROT, TPV>;
  return kWarps * (S_IN * C::QTILE + 2 * C::XTILE) + 1024;
}

template <int D, int G, int ROT, int TPV, int S_IN, int S_OUT, int BITS = 4>
constexpr int inv_smem_bytes() {
  using C = Cfg<D, ROT, TPV, BITS>;
  constexpr int STILE = C::VPW * (D / G) * 4;
  constexpr int STAGE = C::QSTRIDE + ((STILE + 1023) / 1024) * 1024;
  return kWarps * (S_IN * STAGE + S_OUT * C::XTILE) + 1024;
}

}  // namespace kvq
