// kvq_device.cuh -- device building blocks of libkvq (sm_100a).
//
// * PTX wrappers for mbarriers, TMA tensor copies and bulk-group waits.
// * Compile-time twiddle factors (cos/sin of 2 pi k / n in double, rounded
//   once to float) so that every FFT constant is an instruction immediate.
// * Packed fp32x2 arithmetic (f2) and the register-resident Walsh-Hadamard
//   butterfly network; the real FFTs are generated codelets (kvq_rfft.cuh).
// * int4 quantize / pack and unpack / dequantize on 32-bit words.
//
// The method these pieces implement is described in include/kvq.h.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <type_traits>

// Decode-path kernels use programmatic dependent launch (0 disables it).
#ifndef KVQ_PDL
#define KVQ_PDL 1
#endif

namespace kvq {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kRotSRFT = 0;
constexpr int kRotSRHT = 1;

// 1.5 * 2^23: adding it to |t| < 2^22 rounds t to the nearest integer (ties
// to even, the float32 default rounding) and leaves that integer, in two's
// complement, in the low mantissa bits.
constexpr float kRoundMagic = 12582912.0f;
// 2^23 + 8: a float whose bits are 0x4B0000uu equals 2^23 + uu; subtracting
// this gives uu - 8, i.e. the code of an offset-binary nibble uu = q + 8.
constexpr float kUnpackMagic = 8388616.0f;

// ------------------------------------------------------------ constexpr ---

template <int B, int E, typename F>
__device__ __forceinline__ void static_for(F&& f) {
  if constexpr (B < E) {
    f(std::integral_constant<int, B>{});
    static_for<B + 1, E>(f);
  }
}

constexpr int ilog2(int n) {
  int l = 0;
  while ((1 << l) < n) ++l;
  return l;
}

constexpr double kPi = 3.14159265358979323846264338327950288;

// Taylor series, |x| <= pi/4: the first omitted term is below 1e-27.
constexpr double taylor_sin(double x) {
  double x2 = x * x, term = x, sum = x;
  for (int n = 1; n < 13; ++n) {
    term *= -x2 / double((2 * n) * (2 * n + 1));
    sum += term;
  }
  return sum;
}

constexpr double taylor_cos(double x) {
  double x2 = x * x, term = 1.0, sum = 1.0;
  for (int n = 1; n < 13; ++n) {
    term *= -x2 / double((2 * n - 1) * (2 * n));
    sum += term;
  }
  return sum;
}

// cos(2 pi k / n), sin(2 pi k / n) with exact quadrant/octant reduction on
// integers, so e.g. k/n = 1/4 gives exactly (0, 1).
struct CS {
  double c, s;
};

constexpr CS cos_sin_2pi(long k, long n) {
  k %= n;
  if (k < 0) k += n;
  const long q = (4 * k) / n;  // quadrant
  const long r = 4 * k - q * n;  // angle within quadrant = (pi/2) r / n
  double c = 1.0, s = 0.0;
  if (2 * r <= n) {
    const double a = 0.5 * kPi * double(r) / double(n);
    c = taylor_cos(a);
    s = taylor_sin(a);
  } else {
    const double a = 0.5 * kPi * double(n - r) / double(n);
    c = taylor_sin(a);
    s = taylor_cos(a);
  }
  switch (q) {
    case 0: return CS{c, s};
    case 1: return CS{-s, c};
    case 2: return CS{-c, -s};
    default: return CS{s, -c};
  }
}

constexpr float tw_cos(long k, long n) { return float(cos_sin_2pi(k, n).c); }
constexpr float tw_sin(long k, long n) { return float(cos_sin_2pi(k, n).s); }

constexpr double const_sqrt(double x) {  // Newton on a positive argument
  double r = x > 1.0 ? x : 1.0;
  for (int i = 0; i < 200; ++i) r = 0.5 * (r + x / r);
  return r;
}

static_assert(tw_cos(1, 4) == 0.0f && tw_sin(1, 4) == 1.0f, "quarter turn");
static_assert(tw_cos(1, 2) == -1.0f && tw_sin(1, 2) == 0.0f, "half turn");
static_assert(cos_sin_2pi(1, 8).c - 0.70710678118654752 < 4e-16 &&
                  cos_sin_2pi(1, 8).c - 0.70710678118654752 > -4e-16,
              "eighth turn");
static_assert(cos_sin_2pi(1, 6).c - 0.5 < 4e-16 && cos_sin_2pi(1, 6).c - 0.5 > -4e-16,
              "sixth turn");
static_assert(cos_sin_2pi(1, 12).s - 0.5 < 4e-16 && cos_sin_2pi(1, 12).s - 0.5 > -4e-16,
              "twelfth turn");

// ------------------------------------------------------------------ PTX ---

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Limits of a bounded wait: wall time (ns) and number of polls.
#ifndef KVQ_WAIT_LIMIT_NS
#define KVQ_WAIT_LIMIT_NS 2000000000ull
#endif
#ifndef KVQ_WAIT_MAX_POLLS
#define KVQ_WAIT_MAX_POLLS (1u << 26)
#endif

// Wait for phase `parity` of an mbarrier, giving up after KVQ_WAIT_LIMIT_NS
// (~2 s) or KVQ_WAIT_MAX_POLLS polls.  Returns false on time-out; callers
// record the error and stop.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1; it < KVQ_WAIT_MAX_POLLS; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 1023u) == 0 && global_timer_ns() - t0 > KVQ_WAIT_LIMIT_NS) return false;
  }
  return false;
}

__device__ __forceinline__ void tma_load_1d(uint32_t dst, const CUtensorMap* tm, uint32_t bar,
                                            int c0) {
  asm volatile(
      "cp.async.bulk.tensor.1d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(bar), "r"(c0)
      : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* tm, uint32_t bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* tm, uint32_t bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* tm, uint32_t src, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(tm)),
      "r"(src), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* tm, uint32_t src, int c0, int c1,
                                             int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(tm)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Programmatic dependent launch.  A kernel launched with programmatic
// stream serialization may start while the kernel before it in the stream is
// still finishing; pdl_wait() returns once that kernel has completed and its
// memory operations are visible (at once for a launch without the
// attribute), so every global access of such a kernel comes after it.
// pdl_release() lets the next kernel of the stream begin launching its
// blocks once every block of this one has released or exited; it does not
// make any of this kernel's results visible to it.  The decode-path kernels
// release after their main loop: released at kernel entry, the next
// kernel's blocks were placed while this one's were still running and the
// 26-call decode step measured slower at some lengths (1025 rows: 88 us
// against 76 us released late, 86 us without the attribute).
__device__ __forceinline__ void pdl_wait() {
#if KVQ_PDL
  asm volatile("griddepcontrol.wait;" ::: "memory");
#endif
}
__device__ __forceinline__ void pdl_release() {
#if KVQ_PDL
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#endif
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* tm) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tm)) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a));
  return v;
}

__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}

__device__ __forceinline__ void sts128(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w)
               : "memory");
}

__device__ __forceinline__ void sts32(uint32_t a, uint32_t x) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(x) : "memory");
}

// ------------------------------------------------------------- numerics ---

__device__ __forceinline__ float2 half2_bits_to_float2(uint32_t w) {
  __half2 h = *reinterpret_cast<__half2*>(&w);
  return __half22float2(h);
}

__device__ __forceinline__ uint32_t float2_to_half2_bits(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);  // round to nearest even, both lanes
  return *reinterpret_cast<uint32_t*>(&h);
}

// A pair of floats in one 64-bit register pair, operated on by the sm_100
// packed fp32 instructions (add/sub/mul/fma .rn.f32x2).  Complex numbers are
// held as (re, im).
struct f2 {
  uint64_t v;
};

__device__ __forceinline__ f2 mk2(float x, float y) {
  f2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r.v) : "f"(x), "f"(y));
  return r;
}

// The fp16 pair w times the fp16 pair m (+-1 each), widened to f32: one
// mixed-precision multiply-add per half (f16 x f16 + f32 -> f32, exact for a
// sign), adding -0 so that a -0 product stays -0.
__device__ __forceinline__ f2 half2_times_signs(uint32_t w, uint32_t m) {
  float lo, hi;
  asm("{\n\t.reg .b16 a0, a1, s0, s1;\n\t"
      "mov.b32 {a0, a1}, %2;\n\t"
      "mov.b32 {s0, s1}, %3;\n\t"
      "fma.rn.f32.f16 %0, a0, s0, 0f80000000;\n\t"
      "fma.rn.f32.f16 %1, a1, s1, 0f80000000;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(w), "r"(m));
  return mk2(lo, hi);
}
// An f2 from shared memory (8-byte aligned address).
__device__ __forceinline__ f2 lds_f2(uint32_t a) {
  const uint2 v = lds64(a);
  return mk2(__uint_as_float(v.x), __uint_as_float(v.y));
}

__device__ __forceinline__ float lo2(f2 a) {
  float x;
  asm("mov.b64 {%0, _}, %1;" : "=f"(x) : "l"(a.v));
  return x;
}
__device__ __forceinline__ float hi2(f2 a) {
  float y;
  asm("mov.b64 {_, %0}, %1;" : "=f"(y) : "l"(a.v));
  return y;
}
__device__ __forceinline__ f2 add2(f2 a, f2 b) {
  f2 r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r.v) : "l"(a.v), "l"(b.v));
  return r;
}
__device__ __forceinline__ f2 sub2(f2 a, f2 b) {
  f2 r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r.v) : "l"(a.v), "l"(b.v));
  return r;
}
__device__ __forceinline__ f2 mul2(f2 a, f2 b) {
  f2 r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r.v) : "l"(a.v), "l"(b.v));
  return r;
}
__device__ __forceinline__ f2 fma2(f2 a, f2 b, f2 c) {
  f2 r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r.v) : "l"(a.v), "l"(b.v), "l"(c.v));
  return r;
}
__device__ __forceinline__ f2 shfl_xor2(f2 a, int m) {
  return mk2(__shfl_xor_sync(kFull, lo2(a), m), __shfl_xor_sync(kFull, hi2(a), m));
}

// max(a, b, c) in one instruction (three-operand max of sm_100).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// In-place unnormalized Walsh-Hadamard transform (Sylvester order) of the
// 2P reals held as P pairs (element 2p in lo, 2p+1 in hi).
template <int P>
__device__ __forceinline__ void fwht(f2 (&v)[P]) {
#pragma unroll
  for (int p = 0; p < P; ++p) {  // h = 1: inside each pair
    const float a = lo2(v[p]), b = hi2(v[p]);
    v[p] = mk2(a + b, a - b);
  }
  static_for<0, ilog2(P)>([&](auto st) {  // h = 2, 4, ...: between pairs
    constexpr int h = 1 << decltype(st)::value;
#pragma unroll
    for (int p = 0; p < P; ++p) {
      if ((p & h) == 0) {
        const f2 a = v[p], b = v[p + h];
        v[p] = add2(a, b);
        v[p + h] = sub2(a, b);
      }
    }
  });
}

// Max of |x| over the 2P reals held in v[0..P).
template <int P>
__device__ __forceinline__ float absmax2(const f2* v) {
  static_assert(P % 2 == 0, "pairs");
  float m0 = fmaxf(fabsf(lo2(v[0])), fabsf(hi2(v[0])));
  float m1 = fmaxf(fabsf(lo2(v[1])), fabsf(hi2(v[1])));
#pragma unroll
  for (int p = 2; p < P; p += 2) {
    m0 = max3f(m0, fabsf(lo2(v[p])), fabsf(hi2(v[p])));
    m1 = max3f(m1, fabsf(lo2(v[p + 1])), fabsf(hi2(v[p + 1])));
  }
  return fmaxf(m0, m1);
}

// Eight round-to-int bit patterns (low byte = code) -> 8 packed nibbles:
// byte j = (q_{2j} & 0xF) | (q_{2j+1} << 4).
__device__ __forceinline__ uint32_t pack8(const uint32_t (&f)[8]) {
  const uint32_t e = __byte_perm(__byte_perm(f[0], f[2], 0x0040), __byte_perm(f[4], f[6], 0x0040),
                                 0x5410);
  const uint32_t o = __byte_perm(__byte_perm(f[1], f[3], 0x0040), __byte_perm(f[5], f[7], 0x0040),
                                 0x5410);
  return (e & 0x0F0F0F0Fu) | ((o << 4) & 0xF0F0F0F0u);
}

// Codes of a packed word, as 4 pairs of offset floats 2^23 + 8 + q
// (element order: pair j = codes 2j, 2j+1).
__device__ __forceinline__ void unpack8(uint32_t w, f2 (&q)[4]) {
  const uint32_t lo = (w & 0x0F0F0F0Fu) ^ 0x08080808u;
  const uint32_t hi = ((w >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    q[j] = mk2(__uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7650 + j)),
               __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7650 + j)));
}

// Codes of a packed word as 4 pairs of exact signed floats (pair j = codes
// 2j, 2j+1).  One logic op puts two nibbles into an fp16 pair (1032 + q for
// a low nibble, 1152 + 16 q for a high one), and one mixed-precision
// multiply-add per code (f16 x f16 + f32 -> f32, exact) removes the offset:
// five integer and eight floating-point instructions per word, where
// unpack8 and a packed subtraction take eleven integer and four.
__device__ __forceinline__ void unpack8_signed(uint32_t w, f2 (&q)[4]) {
  const uint32_t w8 = w >> 8;
  const uint32_t l0 = (w & 0x000F000Fu) ^ 0x64086408u;   // codes 0, 4
  const uint32_t h0 = (w & 0x00F000F0u) ^ 0x64806480u;   // codes 1, 5
  const uint32_t l1 = (w8 & 0x000F000Fu) ^ 0x64086408u;  // codes 2, 6
  const uint32_t h1 = (w8 & 0x00F000F0u) ^ 0x64806480u;  // codes 3, 7
  float c0, c1, c2, c3, c4, c5, c6, c7;
  asm("{\n\t.reg .b16 a0, a1, b0, b1, d0, d1, e0, e1, one, s16;\n\t"
      "mov.b16 one, 0x3C00;\n\t"
      "mov.b16 s16, 0x2C00;\n\t"
      "mov.b32 {a0, a1}, %8;\n\t"
      "mov.b32 {b0, b1}, %9;\n\t"
      "mov.b32 {d0, d1}, %10;\n\t"
      "mov.b32 {e0, e1}, %11;\n\t"
      "fma.rn.f32.f16 %0, a0, one, 0fC4810000;\n\t"
      "fma.rn.f32.f16 %1, b0, s16, 0fC2900000;\n\t"
      "fma.rn.f32.f16 %2, d0, one, 0fC4810000;\n\t"
      "fma.rn.f32.f16 %3, e0, s16, 0fC2900000;\n\t"
      "fma.rn.f32.f16 %4, a1, one, 0fC4810000;\n\t"
      "fma.rn.f32.f16 %5, b1, s16, 0fC2900000;\n\t"
      "fma.rn.f32.f16 %6, d1, one, 0fC4810000;\n\t"
      "fma.rn.f32.f16 %7, e1, s16, 0fC2900000;\n\t}"
      : "=f"(c0), "=f"(c1), "=f"(c2), "=f"(c3), "=f"(c4), "=f"(c5), "=f"(c6), "=f"(c7)
      : "r"(l0), "r"(h0), "r"(l1), "r"(h1));
  q[0] = mk2(c0, c1);
  q[1] = mk2(c2, c3);
  q[2] = mk2(c4, c5);
  q[3] = mk2(c6, c7);
}

// 32 codes (the low BITS bits of each magic-rounded float, two's
// complement) as BITS words of a little-endian bitstream: code i occupies
// bits [BITS i, BITS i + BITS).
template <int B>
__device__ __forceinline__ void packb(const uint32_t (&f)[32], uint32_t (&w)[B]) {
  if constexpr (B == 8) {
#pragma unroll
    for (int k = 0; k < 8; ++k)
      w[k] = __byte_perm(__byte_perm(f[4 * k], f[4 * k + 1], 0x0040),
                         __byte_perm(f[4 * k + 2], f[4 * k + 3], 0x0040), 0x5410);
  } else {
    constexpr uint32_t mask = (1u << B) - 1u;
#pragma unroll
    for (int k = 0; k < B; ++k) w[k] = 0u;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const uint32_t c = f[i] & mask;
      const int pos = B * i, wi = pos / 32, sh = pos % 32;
      w[wi] |= c << sh;
      if (sh + B > 32) w[wi + 1] |= c >> (32 - sh);
    }
  }
}

// Inverse of packb: the 32 codes as exact floats.
template <int B>
__device__ __forceinline__ void unpackb(const uint32_t (&w)[B], float (&q)[32]) {
  constexpr uint32_t mask = (1u << B) - 1u;
  constexpr uint32_t sign = 1u << (B - 1);
  // offset binary (c ^ sign) in the low mantissa bits of 2^23
  constexpr float off = 8388608.0f + float(1 << (B - 1));
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int pos = B * i, wi = pos / 32, sh = pos % 32;
    uint32_t c;
    if (sh + B > 32) {
      c = __funnelshift_r(w[wi], w[wi + 1], sh);
    } else {
      c = w[wi] >> sh;
    }
    c = (c & mask) ^ sign;
    q[i] = __uint_as_float(c | 0x4B000000u) - off;
  }
}

}  // namespace kvq
