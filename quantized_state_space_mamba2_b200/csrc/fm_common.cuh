// fm_common.cuh -- device-side arithmetic shared by the library's kernels.
//
// Fixed-point conventions (FastMamba, arXiv 2505.18975: power-of-two scales
// and an 8-segment first-order approximation of 2^v, pith.science review,
// "What carries the argument"; word widths and rounding are this library's
// reading, stated in include/fastmamba.h):
//   rshr(a, s) = floor((a + 2^(s-1)) / 2^s) for s > 0, a for s = 0,
//                a * 2^-s for s < 0;   satb(a, b) = clamp(a, +-(2^(b-1)-1)).
// All fp32 stages are written with explicit _rn intrinsics (and the library
// is built with -fmad=false) so that no multiply-add is contracted.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace fm {

// Device error word (per device, per process): 0 = ok; bit 0 = a bounded
// wait gave up; bit 1 = a non-finite value reached an int8 quantiser.  Read
// and cleared by fm_sync_status().  The library is one translation unit
// (fm_lib.cu includes every kernel header), so the definition lives here.
__device__ unsigned int g_error_word = 0;
constexpr unsigned int kErrTimeout = 1u;
constexpr unsigned int kErrNonfinite = 2u;

__device__ __forceinline__ void raise_error(unsigned int bits) { atomicOr(&g_error_word, bits); }

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start while its predecessor in the stream drains; it
// waits here, before its first global memory access, until the predecessor
// has completed and its writes are visible.  Without that launch attribute
// this returns at once.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// ... and lets the next kernel in the stream be scheduled as soon as every
// CTA of this one has started (all of them resident, so the dependents' CTAs
// can only take resources this grid no longer needs); the dependents still
// wait for this grid's completion before touching memory.
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- integers
__device__ __forceinline__ long long rshr64(long long a, int s) {
  if (s > 0) return (a + (1LL << (s - 1))) >> s;  // >> on signed is arithmetic (floor)
  if (s == 0) return a;
  return a * (1LL << (-s));
}

__device__ __forceinline__ long long satb64(long long a, int bits) {
  const long long lim = (1LL << (bits - 1)) - 1;
  return a > lim ? lim : (a < -lim ? -lim : a);
}

// a * 2^k for k >= 0, saturated to +-2^61
__device__ __forceinline__ long long shl_sat61(long long a, int k) {
  const long long LIM = 1LL << 61;
  long long m = a < 0 ? -a : a;
  if (k >= 61 || m > (LIM >> k)) return a < 0 ? -LIM : LIM;
  return a * (1LL << k);
}

// a 2^k with saturation at 2^61 for k >= 0, rshr(a, -k) for k < 0
__device__ __forceinline__ long long pow2_sat61(long long a, int k) {
  return k >= 0 ? shl_sat61(a, k) : rshr64(a, -k);
}

// fp32 -> nearest integer (half to even) clamped to +-lim (NaN -> -lim)
__device__ __forceinline__ int round_clamp(float v, float lim) {
  float r = rintf(v);
  r = fmaxf(r, -lim);
  r = fminf(r, lim);
  return (int)r;
}

// fp32 -> Q.16 int32: clamp(rint(x * 2^16), +-(2^31-1)), NaN -> 0.  One
// round-to-nearest-even conversion (it saturates to [-2^31, 2^31-1] and maps
// NaN to 0), then the symmetric lower bound.
__device__ __forceinline__ int to_q16(float x) {
  return max(__float2int_rn(__fmul_rn(x, 65536.0f)), -2147483647);
}

// The exact float of an integer |v| < 2^22 without the conversion unit:
// 1.5 * 2^23 + v is exact in fp32, and so is the subtraction.
__device__ __forceinline__ float small_i2f(int v) {
  return __fsub_rn(__int_as_float(0x4B400000 + v), 12582912.0f);
}

// The int8 quantiser's rounding: rint(v) clamped to +-127 (NaN -> -127).  The
// clamp commutes with rint for an integer bound; adding 1.5 * 2^23 then
// rounds to the nearest integer (ties to even) in the fp32 add itself.
__device__ __forceinline__ int quant127(float v) {
  const float c = fminf(fmaxf(v, -127.0f), 127.0f);
  return __float_as_int(__fadd_rn(c, 12582912.0f)) - 0x4B400000;
}

// ---------------------------------------------------------------- 2^v unit
// 8 chords of 2^f on [0,1): P_i = rint(2^16 * 2^(i/8)) (i = 0..8), slopes
// S_i = P_(i+1) - P_i, so the curve is exact at every 2^(integer) and
// continuous at segment ends.
__device__ __forceinline__ int pwl_P(int i) {
  // rint(65536 * 2^(i/8)) for i = 0..7
  constexpr int P[8] = {65536, 71468, 77936, 84990, 92682, 101070, 110218, 120194};
  return P[i];
}
__device__ __forceinline__ int pwl_S(int i) {
  // P_(i+1) - P_i with P_8 = 131072
  constexpr int S[8] = {5932, 6468, 7054, 7692, 8388, 9148, 9976, 10878};
  return S[i];
}
constexpr long long kLog2eQ15 = 47274;  // rint(2^15 * log2(e)) = rint(47274.23...)

// The unit below is written in 32-bit integer arithmetic only (32x32->64
// multiplies are several times slower on this GPU); every split is exact.

// 2^(w / 2^16) in Q.16 for w <= 0 (w > 0 is treated as 0); result in [0, 2^16].
// With n = floor(w / 2^16) the integer part is a right shift by k = -n; k >= 32
// (w < -31 * 2^16) gives 0.
__device__ __forceinline__ int pow2_pwl32(int w) {
  if (w > 0) w = 0;
  if (w < -(31 << 16)) return 0;
  const int n = w >> 16;               // floor, in [-31, 0]
  const int f = w & 0xFFFF;
  const int i = f >> 13;
  const int r = f & 8191;
  const int m = pwl_P(i) + ((pwl_S(i) * r + 4096) >> 13);  // < 2^17
  const int k = -n;
  if (k == 0) return m;
  return (m + (1 << (k - 1))) >> k;
}

__device__ __forceinline__ int pow2_pwl(long long w) {
  return w < -(31LL << 16) ? 0 : pow2_pwl32((int)(w > 0 ? 0 : w));
}

// e^(x / 2^16) in Q.16 for x <= 0 (x > 0 is treated as 0):
// 2^rshr(x log2e_Q15, 15).  For |x| >= 2^21 the exponent is below -31 * 2^16
// (result 0); otherwise |x| = ah 2^15 + al and
// rshr(-|x| L, 15) = -ah L + ((2^14 - al L) >> 15), all within int32.
__device__ __forceinline__ int exp_pwl(long long x) {
  if (x >= 0) return 65536;
  if (x <= -(1LL << 21)) return 0;
  const int ax = (int)(-x);
  const int ah = ax >> 15, al = ax & 0x7FFF;
  const int w = -ah * (int)kLog2eQ15 + ((16384 - al * (int)kLog2eQ15) >> 15);
  return pow2_pwl32(w);
}

// SoftPlus: x <= 0 -> e^x; x > 0 -> x + e^-x; clamped to 2^31 - 1
__device__ __forceinline__ int softplus_pwl(int v) {
  long long r = v <= 0 ? (long long)exp_pwl(v) : (long long)v + exp_pwl(-(long long)v);
  return r > 2147483647LL ? 2147483647 : (int)r;
}

// ---------------------------------------------------------------- fast forms
// The same functions for element-wise kernels: the 8 chords are read from a
// shared-memory table (per-lane indices would serialise on the constant
// cache) as (P_i 2^13 + 2^12, S_i), so that one multiply-add and one shift give
// P_i + rshr(S_i r, 13) (P_i 2^13 is a multiple of 2^13; the sum stays below
// 2^31); the SiLU division uses a reciprocal estimate with an exact integer
// correction.  Bit-identical to the forms above.
__device__ __forceinline__ void pwl_table_init(int2 *tab) {
  if (threadIdx.x < 8 && threadIdx.y == 0)
    tab[threadIdx.x] = make_int2(pwl_P(threadIdx.x) * 8192 + 4096, pwl_S(threadIdx.x));
}

// e^-|x| in Q.16 (|x| in Q.16): w = rshr(-|x| log2e_Q15, 15) as in exp_pwl,
// then 2^(w / 2^16) from the table (segment (w >> 13) & 7 and offset w & 8191
// are those of w's fraction w mod 2^16).  |x| is capped at 2^21 (w is then
// below -31 * 2^16), and the rounding shift by k = -floor(w / 2^16) is capped
// at 31, where m + 2^30 < 2^31 already rounds to 0 -- no branches.
__device__ __forceinline__ unsigned exp_neg_abs_t(int x, const int2 *tab) {
  const unsigned ux = x < 0 ? 0u - (unsigned)x : (unsigned)x;
  const int ax = (int)min(ux, 1u << 21);
  const int ah = ax >> 15, al = ax & 0x7FFF;
  const int w = -ah * (int)kLog2eQ15 + ((16384 - al * (int)kLog2eQ15) >> 15);  // <= 0
  const int k = min(-(w >> 16), 31);
  const int2 e = tab[(w >> 13) & 7];
  const unsigned m = ((unsigned)e.y * (unsigned)(w & 8191) + (unsigned)e.x) >> 13;
  return (m + ((1u << k) >> 1)) >> k;
}

// SiLU(x / 2^16) in Q.16 for x in +-(2^31 - 1): sigma from E = e^-|x|;
// x >= 0: floor(2^32 / (2^16 + E)), x < 0: floor(E 2^16 / (2^16 + E));
// result rshr(x sigma, 16) = xh sigma + ((xl sigma + 2^15) >> 16) with
// x = xh 2^16 + xl, xl in [0, 2^16) (both products fit 32 bits).
// One floor division serves both signs: with d = 2^16 + E and q = floor(2^32 / d),
// E 2^16 / d = 2^16 - 2^32 / d, so floor(E 2^16 / d) = 2^16 - ceil(2^32 / d)
// = 2^16 - q - [d does not divide 2^32], and d in [2^16, 2^17] divides 2^32
// only for E = 0 or E = 2^16.  The division: d and 2^32 are exact floats;
// 2^32 rcp(d), truncated, is within 2^-5 of the quotient (a few ulp of
// relative error on a quotient below 2^17), so one correction from the exact
// remainder (mod 2^32) gives the floor.  The float conversions avoid the
// conversion unit (small_i2f and a round-to-zero add of 2^23).
__device__ __forceinline__ int silu_pwl_t(int x, const int2 *tab) {
  const unsigned E = exp_neg_abs_t(x, tab);
  const unsigned d = 65536u + E;
  float rd;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(rd) : "f"(small_i2f((int)d)));
  unsigned q = __float_as_uint(__fadd_rz(__fmul_rz(4294967296.0f, rd), 8388608.0f)) - 0x4B000000u;
  const unsigned rem = 0u - q * d;  // 2^32 - q d (mod 2^32)
  if ((int)rem < 0) q -= 1u;
  else if (rem >= d) q += 1u;
  const unsigned sig = x >= 0 ? q : 65536u - q - ((E - 1u) < 65535u ? 1u : 0u);
  const int xh = x >> 16;
  const unsigned xl = (unsigned)x & 0xFFFFu;
  return xh * (int)sig + (int)((xl * sig + 32768u) >> 16);
}

// rshr(v, k) for int32 v and k in [1, 31] without overflow: floor(v / 2^k) +
// the bit below (round half up)
__device__ __forceinline__ int rshr32(int v, int k) { return (v >> k) + ((v >> (k - 1)) & 1); }

// ---------------------------------------------------------------- PoT exponent
// smallest integer e with a <= Q 2^e (exact), a <= 0 -> -30
__device__ __forceinline__ int pot_exponent(double a, double Q) {
  if (!(a > 0.0)) return -30;
  int e = (int)ceil(log2(a / Q));
  while (a > ldexp(Q, e)) ++e;
  while (a <= ldexp(Q, e - 1)) --e;
  return e;
}

// ---------------------------------------------------------------- warp helpers
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ long long warp_sum_ll(long long v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// In-register FWHT of one 256-block held as 8 consecutive values per lane
// (element i = 8*lane + r): stages s = 0..2 inside the lane, s = 3..7 across
// lanes (xor 1..16), ascending; (a, b) -> (a + b, a - b); then * 1/16.
template <typename T>
__device__ __forceinline__ void fwht256_lane8(T (&v)[8], int lane) {
#pragma unroll
  for (int s = 0; s < 3; ++s) {
    const int h = 1 << s;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i & h) continue;
      T a = v[i], b = v[i + h];
      v[i] = a + b;
      v[i + h] = a - b;
    }
  }
#pragma unroll
  for (int s = 0; s < 5; ++s) {
    const int m = 1 << s;
    // lower lane: v + other, upper lane: other - v; both are other + sg v with
    // sg = +-1 (sg v is exact, so the fused form rounds the same single sum)
    const T sg = (lane & m) ? T(-1) : T(1);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const T other = __shfl_xor_sync(0xffffffffu, v[i], m);
      v[i] = fma(sg, v[i], other);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = v[i] * (T)0.0625;
}

}  // namespace fm
