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
// wait gave up.  Read and cleared by fm_sync_status().  The library is one
// translation unit (fm_lib.cu includes every kernel header), so the
// definition lives here.
__device__ unsigned int g_error_word = 0;
constexpr unsigned int kErrTimeout = 1u;

__device__ __forceinline__ void raise_error(unsigned int bits) { atomicOr(&g_error_word, bits); }

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

// fp32 -> nearest integer (half to even) clamped to +-lim (NaN -> -lim)
__device__ __forceinline__ int round_clamp(float v, float lim) {
  float r = rintf(v);
  r = fmaxf(r, -lim);
  r = fminf(r, lim);
  return (int)r;
}

// fp32 -> Q.16 int32: clamp(rint(x * 2^16), +-(2^31-1)), NaN -> 0
__device__ __forceinline__ int to_q16(float x) {
  if (x != x) return 0;
  float r = rintf(__fmul_rn(x, 65536.0f));
  if (r >= 2147483648.0f) return 2147483647;
  if (r <= -2147483648.0f) return -2147483647;
  return (int)r;
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

// 2^(w / 2^16) in Q.16 for w <= 0 (w > 0 is treated as 0); result in [0, 2^16]
__device__ __forceinline__ int pow2_pwl(long long w) {
  if (w > 0) w = 0;
  long long n = w >> 16;              // floor
  int f = (int)(w - n * 65536);       // [0, 65535]
  int i = f >> 13;
  int r = f & 8191;
  int m = pwl_P(i) + ((pwl_S(i) * r + 4096) >> 13);  // < 2^17
  long long k = -n;
  if (k >= 32) return 0;
  if (k == 0) return m;
  int kk = (int)k;
  return (int)(((long long)m + (1LL << (kk - 1))) >> kk);
}

// e^(x / 2^16) in Q.16 for x <= 0
__device__ __forceinline__ int exp_pwl(long long x) {
  if (x > 0) x = 0;
  return pow2_pwl(rshr64(x * kLog2eQ15, 15));
}

// SoftPlus: x <= 0 -> e^x; x > 0 -> x + e^-x; clamped to 2^31 - 1
__device__ __forceinline__ int softplus_pwl(int v) {
  long long r = v <= 0 ? (long long)exp_pwl(v) : (long long)v + exp_pwl(-(long long)v);
  return r > 2147483647LL ? 2147483647 : (int)r;
}

// SiLU(x / 2^16) in Q.16: sigma from E = e^-|x|; x >= 0: floor(2^32 / (2^16 + E)),
// x < 0: floor(E 2^16 / (2^16 + E)); result rshr(x * sigma, 16).
__device__ __forceinline__ long long silu_pwl(int x) {
  long long ax = x < 0 ? -(long long)x : (long long)x;
  unsigned E = (unsigned)exp_pwl(-ax);
  unsigned d = 65536u + E;  // [2^16, 2^17]
  unsigned sig;
  if (x >= 0) {
    sig = 0xFFFFFFFFu / d;           // floor((2^32 - 1) / d)
    if ((d & (d - 1u)) == 0u) sig += 1u;  // d divides 2^32
  } else if (E >= 65536u) {
    sig = 32768u;                    // 2^32 / 2^17
  } else {
    sig = (E << 16) / d;
  }
  long long prod = (long long)x * (long long)sig;
  return (prod + 32768LL) >> 16;
}

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
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      T other = __shfl_xor_sync(0xffffffffu, v[i], m);
      v[i] = upper ? (other - v[i]) : (v[i] + other);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = v[i] * (T)0.0625;
}

}  // namespace fm
