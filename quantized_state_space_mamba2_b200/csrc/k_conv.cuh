// k_conv.cuh -- power-of-two causal depthwise conv1d (kernel 4) + PWL SiLU.
//
// FastMamba (arXiv 2505.18975): fine-grained power-of-two quantisation of the
// convolution layer (pith.science review, "What carries the argument";
// original abstract); SiLU (Swish, the paper's reference [11]) through the
// shared 2^v approximation unit.  Per channel c and token t:
//   acc = bq[c] + sum_{k=0..3} wq[c,k] u[t-3+k, c]           (int32, exact)
//   x16 = satb(rshr(acc, -(e_w + e_u + 16)), 32)             (to Q.16)
//   out = satb(rshr(SiLU_pwl(x16), e_o + 16), 8)
//
// Layout: each thread owns 8 consecutive channels (8-byte loads/stores, a
// warp covers 256 contiguous bytes of a token row) and walks TCH tokens with
// the 3-token history in registers, so every input byte is read once (plus a
// 3-token halo per chunk).  Grid: (channel groups, token chunks, batch).
#pragma once
#include "fm_common.cuh"

namespace fm {

constexpr int kConvCPT = 8;    // channels per thread
constexpr int kConvThreads = 128;

__device__ __forceinline__ void unpack8(uint2 w, int (&v)[8]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = (int)(int8_t)((w.x >> (8 * i)) & 0xFF);
#pragma unroll
  for (int i = 0; i < 4; ++i) v[4 + i] = (int)(int8_t)((w.y >> (8 * i)) & 0xFF);
}

// amax (nullable, [cc] u32): max |SiLU output| per channel (calibration).
__global__ void __launch_bounds__(kConvThreads) k_conv1d_pot(
    const int8_t *__restrict__ u, int T, int cc, int tch, const int8_t *__restrict__ wq,
    const int32_t *__restrict__ bq, const int32_t *__restrict__ exps, int8_t *conv_state,
    int write_state, int8_t *__restrict__ out, unsigned int *amax) {
  const int c0 = (blockIdx.x * kConvThreads + threadIdx.x) * kConvCPT;
  if (c0 >= cc) return;
  const int b = blockIdx.z;
  const int t0 = blockIdx.y * tch;
  const int t1 = min(T, t0 + tch);
  const int32_t *e_u = exps, *e_w = exps + cc, *e_o = exps + 2 * cc;

  int w[kConvCPT][4], bias[kConvCPT], s_in[kConvCPT], s_out[kConvCPT];
#pragma unroll
  for (int j = 0; j < kConvCPT; ++j) {
    const uint32_t wp = *reinterpret_cast<const uint32_t *>(wq + (long long)(c0 + j) * 4);
#pragma unroll
    for (int k = 0; k < 4; ++k) w[j][k] = (int)(int8_t)((wp >> (8 * k)) & 0xFF);
    bias[j] = bq[c0 + j];
    s_in[j] = -(e_w[c0 + j] + e_u[c0 + j] + 16);
    s_out[j] = e_o[c0 + j] + 16;
  }
  // history h[0] = t-3, h[1] = t-2, h[2] = t-1
  int h[3][kConvCPT];
  const long long rowstride = cc;
  const int8_t *ub = u + (long long)b * T * rowstride;
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const int tt = t0 - 3 + k;
    uint2 raw = make_uint2(0u, 0u);
    if (tt >= 0)
      raw = *reinterpret_cast<const uint2 *>(ub + (long long)tt * rowstride + c0);
    else if (conv_state)
      raw = *reinterpret_cast<const uint2 *>(conv_state + ((long long)b * 3 + (3 + tt)) * cc + c0);
    unpack8(raw, h[k]);
  }
  unsigned int am[kConvCPT];
#pragma unroll
  for (int j = 0; j < kConvCPT; ++j) am[j] = 0u;

  for (int t = t0; t < t1; ++t) {
    int cur[kConvCPT];
    unpack8(*reinterpret_cast<const uint2 *>(ub + (long long)t * rowstride + c0), cur);
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int j = 0; j < kConvCPT; ++j) {
      const int acc = bias[j] + w[j][0] * h[0][j] + w[j][1] * h[1][j] + w[j][2] * h[2][j] +
                      w[j][3] * cur[j];
      const int x16 = (int)satb64(rshr64((long long)acc, s_in[j]), 32);
      const long long s = silu_pwl(x16);
      if (amax) {
        const unsigned int a = (unsigned int)(s < 0 ? -s : s);
        am[j] = a > am[j] ? a : am[j];
      }
      const uint32_t code = (uint32_t)((int)satb64(rshr64(s, s_out[j]), 8) & 0xFF);
      if (j < 4) lo |= code << (8 * j);
      else hi |= code << (8 * (j - 4));
      h[0][j] = h[1][j];
      h[1][j] = h[2][j];
      h[2][j] = cur[j];
    }
    *reinterpret_cast<uint2 *>(out + ((long long)b * T + t) * rowstride + c0) = make_uint2(lo, hi);
  }
  if (amax) {
#pragma unroll
    for (int j = 0; j < kConvCPT; ++j) atomicMax(amax + c0 + j, am[j]);
  }
  // single-chunk launches own the whole sequence of their channels, so the
  // thread that read the old history also writes the new one
  if (write_state && conv_state) {
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int j = 0; j < kConvCPT; ++j) {
        const uint32_t c = (uint32_t)(h[k][j] & 0xFF);
        if (j < 4) lo |= c << (8 * j);
        else hi |= c << (8 * (j - 4));
      }
      *reinterpret_cast<uint2 *>(conv_state + ((long long)b * 3 + k) * cc + c0) = make_uint2(lo, hi);
    }
  }
}

// Multi-chunk launches: replace the conv state by the last 3 inputs after the
// conv kernel has finished reading it (stream order).  T >= 3 here.
__global__ void k_conv_state_update(const int8_t *__restrict__ u, int B, int T, int cc,
                                    int8_t *__restrict__ conv_state) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long n = (long long)B * 3 * cc;
  if (i >= n) return;
  const int c = (int)(i % cc);
  const int k = (int)((i / cc) % 3);
  const int b = (int)(i / (3LL * cc));
  conv_state[i] = u[((long long)b * T + (T - 3 + k)) * cc + c];
}

}  // namespace fm
