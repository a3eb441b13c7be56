// k_conv.cuh -- power-of-two causal depthwise conv1d (kernel 4) + PWL SiLU.
//
// FastMamba (arXiv 2505.18975): fine-grained power-of-two quantisation of the
// convolution layer (pith.science review, "What carries the argument";
// original abstract); SiLU (Swish, the paper's reference [11]) through the
// shared 2^v approximation unit.  Per channel c and token t:
//   acc = bq[c] + sum_{k=0..3} wq[c,k] u[t-3+k, c]           (exact integer)
//   x16 = satb(rshr(acc, -(e_w + e_u + 16)), 32)             (to Q.16)
//   out = satb(rshr(SiLU_pwl(x16), e_o + 16), 8)
//
// Layout: each thread owns 4 consecutive channels of one token (4-byte loads
// of the 4-row window t-3 .. t and one 4-byte store); a warp covers 128
// contiguous bytes of each row and the window rows shared by neighbouring
// tokens come from L1/L2.  Every (token, channel) output is independent, so
// the grid is (channel groups / 64, T, batch) of 64-thread blocks with few
// registers per thread (high occupancy hides the PWL SiLU's latency).  The
// conv state (the 3 inputs before the first token) is read here and replaced
// afterwards by k_conv_state_update, in stream order.
#pragma once
#include "fm_common.cuh"

namespace fm {

constexpr int kConvCPT = 4;       // channels per thread
constexpr int kConvThreads = 64;  // threads per block

__device__ __forceinline__ void unpack4(uint32_t w, int (&v)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = (int)(int8_t)((w >> (8 * i)) & 0xFF);
}

// amax (nullable, [cc] u32): max |SiLU output| per channel (calibration).
__global__ void __launch_bounds__(kConvThreads) k_conv1d_pot(
    const int8_t *__restrict__ u, int T, int cc, const int8_t *__restrict__ wq,
    const int32_t *__restrict__ bq, const int32_t *__restrict__ exps,
    const int8_t *__restrict__ conv_state, int8_t *__restrict__ out, unsigned int *amax) {
  __shared__ int tab[8];
  pwl_table_init(tab);
  __syncthreads();
  const int c0 = (blockIdx.x * kConvThreads + threadIdx.x) * kConvCPT;
  if (c0 >= cc) return;
  const int t = blockIdx.y;
  const int b = blockIdx.z;
  const int8_t *ub = u + (long long)b * T * cc;
  int win[4][kConvCPT];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int tt = t - 3 + r;
    uint32_t raw = 0u;
    if (tt >= 0)
      raw = *reinterpret_cast<const uint32_t *>(ub + (long long)tt * cc + c0);
    else if (conv_state)
      raw = *reinterpret_cast<const uint32_t *>(conv_state + ((long long)b * 3 + (3 + tt)) * cc + c0);
    unpack4(raw, win[r]);
  }
  const uint4 wp = *reinterpret_cast<const uint4 *>(wq + (long long)c0 * 4);  // 4 taps x 4 channels
  const int4 bias = *reinterpret_cast<const int4 *>(bq + c0);
  const int4 eu = *reinterpret_cast<const int4 *>(exps + c0);
  const int4 ew = *reinterpret_cast<const int4 *>(exps + cc + c0);
  const int4 eo = *reinterpret_cast<const int4 *>(exps + 2 * cc + c0);
  const uint32_t wr[4] = {wp.x, wp.y, wp.z, wp.w};
  const int bs[4] = {bias.x, bias.y, bias.z, bias.w};
  const int s_in[4] = {-(ew.x + eu.x + 16), -(ew.y + eu.y + 16), -(ew.z + eu.z + 16),
                       -(ew.w + eu.w + 16)};
  const int s_out[4] = {eo.x + 16, eo.y + 16, eo.z + 16, eo.w + 16};
  uint32_t packed = 0;
#pragma unroll
  for (int j = 0; j < kConvCPT; ++j) {
    int w[4];
    unpack4(wr[j], w);
    const int dot = w[0] * win[0][j] + w[1] * win[1][j] + w[2] * win[2][j] + w[3] * win[3][j];
    int x16;
    const int si = s_in[j];
    if (bs[j] >= -(1 << 29) && bs[j] <= (1 << 29) && si >= -30 && si <= 29) {
      // 32-bit path: |acc| < 2^30 (the taps add at most 4 * 127^2)
      const int acc = bs[j] + dot;
      if (si > 0) {
        x16 = rshr32(acc, si);
      } else {
        const int k = -si, lim = 0x7FFFFFFF >> k;
        x16 = acc > lim ? 2147483647 : (acc < -lim ? -2147483647 : acc * (1 << k));
      }
    } else {
      x16 = (int)satb64(rshr64((long long)bs[j] + dot, si), 32);
    }
    const int sv = silu_pwl_t(x16, tab);
    if (amax) atomicMax(amax + c0 + j, (unsigned int)(sv < 0 ? -sv : sv));
    const int so = s_out[j];
    int code;
    if (so >= 1 && so <= 31) {
      code = min(max(rshr32(sv, so), -127), 127);
    } else {
      code = (int)satb64(rshr64(sv, so), 8);
    }
    packed |= ((uint32_t)(code & 0xFF)) << (8 * j);
  }
  *reinterpret_cast<uint32_t *>(out + ((long long)b * T + t) * cc + c0) = packed;
}

// After the conv: the state becomes the last 3 inputs (oldest first).  One
// thread per (b, c) reads everything it writes, so it works in place for any
// T (for T < 3 the older entries shift down).
__global__ void k_conv_state_update(const int8_t *__restrict__ u, int B, int T, int cc,
                                    int8_t *__restrict__ conv_state) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)B * cc) return;
  const int c = (int)(i % cc);
  const int b = (int)(i / cc);
  int8_t *st = conv_state + (long long)b * 3 * cc + c;
  int8_t old[3] = {st[0], st[cc], st[2 * cc]};
  int8_t nw[3];
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const int tt = T - 3 + k;
    nw[k] = tt >= 0 ? u[((long long)b * T + tt) * cc + c] : old[3 + tt];
  }
  st[0] = nw[0];
  st[cc] = nw[1];
  st[2 * cc] = nw[2];
}

}  // namespace fm
