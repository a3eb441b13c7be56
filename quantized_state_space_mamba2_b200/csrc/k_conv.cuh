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
// Layout: each thread owns 4 consecutive channels and TT consecutive tokens
// (4 for prefill, 1 for decode steps).  It loads the TT + 3 input rows of its channels once (4-byte
// words: byte j = channel j), transposes the first window so that each
// channel's 4 taps sit in one word (tap k = byte k), and slides it one token
// at a time with one byte permute per channel; each 4-tap dot product is one
// dp4a against the channel's packed weights.  A block is 64 channel quads
// (256 channels) x TG token groups; grid (token tiles, channel groups, batch).  Every (token, channel) output is
// independent.  The conv state (the 3 inputs before the first token) is read
// here and replaced afterwards by k_conv_state_update, in stream order -- or,
// for a single token (a decode step), by the same thread that read it
// (state_out).
#pragma once
#include "fm_common.cuh"

namespace fm {

constexpr int kConvCPT = 4;        // channels per thread
constexpr int kConvTT = 4;         // tokens per thread (prefill)
constexpr int kConvQuads = 64;     // channel quads per block (256 channels)
constexpr int kConvTG = 2;         // token groups per block (prefill)
constexpr int kConvTokens = kConvTT * kConvTG;  // tokens per block (prefill)

// tap k of channel j -> byte k of column j, from the rows (byte j = channel j)
// of tokens t-3 .. t
__device__ __forceinline__ void conv_transpose4(uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3,
                                                uint32_t (&col)[4]) {
  const uint32_t a = __byte_perm(r0, r1, 0x5140), b = __byte_perm(r2, r3, 0x5140);
  const uint32_t c = __byte_perm(r0, r1, 0x7362), d = __byte_perm(r2, r3, 0x7362);
  col[0] = __byte_perm(a, b, 0x5410);
  col[1] = __byte_perm(a, b, 0x7632);
  col[2] = __byte_perm(c, d, 0x5410);
  col[3] = __byte_perm(c, d, 0x7632);
}

// amax (nullable, [cc] u32): max |SiLU output| per channel (calibration).
// TOK (per-token output exponents, the x of each head, B and C each a group;
// e_tok non-null): the codes of token t and group g are
// satb(rshr(s, e + 16), 8) with e = max(E(max_g |s|, 127) - 16, e_o - 16), E
// the power-of-two exponent of the calibration; e_tok[t, g] (int32
// [B*T, nh + 2]) receives e.  A head's 64 x channels are 16 consecutive
// threads and B, C one warp each (the x | B | C boundaries are multiples of
// 256 channels), so the group maximum is a shuffle reduction.
// CALIB: amax is non-null (calibration); otherwise it is not read.
// The common case takes a short path: when none of the thread's 4 channels
// can saturate x16 (|b| + 4 128^2, shifted to Q.16, stays inside int32) nor
// overflow the output's rounding add, x16 = (dp4a(taps, w, b + rounding bias)
// >> right) << left and the output code is a plain add-and-shift, both exact;
// any other thread runs the general 64-bit form.
template <int TT, int TG, bool TOK = false, bool CALIB = false>
__global__ void __launch_bounds__(kConvQuads *TG) k_conv1d_pot(
    const int8_t *__restrict__ u, int T, int cc, const int8_t *__restrict__ wq,
    const int32_t *__restrict__ bq, const int32_t *__restrict__ exps,
    const int8_t *conv_state, int8_t *__restrict__ out, unsigned int *amax,
    int8_t *state_out, int32_t *e_tok = nullptr, int di = 0, int hd = 0, int ds = 0) {
  pdl_wait();
  pdl_trigger();
  __shared__ int2 tab[8];
  pwl_table_init(tab);
  __syncthreads();
  const int quad = threadIdx.x % kConvQuads, tg = threadIdx.x / kConvQuads;
  const int c0 = (blockIdx.y * kConvQuads + quad) * kConvCPT;
  if (c0 >= cc) return;
  const int t0 = (blockIdx.x * TG + tg) * TT;
  if (t0 >= T) return;
  const int b = blockIdx.z;
  const int8_t *ub = u + (long long)b * T * cc;
  // input rows t0-3 .. t0+TT-1 (rows past the end are never used)
  uint32_t row[TT + 3];
#pragma unroll
  for (int r = 0; r < TT + 3; ++r) {
    const int tt = t0 - 3 + r;
    uint32_t raw = 0u;
    if (tt >= 0) {
      if (tt < T) raw = *reinterpret_cast<const uint32_t *>(ub + (long long)tt * cc + c0);
    } else if (conv_state) {
      raw = *reinterpret_cast<const uint32_t *>(conv_state + ((long long)b * 3 + (3 + tt)) * cc + c0);
    }
    row[r] = raw;
  }
  if (state_out) {  // T == 1 (one token per thread): the new state is rows t-2 .. t
#pragma unroll
    for (int r = 0; r < 3; ++r)
      *reinterpret_cast<uint32_t *>(state_out + ((long long)b * 3 + r) * cc + c0) = row[r + 1];
  }
  const uint4 wp = *reinterpret_cast<const uint4 *>(wq + (long long)c0 * 4);  // 4 taps x 4 channels
  const int4 bias = *reinterpret_cast<const int4 *>(bq + c0);
  const int4 eu = *reinterpret_cast<const int4 *>(exps + c0);
  const int4 ew = *reinterpret_cast<const int4 *>(exps + cc + c0);
  const int4 eo = *reinterpret_cast<const int4 *>(exps + 2 * cc + c0);
  const int wr[4] = {(int)wp.x, (int)wp.y, (int)wp.z, (int)wp.w};
  const int bs[4] = {bias.x, bias.y, bias.z, bias.w};
  const int s_in[4] = {-(ew.x + eu.x + 16), -(ew.y + eu.y + 16), -(ew.z + eu.z + 16),
                       -(ew.w + eu.w + 16)};
  const int s_out[4] = {eo.x + 16, eo.y + 16, eo.z + 16, eo.w + 16};
  // short-path constants: dp4a accumulator (bias + the rounding bias of a
  // right shift), right and left shifts to Q.16, the output's rounding bias
  int cb[4], rsh[4], lsh[4], rob[4];
  bool easy = !TOK;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int si = s_in[j], so = s_out[j];
    const bool ok = bs[j] >= -(1 << 29) && bs[j] <= (1 << 29) && si >= -30 && si <= 29 &&
                    so >= 1 && so <= 31;
    rsh[j] = si > 0 ? si : 0;
    lsh[j] = si > 0 ? 0 : -si;
    cb[j] = ok ? bs[j] + (si > 0 ? 1 << (si - 1) : 0) : 0;
    rob[j] = ok ? 1 << (so - 1) : 0;
    // |x16| bound: |acc| <= |b| + 4 128^2 (any int8 codes and weights, + the
    // rounding bias), then shifted
    const long long ab = (long long)(bs[j] < 0 ? -(long long)bs[j] : bs[j]) + 65536 +
                         (si > 0 && si < 62 ? (1LL << (si - 1)) : 0);
    const long long xb = ok ? (si > 0 ? (ab >> si) + 1 : ab << lsh[j]) : (1LL << 40);
    // |SiLU(x16)| <= |x16|, so the output's rounding add cannot overflow either
    easy = easy && ok && xb + (1LL << (so - 1)) <= 2147483647LL;
  }
  uint32_t col[4];
  conv_transpose4(row[0], row[1], row[2], row[3], col);
  const int nt = min(TT, T - t0);
#pragma unroll
  for (int k = 0; k < TT; ++k) {
    if (k > 0) {  // slide: drop the oldest tap, append byte j of the new row
      const uint32_t nr = row[k + 3];
      col[0] = __byte_perm(col[0], nr, 0x4321);
      col[1] = __byte_perm(col[1], nr, 0x5321);
      col[2] = __byte_perm(col[2], nr, 0x6321);
      col[3] = __byte_perm(col[3], nr, 0x7321);
    }
    if (k >= nt) break;
    uint32_t packed = 0;
    if constexpr (TOK) {  // per-token exponents (the warp is all x, all B or all C: uniform)
      int sv[kConvCPT];
      int m = 0;
#pragma unroll
      for (int j = 0; j < kConvCPT; ++j) {
        const long long acc = (long long)bs[j] + __dp4a((int)col[j], wr[j], 0);
        sv[j] = silu_pwl_t((int)satb64(rshr64(acc, s_in[j]), 32), tab);
        m = max(m, sv[j] < 0 ? -sv[j] : sv[j]);
      }
      const bool xgrp = c0 < di;
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (!xgrp) m = max(m, __shfl_xor_sync(0xffffffffu, m, 16));
      const int e = max(pot_exponent((double)m, 127.0) - 16, s_out[0] - 32);
#pragma unroll
      for (int j = 0; j < kConvCPT; ++j)
        packed |= ((uint32_t)((int)satb64(rshr64(sv[j], e + 16), 8) & 0xFF)) << (8 * j);
      const int lane = threadIdx.x & 31;
      if ((lane & (xgrp ? 15 : 31)) == 0) {
        const int nh = di / hd;
        const int g = xgrp ? c0 / hd : (c0 < di + ds ? nh : nh + 1);
        e_tok[((long long)b * T + t0 + k) * (nh + 2) + g] = e;
      }
      *reinterpret_cast<uint32_t *>(out + ((long long)b * T + t0 + k) * cc + c0) = packed;
      continue;
    }
    if (easy) {
#pragma unroll
      for (int j = 0; j < kConvCPT; ++j) {
        const int x16 = (__dp4a((int)col[j], wr[j], cb[j]) >> rsh[j]) << lsh[j];
        const int sv = silu_pwl_t(x16, tab);
        if constexpr (CALIB) atomicMax(amax + c0 + j, (unsigned int)(sv < 0 ? -sv : sv));
        const int code = min(max((sv + rob[j]) >> s_out[j], -127), 127);
        packed |= ((uint32_t)(code & 0xFF)) << (8 * j);
      }
    } else {
#pragma unroll
      for (int j = 0; j < kConvCPT; ++j) {
        const long long acc = (long long)bs[j] + __dp4a((int)col[j], wr[j], 0);
        const int x16 = (int)satb64(rshr64(acc, s_in[j]), 32);
        const int sv = silu_pwl_t(x16, tab);
        if constexpr (CALIB) atomicMax(amax + c0 + j, (unsigned int)(sv < 0 ? -sv : sv));
        const int code = (int)satb64(rshr64(sv, s_out[j]), 8);
        packed |= ((uint32_t)(code & 0xFF)) << (8 * j);
      }
    }
    *reinterpret_cast<uint32_t *>(out + ((long long)b * T + t0 + k) * cc + c0) = packed;
  }
}

// After the conv: the state becomes the last 3 inputs (oldest first).  One
// thread per (b, c) reads everything it writes, so it works in place for any
// T (for T < 3 the older entries shift down).
__global__ void k_conv_state_update(const int8_t *__restrict__ u, int B, int T, int cc,
                                    int8_t *__restrict__ conv_state) {
  pdl_wait();
  pdl_trigger();
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
