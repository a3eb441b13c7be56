// k_rows.cuh -- row-wise kernels: Hadamard rotation + int8 quantisation of
// the linear-layer inputs, the fused gate + gated RMSNorm in front of
// out_proj, and the offline fp64 weight rotation.
//
// FastMamba (arXiv 2505.18975), pith.science review: "What carries the
// argument" (Y = (XH)(H^T W^T), H orthonormal after 1/sqrt(n)); Referee
// Report, major comment 1 (scales from the max of the rotated tensors, static
// scales in the hardware of Fig. 6); minor comment 2 (H depends only on the
// dimension).  Gate-then-normalise order and RMSNorm are those of Mamba2 (the
// paper's references [2], [10]).
//
// Layout: one CTA per row, one warp per one or two 256-column Hadamard
// blocks (two when the row has an even number of blocks), each lane holding 8
// consecutive elements of each block (two 16-byte loads per block), so the
// whole row's rotation happens in registers and shuffles; HBM traffic is one
// read of the row and one write of its codes.
#pragma once
#include "fm_common.cuh"

namespace fm {

constexpr int kMaxBlocks = 32;  // K <= 8192

// 8 consecutive floats from a 32-byte-aligned address (two 16-byte loads;
// the entry points require 16-byte-aligned tensors and every caller's offset
// is a multiple of 8 elements)
__device__ __forceinline__ void load8(const float *p, float (&v)[8]) {
  const float4 a = *reinterpret_cast<const float4 *>(p);
  const float4 b = *reinterpret_cast<const float4 *>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Row max over all warps of the CTA (every thread returns the result): each
// warp reduces the warps' maxima itself (lane i reads warp i's), so one
// barrier suffices.  Called once per kernel (s_red is not reused).
__device__ __forceinline__ float cta_max(float v, float *s_red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  v = warp_max(v);
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  return warp_max(lane < nw ? s_red[lane] : 0.0f);
}

// Rotation (optional) + per-row or static quantisation of this lane's BPW
// groups of 8 elements, group b at column 256 * (BPW * warp + b) + 8 * lane;
// thread 0 writes s_x / amax_row.  The BPW blocks' transforms are independent
// (more work in flight per warp, half the warps per row for BPW = 2).
template <int BPW>
__device__ __forceinline__ void rotate_quant_store(float (&v)[BPW][8], int rotate, int mode,
                                                   const float *static_amax, int8_t *qrow,
                                                   float *sx_out, float *amax_out,
                                                   float *s_red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (rotate) {
#pragma unroll
    for (int b = 0; b < BPW; ++b) fwht256_lane8(v[b], lane);
  }
  float a = 0.0f;
  bool finite = true;  // fmaxf drops NaN, so non-finite values are flagged apart
#pragma unroll
  for (int b = 0; b < BPW; ++b)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float m = fabsf(v[b][i]);
      finite = finite && (m <= 3.402823466e38f);
      a = fmaxf(a, m);
    }
  if (!finite) raise_error(kErrNonfinite);
  const float amax = cta_max(a, s_red);
  const float use = (mode == 0) ? amax : *static_amax;
  const float inv = use > 0.0f ? __fdiv_rn(127.0f, use) : 0.0f;
#pragma unroll
  for (int b = 0; b < BPW; ++b) {
    uint32_t lo = 0, hi = 0;
    if (use > 0.0f) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t c = (uint32_t)(quant127(__fmul_rn(v[b][i], inv)) & 0xFF);
        if (i < 4) lo |= c << (8 * i);
        else hi |= c << (8 * (i - 4));
      }
    }
    *reinterpret_cast<uint2 *>(qrow + (warp * BPW + b) * 256 + lane * 8) = make_uint2(lo, hi);
  }
  if (threadIdx.x == 0) {
    *sx_out = use > 0.0f ? __fdiv_rn(use, 127.0f) : 0.0f;
    if (amax_out) *amax_out = amax;
  }
}

// a0 + a1 (and a10's tail): blockDim = 32 * (K / 256 / BPW), grid = M.
template <int BPW>
__global__ void __launch_bounds__(1024) k_hadamard_quant(const float *__restrict__ x, int K,
                                                         const float *__restrict__ prenorm_w,
                                                         int rotate, int mode,
                                                         const float *static_amax,
                                                         int8_t *__restrict__ q, float *s_x,
                                                         float *amax_row) {
  pdl_wait();
  pdl_trigger();
  __shared__ double s_blk[kMaxBlocks];
  __shared__ float s_red[kMaxBlocks];
  __shared__ float s_rstd;
  const long long row = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = (blockDim.x >> 5) * BPW;  // 256-blocks in the row
  float v[BPW][8];
#pragma unroll
  for (int b = 0; b < BPW; ++b) {
    const float *src = x + row * K + (warp * BPW + b) * 256 + lane * 8;
    const float4 p = *reinterpret_cast<const float4 *>(src);
    const float4 r = *reinterpret_cast<const float4 *>(src + 4);
    v[b][0] = p.x; v[b][1] = p.y; v[b][2] = p.z; v[b][3] = p.w;
    v[b][4] = r.x; v[b][5] = r.y; v[b][6] = r.z; v[b][7] = r.w;
  }
  if (prenorm_w) {
    // RMSNorm (eps 1e-5): sum of squares in double in the fixed order
    // (lane-sequential 8, xor tree over the warp, blocks in increasing order)
#pragma unroll
    for (int b = 0; b < BPW; ++b) {
      double P = 0.0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const double e = (double)v[b][i];
        P = __dadd_rn(P, __dmul_rn(e, e));
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) P = __dadd_rn(P, __shfl_xor_sync(0xffffffffu, P, o));
      if (lane == 0) s_blk[warp * BPW + b] = P;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      double tot = 0.0;
      for (int b = 0; b < nb; ++b) tot = __dadd_rn(tot, s_blk[b]);
      const double var = __ddiv_rn(tot, (double)K);
      s_rstd = (float)__drcp_rn(__dsqrt_rn(__dadd_rn(var, 1e-5)));
    }
    __syncthreads();
    const float rstd = s_rstd;
#pragma unroll
    for (int b = 0; b < BPW; ++b) {
      float w[8];
      load8(prenorm_w + (warp * BPW + b) * 256 + lane * 8, w);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[b][i] = __fmul_rn(__fmul_rn(v[b][i], rstd), w[i]);
    }
  }
  rotate_quant_store<BPW>(v, rotate, mode, static_amax, q + row * K, s_x + row,
                          amax_row ? amax_row + row : nullptr, s_red);
}

// a9 + a10: gate y * SiLU(z), g_q int16 at e_g, exact-integer RMSNorm,
// rotation, quantisation.  blockDim = 32 * (di / 256 / BPW), grid = M.
// gstat (nullable, [nh] u64): max |g| per head (calibration).
template <int BPW>
__global__ void __launch_bounds__(1024) k_gate_norm_quant(
    const int32_t *__restrict__ y, const float *__restrict__ z, int di, int hd,
    const int32_t *__restrict__ e_y, const int32_t *__restrict__ e_g_ptr,
    const float *__restrict__ norm_w, int rotate, int mode, const float *static_amax,
    int8_t *__restrict__ q, float *s_x, float *amax_row, unsigned long long *gstat) {
  pdl_wait();
  pdl_trigger();
  __shared__ long long s_ss[kMaxBlocks];
  __shared__ float s_red[kMaxBlocks];
  __shared__ float s_rstd;
  __shared__ int2 tab[8];
  pwl_table_init(tab);
  __syncthreads();
  const long long row = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = blockDim.x >> 5;
  const int e_g = *e_g_ptr;
  int gq[BPW][8];
  long long ss = 0;
#pragma unroll
  for (int b = 0; b < BPW; ++b) {
    const int col = (warp * BPW + b) * 256 + lane * 8;
    const int head = col / hd;  // hd is a multiple of 8: the lane's 8 columns share a head
    const int sg_shift = e_g - e_y[head] + 16;
    int32_t yv[8];
    float zv[8];
    {
      const int4 p = *reinterpret_cast<const int4 *>(y + row * di + col);
      const int4 r = *reinterpret_cast<const int4 *>(y + row * di + col + 4);
      yv[0] = p.x; yv[1] = p.y; yv[2] = p.z; yv[3] = p.w;
      yv[4] = r.x; yv[5] = r.y; yv[6] = r.z; yv[7] = r.w;
      const float4 c = *reinterpret_cast<const float4 *>(z + row * di + col);
      const float4 d = *reinterpret_cast<const float4 *>(z + row * di + col + 4);
      zv[0] = c.x; zv[1] = c.y; zv[2] = c.z; zv[3] = c.w;
      zv[4] = d.x; zv[5] = d.y; zv[6] = d.z; zv[7] = d.w;
    }
    unsigned ss0 = 0, ss1 = 0;  // g_q^2 < 2^30: four per partial fit 32 bits
    unsigned long long gmax = 0;
    int sg[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) sg[i] = silu_pwl_t(to_q16(zv[i]), tab);
    if (!gstat && sg_shift >= 33 && sg_shift <= 63) {
      // the usual case (a calibrated layer's shift is 33..40): with g = hi 2^32 + lo,
      // floor((g + 2^(s-1)) / 2^s) = floor((hi + 2^(s-33)) / 2^(s-32)) because
      // lo / 2^32 < 1 cannot carry the integer numerator past a multiple of
      // 2^(s-32); |hi| < 2^30, so the sum stays in int32
      const int rb = 1 << (sg_shift - 33), sh = sg_shift - 32;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        gq[b][i] = min(max((__mulhi(yv[i], sg[i]) + rb) >> sh, -32767), 32767);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        // g = y sg as a 64-bit value from two 32-bit multiplies
        const long long g = (long long)(((unsigned long long)(unsigned)__mulhi(yv[i], sg[i]) << 32) |
                                        (unsigned)(yv[i] * sg[i]));
        if (gstat) {
          const unsigned long long ag = (unsigned long long)(g < 0 ? -g : g);
          gmax = ag > gmax ? ag : gmax;
        }
        gq[b][i] = (int)satb64(rshr64(g, sg_shift), 16);
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const unsigned sq = (unsigned)(gq[b][i] * gq[b][i]);
      if (i < 4) ss0 += sq;
      else ss1 += sq;
    }
    ss += (long long)ss0 + ss1;
    if (gstat) {
      // the 8 lanes of a 64-column head combine, one atomic per head
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) {
        const unsigned long long other = __shfl_xor_sync(0xffffffffu, gmax, o);
        gmax = other > gmax ? other : gmax;
      }
      if ((lane & 7) == 0) atomicMax(gstat + head, gmax);
    }
  }
  ss = warp_sum_ll(ss);
  if (lane == 0) s_ss[warp] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    long long tot = 0;
    for (int w = 0; w < nw; ++w) tot += s_ss[w];
    const double var = __ddiv_rn(ldexp((double)tot, 2 * e_g), (double)di);
    s_rstd = (float)__drcp_rn(__dsqrt_rn(__dadd_rn(var, 1e-5)));
  }
  __syncthreads();
  const float rstd = s_rstd;
  const float scale = ldexpf(1.0f, e_g);
  float v[BPW][8];
#pragma unroll
  for (int b = 0; b < BPW; ++b) {
    float w[8];
    load8(norm_w + (warp * BPW + b) * 256 + lane * 8, w);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      v[b][i] = __fmul_rn(__fmul_rn(__fmul_rn(small_i2f(gq[b][i]), scale), rstd), w[i]);
  }
  rotate_quant_store<BPW>(v, rotate, mode, static_amax, q + row * di, s_x + row,
                          amax_row ? amax_row + row : nullptr, s_red);
}

// Offline weight preparation: W' = W H (fp64, same butterfly order),
// s_w = fl32(max|W'| / 127), Wq = satb(rint(W' / s_w), 8).  grid = N rows.
__global__ void __launch_bounds__(1024) k_prepare_linear(const float *__restrict__ W, int K,
                                                         int rotate, int8_t *__restrict__ Wq,
                                                         float *__restrict__ s_w) {
  __shared__ double s_red[kMaxBlocks];
  __shared__ double s_amax;
  const long long row = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nb = blockDim.x >> 5;
  const int col = warp * 256 + lane * 8;
  double v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = (double)W[row * K + col + i];
  if (rotate) fwht256_lane8(v, lane);
  double a = 0.0;
#pragma unroll
  for (int i = 0; i < 8; ++i) a = fmax(a, fabs(v[i]));
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) a = fmax(a, __shfl_xor_sync(0xffffffffu, a, o));
  if (lane == 0) s_red[warp] = a;
  __syncthreads();
  if (threadIdx.x == 0) {
    double m = 0.0;
    for (int b = 0; b < nb; ++b) m = fmax(m, s_red[b]);
    s_amax = m;
  }
  __syncthreads();
  const float s = (float)__ddiv_rn(s_amax, 127.0);
  if (threadIdx.x == 0) s_w[row] = s;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int c = 0;
    if (s > 0.0f) {
      double r = rint(__ddiv_rn(v[i], (double)s));
      r = fmin(fmax(r, -127.0), 127.0);
      c = (int)r;
    }
    Wq[row * K + col + i] = (int8_t)c;
  }
}

}  // namespace fm
