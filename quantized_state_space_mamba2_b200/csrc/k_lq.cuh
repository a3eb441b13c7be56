// k_lq.cuh -- the FastMamba-LQ variant: the conv1d, the selective scan and
// the gate in exact fp32 arithmetic, between the same Hadamard-rotated W8A8
// linears as the full method.
//
// FastMamba (arXiv 2505.18975) reports this variant beside the fully
// quantised model (pith.science review, Desk Editor's Note: "LQ" quantises
// only the linear layers).  The arithmetic is Mamba2's own (the paper's
// reference [2]; block flow of its Figure 2): per channel c and token t
//   xo[t, c]  = SiLU(b[c] + sum_{k=0..3} w[c, k] u[t-3+k, c])   (causal conv)
//   dt[t, h]  = SoftPlus(dt_raw[t, h] + dt_bias[h]),  dA = exp(dt A[h]),
//               A[h] = -exp(A_log[h])
//   h[p, n]  <- dA h[p, n] + (dt x[t, p]) B[t, n]
//   y[t, p]   = sum_n C[t, n] h[p, n] + D[h] x[t, p]
//   g[t, p]   = y[t, p] SiLU(z[t, p])                          (the gate)
// with exact exp / log1p / division (CUDA's expf, log1pf), no PWL unit and
// no power-of-two codes.  The gated RMSNorm and the out_proj input's
// rotation + int8 quantisation that follow are k_hadamard_quant with the
// norm weight as its pre-norm weight.
#pragma once
#include "fm_common.cuh"
#include "k_gemm.cuh"

namespace fm {

__device__ __forceinline__ float silu_f32(float v) {
  return __fdiv_rn(v, __fadd_rn(1.0f, expf(-v)));
}
// SoftPlus(x) = log(1 + e^x); above 20 it equals x to fp32 precision
__device__ __forceinline__ float softplus_f32(float x) {
  return x > 20.0f ? x : log1pf(expf(x));
}

// ------------------------------------------------------------------ conv
// One thread per (channel, run of kLqConvTT tokens); a block is 256 channels.
// u rows have stride ldu floats (the in_proj output [M, n_in] read in place);
// out is [B, T, cc].  conv_state [B, 3, cc] (nullable) holds the 3 inputs
// before token 0, oldest first; it is read here and replaced afterwards by
// k_lq_conv_state_update in stream order.
constexpr int kLqConvTT = 16;

__global__ void __launch_bounds__(256) k_lq_conv(const float *__restrict__ u, long long ldu,
                                                 int T, int cc, const float *__restrict__ w,
                                                 const float *__restrict__ bias,
                                                 const float *__restrict__ conv_state,
                                                 float *__restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const int c = blockIdx.y * 256 + threadIdx.x;
  const int t0 = blockIdx.x * kLqConvTT;
  const int b = blockIdx.z;
  if (c >= cc || t0 >= T) return;
  const float4 wc = *reinterpret_cast<const float4 *>(w + (long long)c * 4);
  const float bc = bias[c];
  const float *ub = u + (long long)b * T * ldu + c;
  // the window: inputs t-3, t-2, t-1 before token t0
  float win[3];
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const int t = t0 - 3 + k;
    win[k] = t >= 0 ? ub[(long long)t * ldu]
                    : (conv_state ? conv_state[((long long)b * 3 + (3 + t)) * cc + c] : 0.0f);
  }
  float *ob = out + (long long)b * T * cc + c;
  const int nt = min(kLqConvTT, T - t0);
#pragma unroll 4
  for (int i = 0; i < nt; ++i) {
    const float cur = ub[(long long)(t0 + i) * ldu];
    float acc = bc;
    acc = __fmaf_rn(wc.x, win[0], acc);
    acc = __fmaf_rn(wc.y, win[1], acc);
    acc = __fmaf_rn(wc.z, win[2], acc);
    acc = __fmaf_rn(wc.w, cur, acc);
    ob[(long long)(t0 + i) * cc] = silu_f32(acc);
    win[0] = win[1];
    win[1] = win[2];
    win[2] = cur;
  }
}

// New conv state: the last 3 of (old state, the T inputs).  One thread per
// (sequence, channel) reads everything it needs before writing.
__global__ void __launch_bounds__(256) k_lq_conv_state_update(const float *__restrict__ u,
                                                              long long ldu, int B, int T, int cc,
                                                              float *conv_state) {
  pdl_wait();
  pdl_trigger();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)B * cc) return;
  const int b = (int)(i / cc), c = (int)(i % cc);
  float *st = conv_state + (long long)b * 3 * cc + c;
  float nv[3];
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const int t = T - 3 + k;  // index into (old state ++ inputs), old state at -3..-1
    nv[k] = t >= 0 ? u[((long long)b * T + t) * ldu + c] : st[(long long)(3 + t) * cc];
  }
#pragma unroll
  for (int k = 0; k < 3; ++k) st[(long long)k * cc] = nv[k];
}

// ------------------------------------------------------------------ scan
// Grid (hd / (4 CPW), nh, B), 4 warps; warp w owns channels p0 .. p0 + CPW - 1
// of head h, lane l the states n = 4l .. 4l + 3 of each (CPW x 4 fp32 state
// cells in registers for the whole sequence).  The sequence runs in 32-token
// chunks staged in shared memory, two buffers: while the warps run chunk c,
// chunk c + 1's B and C rows and the CTA's x values are on their way (cp.async,
// 16 bytes a piece, whole rows per warp), and 32 threads compute its dt and
// dA.  Each step adds its C h partial sums to a 32-entry buffer (32 / CPW
// steps x CPW channels); a full buffer is reduced across the warp by a
// reduce-scatter (5 xor-shuffle stages), after which lane j holds the total
// of entry j and writes that output.
//   xo     [B, T, cc] conv output (x | B | C)
//   dt_raw rows of stride ld_dt (column h), z rows of stride ld_z (nullable:
//          no gate, y is written)
//   state  [B, nh, hd, ds] fp32 in/out (nullable: zero initial state)
//   out    [B, T, di]: g = y SiLU(z), or y
constexpr int kLqChunk = 32;

template <int CPW>
struct LqScanSmem {
  float Bm[2][kLqChunk][128];
  float Cm[2][kLqChunk][128];
  float X[2][kLqChunk][4 * CPW];
  float dt[2][kLqChunk];
  float dA[2][kLqChunk];
};

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int CPW>
__global__ void __launch_bounds__(128) k_lq_scan(
    const float *__restrict__ xo, const float *__restrict__ dt_raw, long long ld_dt,
    const float *__restrict__ z, long long ld_z, int T, int nh, int cc, int di,
    const float *__restrict__ dt_bias, const float *__restrict__ a_log,
    const float *__restrict__ Dp, float *state, float *__restrict__ out) {
  pdl_wait();
  pdl_trigger();
  static_assert(CPW == 1 || CPW == 2 || CPW == 4, "CPW");
  constexpr int SB = 32 / CPW;  // steps per reduction
  constexpr int hd = 64, ds = 128, CH = 4 * CPW;  // channels per CTA
  extern __shared__ __align__(16) uint8_t smem_raw[];
  LqScanSmem<CPW> &sm = *reinterpret_cast<LqScanSmem<CPW> *>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int pc0 = blockIdx.x * CH;            // the CTA's first channel
  const int p0 = pc0 + warp * CPW;            // this warp's first channel
  const int n0 = lane * 4;
  const float A = -expf(a_log[h]);
  const float Dh = Dp[h];
  const float bias = dt_bias[h];
  const long long bh = (long long)b * nh + h;
  const float *xrow = xo + (long long)b * T * cc;

  // stage chunk c into buffer c & 1 (B, C rows and the CTA's x: cp.async;
  // dt, dA of its 32 tokens: warp 0)
  auto stage = [&](int c) {
    const int t0 = c * kLqChunk, nt = min(kLqChunk, T - t0), buf = c & 1;
    for (int i = tid; i < kLqChunk * 64; i += 128) {   // 64 pieces per token: 32 B, 32 C
      const int s = i >> 6, k = i & 63;
      if (s < nt) {
        const float *src = xrow + (long long)(t0 + s) * cc + di + k * 4;
        float *dst = k < 32 ? &sm.Bm[buf][s][k * 4] : &sm.Cm[buf][s][(k - 32) * 4];
        cp_async16(dst, src);
      }
    }
    for (int i = tid; i < kLqChunk * CPW; i += 128) {  // CPW pieces of 4 channels per token
      const int s = i / CPW, k = i % CPW;
      if (s < nt) cp_async16(&sm.X[buf][s][k * 4], xrow + (long long)(t0 + s) * cc + h * hd + pc0 + k * 4);
    }
    cp_async_commit();
    if (warp == 0) {
      float dtl = 0.0f, dAl = 0.0f;
      if (lane < nt) {
        const float v = __fadd_rn(dt_raw[((long long)b * T + t0 + lane) * ld_dt + h], bias);
        dtl = softplus_f32(v);
        dAl = expf(__fmul_rn(dtl, A));
      }
      sm.dt[buf][lane] = dtl;
      sm.dA[buf][lane] = dAl;
    }
  };

  float hs[CPW][4];
  float *st = state ? state + (bh * hd + p0) * ds + n0 : nullptr;
#pragma unroll
  for (int c = 0; c < CPW; ++c) {
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (st) v = *reinterpret_cast<const float4 *>(st + (long long)c * ds);
    hs[c][0] = v.x;
    hs[c][1] = v.y;
    hs[c][2] = v.z;
    hs[c][3] = v.w;
  }
  const int nch = (T + kLqChunk - 1) / kLqChunk;
  stage(0);
  float part[32];
#pragma unroll 1
  for (int ch = 0; ch < nch; ++ch) {
    if (ch + 1 < nch) {
      stage(ch + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();  // chunk ch staged (copies and dt / dA) for every warp
    const int buf = ch & 1, t0 = ch * kLqChunk, nt = min(kLqChunk, T - t0);
#pragma unroll 1
    for (int s0 = 0; s0 < kLqChunk; s0 += SB) {
#pragma unroll
      for (int k = 0; k < SB; ++k) {
        const int s = s0 + k;
        if (s < nt) {
          const float dts = sm.dt[buf][s], dAs = sm.dA[buf][s];
          const float4 Bv = *reinterpret_cast<const float4 *>(&sm.Bm[buf][s][n0]);
          const float4 Cv = *reinterpret_cast<const float4 *>(&sm.Cm[buf][s][n0]);
#pragma unroll
          for (int c = 0; c < CPW; ++c) {
            const float dtx = __fmul_rn(dts, sm.X[buf][s][warp * CPW + c]);
            hs[c][0] = __fmaf_rn(dAs, hs[c][0], __fmul_rn(dtx, Bv.x));
            hs[c][1] = __fmaf_rn(dAs, hs[c][1], __fmul_rn(dtx, Bv.y));
            hs[c][2] = __fmaf_rn(dAs, hs[c][2], __fmul_rn(dtx, Bv.z));
            hs[c][3] = __fmaf_rn(dAs, hs[c][3], __fmul_rn(dtx, Bv.w));
            float a = __fmul_rn(Cv.x, hs[c][0]);
            a = __fmaf_rn(Cv.y, hs[c][1], a);
            a = __fmaf_rn(Cv.z, hs[c][2], a);
            a = __fmaf_rn(Cv.w, hs[c][3], a);
            part[k * CPW + c] = a;
          }
        } else {
#pragma unroll
          for (int c = 0; c < CPW; ++c) part[k * CPW + c] = 0.0f;
        }
      }
      // reduce-scatter: afterwards part[0] on lane j is the warp total of entry j
#pragma unroll
      for (int m = 16; m >= 1; m >>= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < m; ++i) {
          const float send = upper ? part[i] : part[i + m];
          const float keep = upper ? part[i + m] : part[i];
          part[i] = __fadd_rn(keep, __shfl_xor_sync(0xffffffffu, send, m));
        }
      }
      const int s = s0 + lane / CPW, c = lane % CPW;
      if (s < nt) {
        const long long r = (long long)b * T + t0 + s;
        float y = __fmaf_rn(Dh, sm.X[buf][s][warp * CPW + c], part[0]);
        if (z) y = __fmul_rn(y, silu_f32(z[r * ld_z + h * hd + p0 + c]));
        out[r * di + h * hd + p0 + c] = y;
      }
    }
    __syncthreads();  // every warp is done with buffer buf before it is refilled
  }
  if (st) {
#pragma unroll
    for (int c = 0; c < CPW; ++c)
      *reinterpret_cast<float4 *>(st + (long long)c * ds) =
          make_float4(hs[c][0], hs[c][1], hs[c][2], hs[c][3]);
  }
}

}  // namespace fm
