// k_scan.cuh -- selective scan in power-of-two fixed point.
//
// FastMamba (arXiv 2505.18975): power-of-two fixed point for the SSM block
// (pith.science review, "What carries the argument"; Figure 7 caption, SSM
// module with the nonlinear approximation unit); e^Delta through the
// shift-based exponential (verdict record, supporting citation [15]);
// SoftPlus(x) ~ e^x for x <= 0 (Referee minor comment 5, Eq. (5)) and
// SoftPlus(x) = x + SoftPlus(-x) (citation [16]).  Mamba2 recurrence (the
// paper's reference [2]) per (batch b, head h, p, n), t in order:
//   dt_q = SoftPlus_pwl(to_q16(dt_raw + dt_bias)),  dA_q = 2^(-rshr(dt_q A_q, 12))
//   u    = satb(rshr(dt_q x[p], s_h), 24)                  s_h = e_h - e_B - e_x + 16
//   h    = clamp(rshr(dA_q h, 16) + u B[n], +-(2^30 - 1))
//   y[p] = satb(rshr(sum_n C[n] h, s_y) + rshr(D_q x[p], s_D), 32)
//
// Mapping: one CTA per (b, h, 8 consecutive p); 16 threads per p, each owning
// 8 consecutive n of the state in registers (the state never leaves the SM
// during a prefill).  Per chunk of 32 tokens the CTA stages B and C (expanded
// to int32), dt_q, dA_q and the per-(t, p) factor u in shared memory; the
// sequential loop then costs per state cell one 32x32->64 multiply-add, one
// funnel shift, one multiply-add, a clamp and one 64-bit multiply-accumulate
// for C.h, and the 16-lane C.h reduction is a shuffle tree.
#pragma once
#include "fm_common.cuh"

namespace fm {

constexpr int kScanNPT = 8;                 // n per thread
constexpr int kScanTPP = 16;                // threads per p (kScanNPT * kScanTPP = d_state = 128)
constexpr int kScanPC = 8;                  // p per CTA
constexpr int kScanThreads = kScanTPP * kScanPC;  // 128
constexpr int kScanTCH = 32;                // tokens per staged chunk
constexpr int kDState = 128;
constexpr long long kHLim = (1LL << 30) - 1;

struct ScanArgs {
  const int8_t *xbc;      // [B, T, cc]: x | B | C
  const float *dt_raw;    // [B, T, nh]
  int T, nh, hd, cc, di;
  const float *dt_bias;
  const int32_t *A_q, *D_q;
  const int32_t *e_x, *e_B, *e_C, *e_h, *e_y, *e_D;  // device pointers into the exponent table
  int32_t *state;         // [B, nh, hd, ds] or null
  int32_t *y;             // [B, T, di]
  unsigned long long *stat;  // [nh]: MODE 1 max|y_f|, MODE 2 max|h64|
  // state spec: the clamp +-hlim and the increment's guard bits g (the
  // increment is rshr(ug B, g) with ug = satb(rshr(dt_q x, s_h - g), 24));
  // the method as built is hlim = 2^30 - 1, g = 0
  int hlim, guard;
  // per-token conv-output exponents [B*T, nh + 2] (x per head, B, C) or null
  // (the static e_x, e_B, e_C); the state and output exponents stay static
  const int32_t *e_tok;
};

// rshr(v, g) for g in [0, 7] (g = 0: v)
__device__ __forceinline__ int rshr_guard(int v, int g) {
  return g ? (v + (1 << (g - 1))) >> g : v;
}

// MODE 0: the scan.  MODE 1: the scan + max |y| at the finer term exponent
// (calibration of e_y).  MODE 2: calibration of e_h -- 64-bit state at the
// finest exponent (s_h = 1, u unclamped, state saturating at +-2^46), no y.
template <int MODE>
__global__ void __launch_bounds__(kScanThreads) k_ssm_scan_pot(ScanArgs a) {
  using StateT = typename std::conditional<MODE == 2, long long, int>::type;
  __shared__ __align__(16) int sB[kScanTCH][kDState];
  __shared__ __align__(16) int sC[kScanTCH][kDState];
  __shared__ int sdA[kScanTCH];
  __shared__ int sdt[kScanTCH];
  __shared__ long long su[kScanTCH][kScanPC];
  __shared__ int sx[kScanTCH][kScanPC];
  __shared__ int sy[kScanTCH][kScanPC];
  // per-token shifts (per-token exponents): u, output, skip, and the two
  // statistic exponents of MODE 1
  __shared__ int tsh[kScanTCH], tsy[kScanTCH], tsD[kScanTCH], tyc[kScanTCH], tyd[kScanTCH];

  const int tid = threadIdx.x;
  const int pp = tid / kScanTPP;
  const int n0 = (tid % kScanTPP) * kScanNPT;
  const int pbase = blockIdx.x * kScanPC;
  const int p = pbase + pp;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int T = a.T, cc = a.cc, di = a.di, hd = a.hd, nh = a.nh;

  const int e_x = a.e_x[h], e_B = *a.e_B, e_C = *a.e_C;
  const int e_h = MODE == 2 ? e_x + e_B - 15 : a.e_h[h];
  const int e_y = MODE == 0 ? a.e_y[h] : 0;
  const int e_D = a.e_D[h];
  const int ef = min(e_C + e_h, e_D + e_x);
  const long long Dq = a.D_q[h];
  const long long Aq = a.A_q[h];
  const float dtb = a.dt_bias[h];

  StateT hs[kScanNPT];
  long long *st_base = nullptr;
  int32_t *st_ptr = a.state ? a.state + ((((long long)b * nh + h) * hd + p) * kDState + n0) : nullptr;
  (void)st_base;
  if (MODE != 2 && st_ptr) {
    const int4 v0 = *reinterpret_cast<const int4 *>(st_ptr);
    const int4 v1 = *reinterpret_cast<const int4 *>(st_ptr + 4);
    hs[0] = v0.x; hs[1] = v0.y; hs[2] = v0.z; hs[3] = v0.w;
    hs[4] = v1.x; hs[5] = v1.y; hs[6] = v1.z; hs[7] = v1.w;
  } else {
#pragma unroll
    for (int j = 0; j < kScanNPT; ++j) hs[j] = 0;
  }
  unsigned long long smax = 0;

  const long long rowbase = (long long)b * T;
  for (int t0 = 0; t0 < T; t0 += kScanTCH) {
    const int nt = min(kScanTCH, T - t0);
    // per-step dt_q and dA_q
    if (tid < nt) {
      const float xf = __fadd_rn(a.dt_raw[(rowbase + t0 + tid) * nh + h], dtb);
      const int dtq = softplus_pwl(to_q16(xf));
      sdt[tid] = dtq;
      sdA[tid] = pow2_pwl(-rshr64((long long)dtq * Aq, 12));
      int ex = e_x, eb = e_B, ec = e_C;
      if (a.e_tok) {
        const int32_t *et = a.e_tok + (rowbase + t0 + tid) * (nh + 2);
        ex = et[h];
        eb = et[nh];
        ec = et[nh + 1];
      }
      // MODE 2 keeps the state at the static finest exponent: u takes the
      // token's own shift 1 + (e_x + e_B) - (ex + eb)
      tsh[tid] = MODE == 2 ? 1 + e_x + e_B - ex - eb : e_h - eb - ex + 16;
      tsy[tid] = e_y - ec - e_h;
      tsD[tid] = e_y - e_D - ex;
      tyc[tid] = ec + e_h - ef;
      tyd[tid] = e_D + ex - ef;
    }
    // B and C rows (contiguous 256 bytes after x), expanded to int32
    for (int i = tid; i < nt * 16; i += kScanThreads) {
      const int tt = i >> 4, k = i & 15;
      const uint4 raw = *reinterpret_cast<const uint4 *>(a.xbc + (rowbase + t0 + tt) * cc + di + k * 16);
      int *dst = k < 8 ? &sB[tt][k * 16] : &sC[tt][(k - 8) * 16];
      const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        int4 o;
        o.x = (int)(int8_t)(w4[q] & 0xFF);
        o.y = (int)(int8_t)((w4[q] >> 8) & 0xFF);
        o.z = (int)(int8_t)((w4[q] >> 16) & 0xFF);
        o.w = (int)(int8_t)((w4[q] >> 24) & 0xFF);
        *reinterpret_cast<int4 *>(dst + 4 * q) = o;
      }
    }
    // this CTA's 8 x values per token
    for (int i = tid; i < nt * kScanPC; i += kScanThreads) {
      const int tt = i / kScanPC, q = i % kScanPC;
      sx[tt][q] = (int)a.xbc[(rowbase + t0 + tt) * cc + (long long)h * hd + pbase + q];
    }
    __syncthreads();
    for (int i = tid; i < nt * kScanPC; i += kScanThreads) {
      const int tt = i / kScanPC, q = i % kScanPC;
      const long long prod = (long long)sdt[tt] * sx[tt][q];
      const int sh = tsh[tt];
      su[tt][q] = MODE == 2 ? (sh >= 0 ? rshr64(prod, sh) : shl_sat61(prod, -sh))
                            : satb64(rshr64(prod, sh - a.guard), 24);
    }
    __syncthreads();

#pragma unroll 1
    for (int tt = 0; tt < nt; ++tt) {
      const long long dA = sdA[tt];
      const long long uu = su[tt][pp];
      int Bv[kScanNPT], Cv[kScanNPT];
      *reinterpret_cast<int4 *>(&Bv[0]) = *reinterpret_cast<const int4 *>(&sB[tt][n0]);
      *reinterpret_cast<int4 *>(&Bv[4]) = *reinterpret_cast<const int4 *>(&sB[tt][n0 + 4]);
      long long acc = 0;
      if (MODE == 2) {
        const long long LIM = 1LL << 46;
#pragma unroll
        for (int j = 0; j < kScanNPT; ++j) {
          long long hn = ((dA * (long long)hs[j] + 32768LL) >> 16) + uu * Bv[j];
          hn = hn > LIM ? LIM : (hn < -LIM ? -LIM : hn);
          hs[j] = (StateT)hn;
          const unsigned long long ah = (unsigned long long)(hn < 0 ? -hn : hn);
          smax = ah > smax ? ah : smax;
        }
        continue;
      }
      *reinterpret_cast<int4 *>(&Cv[0]) = *reinterpret_cast<const int4 *>(&sC[tt][n0]);
      *reinterpret_cast<int4 *>(&Cv[4]) = *reinterpret_cast<const int4 *>(&sC[tt][n0 + 4]);
      const int u32 = (int)uu;
#pragma unroll
      for (int j = 0; j < kScanNPT; ++j) {
        const int dec = (int)((dA * (long long)hs[j] + 32768LL) >> 16);
        int hn = dec + rshr_guard(u32 * Bv[j], a.guard);
        hn = min(max(hn, -a.hlim), a.hlim);
        hs[j] = (StateT)hn;
        acc += (long long)Cv[j] * hn;
      }
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if ((tid % kScanTPP) == 0) {
        const long long dx = Dq * sx[tt][pp];
        sy[tt][pp] = (int)satb64(rshr64(acc, tsy[tt]) + rshr64(dx, tsD[tt]), 32);
        if (MODE == 1) {
          long long yf = pow2_sat61(acc, tyc[tt]) + pow2_sat61(dx, tyd[tt]);
          const unsigned long long ay = (unsigned long long)(yf < 0 ? -yf : yf);
          smax = ay > smax ? ay : smax;
        }
      }
    }
    __syncthreads();
    if (MODE != 2) {
      for (int i = tid; i < nt * kScanPC; i += kScanThreads) {
        const int tt = i / kScanPC, q = i % kScanPC;
        a.y[(rowbase + t0 + tt) * di + (long long)h * hd + pbase + q] = sy[tt][q];
      }
    }
    __syncthreads();
  }
  if (MODE != 2 && st_ptr) {
    *reinterpret_cast<int4 *>(st_ptr) = make_int4((int)hs[0], (int)hs[1], (int)hs[2], (int)hs[3]);
    *reinterpret_cast<int4 *>(st_ptr + 4) = make_int4((int)hs[4], (int)hs[5], (int)hs[6], (int)hs[7]);
  }
  if (MODE != 0) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const unsigned long long other = __shfl_xor_sync(0xffffffffu, smax, o);
      smax = other > smax ? other : smax;
    }
    if ((tid & 31) == 0) atomicMax(a.stat + h, smax);
  }
}

}  // namespace fm
