// k_ssd.cuh -- the chunked (state-space-dual) scan mode on the tensor cores.
//
// Mamba2's chunked algorithm (reference [2] of the FastMamba paper,
// "Transformers are SSMs") on the quantised method's inputs: the conv's int8
// x / B / C codes, the PWL SoftPlus dt_q and the step's log2 decay
// w = -rshr(dt_q A_q, 12) (FastMamba, arXiv 2505.18975: power-of-two fixed
// point for the SSM block and a shift-based exponential, pith.science review
// "What carries the argument").  Inside a chunk of kSsdQ tokens, with W the
// running sum of w:
//   intra   G = Cq Bq^T (kind::i8, exact), M[t, s] = bf16(G a(s, t) dt[s]) for s <= t
//   inter   Ca[t, n] = bf16(2^W[t] Cq[t, n])
//   Y[t, p] = sum_s M[t, s] X[s, p] + sum_n Ca[t, n] bf16(H[p, n])   (kind::f16, fp32)
//   state   dH[p, n] = sum_s X[s, p] bf16(2^(W[end] - W[s]) dt[s] Bq[s, n])
//           H_next = 2^W[end] H + dH
// Three kernels: k_ssd_state (per chunk: dH and the chunk's decay),
// k_ssd_pass (one thread per state cell, sequential over chunks: the state
// entering each chunk), k_ssd_out (per chunk: Y and the int32 y codes).  Operand tiles are
// written by the threads into 128-byte-swizzled K-major shared memory (rows
// of 128 bytes, 8-row groups 1024 bytes apart, 16-byte pieces XOR-ed with
// the row's index within its group), the layout sw128_desc() describes; one
// thread issues the MMAs, every wait is bounded.
#pragma once
#include <cuda_bf16.h>

#include "fm_common.cuh"
#include "k_gemm.cuh"

namespace fm {

constexpr int kSsdQ = 128;        // tokens per chunk
constexpr int kSsdThreads = 128;  // one thread per token (and TMEM lane)
constexpr int kSsdHd = 64, kSsdDs = 128;

struct SsdArgs {
  const int8_t *xbc;    // [B, T, cc] conv output: x | B | C
  const float *dt_raw;  // [B, T, nh]
  int T, nh, cc, di, nch;
  const float *dt_bias;
  const int32_t *A_q, *D_q;
  const int32_t *e_x, *e_B, *e_C, *e_h, *e_y, *e_D;
  int32_t *state;       // [B, nh, 64, 128] int32 at e_h (nullable)
  int32_t *y;           // [B, T, di]
  float *dH;            // [B, nh, nch, 64, 128] chunk state contributions (code units)
  float *achunk;        // [B, nh, nch] 2^(W at the chunk's last token)
  uint16_t *Hin;        // [B, nh, nch, 64, 128] bf16 state entering each chunk
};

// byte offset of (row r, byte k) in a K-major tile of `rows` rows whose rows
// are cut into 128-byte swizzle atoms (atom k / 128 holds bytes [128j, 128j+128))
__device__ __forceinline__ uint32_t sw128_off(int r, int k, int rows) {
  const int atom = k >> 7, kb = k & 127;
  return (uint32_t)(atom * rows * 128 + (r >> 3) * 1024 + (r & 7) * 128 +
                    ((((kb >> 4) ^ (r & 7)) << 4) | (kb & 15)));
}
__device__ __forceinline__ uint32_t bf16_bits(float v) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v));
}
// kind::f16 instruction descriptor: D fp32 (bits 4-5 = 1), A and B bf16
// (bits 7-9 = 1, 10-12 = 1), both K-major, N >> 3 at 17-22, M >> 4 at 24-28
__host__ __device__ constexpr uint32_t bf16_idesc(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t *slot, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(slot)),
               "r"(cols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t base, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(cols)
               : "memory");
}
// fl32(2^(fl32(e 2^-16))) for an integer exponent e <= 0 (Q.16)
__device__ __forceinline__ float pow2_q16(long long e) {
  return exp2f(__fmul_rn(__ll2float_rn(e), 1.0f / 65536.0f));
}
// The same for e <= 0 with e clamped at -(2^22 - 1) (a decay below 2^-63.99,
// far under the mode's error budget), so that the exponent converts exactly
// without the conversion unit.
__device__ __forceinline__ float pow2_q16_decay(long long e) {
  const int ec = (int)(e < -4194303LL ? -4194303LL : e);
  return exp2f(__fmul_rn(small_i2f(ec), 1.0f / 65536.0f));
}
// k_ssd_out's x-code tile [128 s][64 B] with its 16-byte pieces XOR-ed by
// (s >> 1) & 3: a warp reading one piece of 32 consecutive rows, or 32 bytes
// of one row, touches distinct banks.
__device__ __forceinline__ int xt_off(int s, int b) {
  return s * 64 + ((((b >> 4) ^ (s >> 1)) & 3) << 4) + (b & 15);
}

// dt_q and w of token t of the chunk (0 past the end); W = inclusive prefix
// sum of w over the chunk's 128 tokens (one per thread), into sW[t].  Threads
// t >= kSsdQ of a wider block only pass its barrier.
// The per-thread inputs of ssd_chunk_decay, loaded at the kernel's start so
// that their latency overlaps the tile loads: this thread's token's dt_raw
// (0 past the end), dt_bias[h] and A_q[h].
struct SsdDecayIn {
  float dt_raw, bias;
  int A_q;
};
__device__ __forceinline__ SsdDecayIn ssd_decay_in(const SsdArgs &a, int b, int h, int t0,
                                                  int nt) {
  const int t = threadIdx.x;
  SsdDecayIn in;
  in.dt_raw = t < nt ? a.dt_raw[((long long)b * a.T + t0 + t) * a.nh + h] : 0.0f;
  in.bias = a.dt_bias[h];
  in.A_q = a.A_q[h];
  return in;
}
__device__ __forceinline__ int ssd_chunk_decay(const SsdDecayIn &in, int nt, long long *sW,
                                               long long *wtot) {
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  int dtq = 0;
  long long w = 0;
  if (t < nt) {
    const float xf = __fadd_rn(in.dt_raw, in.bias);
    dtq = softplus_pwl(to_q16(xf));
    w = -rshr64((long long)dtq * in.A_q, 12);
  }
  long long v = w;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31 && t < kSsdQ) wtot[warp] = v;
  __syncthreads();
  if (t < kSsdQ) {
    for (int k = 0; k < warp; ++k) v += wtot[k];
    sW[t] = v;
  }
  return dtq;
}

// ------------------------------------------------------------ chunk state
struct SsdStateSmem {
  static constexpr int kU = 0;                         // [128 n x 256 B] bf16
  static constexpr int kX = kU + kSsdDs * 256;         // [64 p x 256 B] bf16
  static constexpr int kBt = kX + kSsdHd * 256;        // [128 s][128 n] int8
  static constexpr int kXt = kBt + kSsdQ * 128;        // [128 s][64 p] int8
  static constexpr int kK = kXt + kSsdQ * 64;          // [128] fp32
  static constexpr int kW = kK + kSsdQ * 4;            // [128] int64
  static constexpr int kWt = kW + kSsdQ * 8;           // [4] int64
  static constexpr int kBar = kWt + 32;                // mbarrier
  static constexpr int kSlot = kBar + 8;               // TMEM address
  static constexpr int kBytes = kSlot + 16 + 1024;     // + alignment slack
};

// grid (nch, nh, B), 128 threads
__global__ void __launch_bounds__(kSsdThreads) k_ssd_state(SsdArgs a) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  using L = SsdStateSmem;
  uint8_t *sU = sm + L::kU, *sX = sm + L::kX;
  int8_t *Bt = reinterpret_cast<int8_t *>(sm + L::kBt);
  int8_t *Xt = reinterpret_cast<int8_t *>(sm + L::kXt);
  float *Ks = reinterpret_cast<float *>(sm + L::kK);
  long long *sW = reinterpret_cast<long long *>(sm + L::kW);
  long long *wtot = reinterpret_cast<long long *>(sm + L::kWt);
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + L::kBar);
  uint32_t *slot = reinterpret_cast<uint32_t *>(sm + L::kSlot);

  const int t = threadIdx.x, warp = t >> 5;
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int t0 = c * kSsdQ, nt = min(kSsdQ, a.T - t0);
  const long long row0 = (long long)b * a.T + t0;
  const long long bh = (long long)b * a.nh + h;

  const SsdDecayIn din = ssd_decay_in(a, b, h, t0, nt);
  if (t == 0) {
    mbar_init(bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) tmem_alloc(slot, 64);
  // raw code tiles, zero past the end of the sequence
#pragma unroll
  for (int i = t; i < kSsdQ * 8; i += kSsdThreads) {
    const int s = i >> 3, k = i & 7;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (s < nt) v = *reinterpret_cast<const uint4 *>(a.xbc + (row0 + s) * a.cc + a.di + k * 16);
    *reinterpret_cast<uint4 *>(Bt + s * 128 + k * 16) = v;
  }
#pragma unroll
  for (int i = t; i < kSsdQ * 4; i += kSsdThreads) {
    const int s = i >> 2, k = i & 3;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (s < nt)
      v = *reinterpret_cast<const uint4 *>(a.xbc + (row0 + s) * a.cc + (long long)h * kSsdHd + k * 16);
    *reinterpret_cast<uint4 *>(Xt + s * 64 + k * 16) = v;
  }
  const int dtq = ssd_chunk_decay(din, nt, sW, wtot);
  __syncthreads();
  const long long Wend = sW[kSsdQ - 1];
  const float dtf = __fmul_rn(__int2float_rn(dtq), 1.0f / 65536.0f);
  Ks[t] = __fmul_rn(pow2_q16(Wend - sW[t]), dtf);
  if (t == 0) a.achunk[bh * a.nch + c] = pow2_q16(Wend);
  __syncthreads();
  {  // row n = t of U: U[n][s] = bf16(K[s] Bq[s][n])
    const int n = t;
#pragma unroll 1
    for (int s = 0; s < kSsdQ; s += 8) {
      uint32_t pk[4];
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        const float u0 = __fmul_rn(Ks[s + j], (float)Bt[(s + j) * 128 + n]);
        const float u1 = __fmul_rn(Ks[s + j + 1], (float)Bt[(s + j + 1) * 128 + n]);
        pk[j / 2] = bf16_bits(u0) | (bf16_bits(u1) << 16);
      }
      *reinterpret_cast<uint4 *>(sU + sw128_off(n, s * 2, kSsdDs)) =
          make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
  }
  if (t < kSsdHd) {  // row p = t of X': X'[p][s] = bf16(X[s][p])
    const int p = t;
#pragma unroll 1
    for (int s = 0; s < kSsdQ; s += 8) {
      uint32_t pk[4];
#pragma unroll
      for (int j = 0; j < 8; j += 2)
        pk[j / 2] = bf16_bits((float)Xt[(s + j) * 64 + p]) |
                    (bf16_bits((float)Xt[(s + j + 1) * 64 + p]) << 16);
      *reinterpret_cast<uint4 *>(sX + sw128_off(p, s * 2, kSsdHd)) =
          make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  if (t == 0) {
    constexpr uint32_t idesc = bf16_idesc(128, 64);
#pragma unroll
    for (int k = 0; k < kSsdQ / 16; ++k) {
      const int atom = k >> 2, kk = k & 3;  // 4 K-steps of 32 bytes per 128-byte atom
      const uint64_t ad = sw128_desc(smem_u32(sU + atom * kSsdDs * 128)) + (uint64_t)(2 * kk);
      const uint64_t bd = sw128_desc(smem_u32(sX + atom * kSsdHd * 128)) + (uint64_t)(2 * kk);
      mma_bf16(tmem, ad, bd, idesc, k > 0 ? 1u : 0u);
    }
    mma_commit(bar);
  }
  const bool ok = mbar_drain(bar, 0);
  tc_fence_after();
  // TMEM lane n = t holds dH^T row n: 64 columns p
  float *dst = a.dH + (bh * a.nch + c) * (kSsdHd * kSsdDs) + t;
#pragma unroll 1
  for (int c0 = 0; c0 < kSsdHd; c0 += 32) {
    uint32_t r[32];
    tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, r);
    if (ok)
#pragma unroll
      for (int j = 0; j < 32; ++j) dst[(c0 + j) * kSsdDs] = __uint_as_float(r[j]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

// ------------------------------------------------------------ state passing
// grid (64 * 128 / 256, nh, B), 256 threads: one state cell per thread,
// sequential over the chunks; each group of 8 chunks' decays and dH are loaded
// before the recurrence consumes them, so the loads overlap.
constexpr int kSsdPassGroup = 8;
__global__ void __launch_bounds__(256) k_ssd_pass(SsdArgs a) {
  pdl_wait();
  pdl_trigger();
  constexpr int kCells = kSsdHd * kSsdDs;
  const int e = blockIdx.x * 256 + threadIdx.x;  // cell p * 128 + n
  const int h = blockIdx.y, b = blockIdx.z;
  const long long bh = (long long)b * a.nh + h;
  const int u_sh = a.e_h[h] - a.e_x[h] - *a.e_B;  // state word -> code units
  float H = a.state ? __fmul_rn(__int2float_rn(a.state[bh * kCells + e]), pow2f(u_sh)) : 0.0f;
  const float *__restrict__ dH = a.dH + bh * a.nch * kCells + e;
  const float *__restrict__ ach = a.achunk + bh * a.nch;
  uint16_t *__restrict__ Hin = a.Hin + bh * a.nch * kCells + e;
#pragma unroll 1
  for (int c0 = 0; c0 < a.nch; c0 += kSsdPassGroup) {
    float d[kSsdPassGroup], ac[kSsdPassGroup];
#pragma unroll
    for (int k = 0; k < kSsdPassGroup; ++k) {
      const int c = c0 + k;
      d[k] = c < a.nch ? dH[(long long)c * kCells] : 0.0f;
      ac[k] = c < a.nch ? ach[c] : 1.0f;
    }
#pragma unroll
    for (int k = 0; k < kSsdPassGroup; ++k) {
      const int c = c0 + k;
      if (c < a.nch) {
        Hin[(long long)c * kCells] = (uint16_t)bf16_bits(H);
        H = __fadd_rn(__fmul_rn(ac[k], H), d[k]);
      }
    }
  }
  if (a.state) {
    float v = rintf(__fmul_rn(H, pow2f(-u_sh)));
    v = fminf(fmaxf(v, -1073741823.0f), 1073741823.0f);
    a.state[bh * kCells + e] = (int32_t)v;
  }
}

// ------------------------------------------------------------ chunk output
// Two threads per token row (256 threads, 8 warps): warps w and w + 4 read
// the same TMEM lanes (32 (w mod 4) ..) and split the row's columns.  M reuses
// the int8 C / B tiles: it is written only after the MMA that reads them has
// completed (the wait on bar[0]), which keeps the CTA at 107 KB (two per SM).
constexpr int kSsdOutThreads = 256;
struct SsdOutSmem {
  static constexpr int kC8 = 0;                        // [128 t x 128 B] int8 (A of G)
  static constexpr int kB8 = kC8 + kSsdQ * 128;        // [128 s x 128 B] int8 (B of G)
  static constexpr int kM = kC8;                       // [128 t x 256 B] bf16, over C8 + B8
  static constexpr int kCa = kB8 + kSsdQ * 128;        // [128 t x 256 B] bf16
  static constexpr int kX = kCa + kSsdQ * 256;         // [64 p x 256 B] bf16
  static constexpr int kH = kX + kSsdHd * 256;         // [64 p x 256 B] bf16
  static constexpr int kXt = kH + kSsdHd * 256;        // [128 s][64 p] int8
  static constexpr int kDt = kXt + kSsdQ * 64;         // [128] fp32 dt
  static constexpr int kW = kDt + kSsdQ * 4;           // [128] int64
  static constexpr int kWt = kW + kSsdQ * 8;           // [4] int64
  static constexpr int kBar = kWt + 32;                // 2 mbarriers
  static constexpr int kSlot = kBar + 16;
  static constexpr int kBytes = kSlot + 16 + 1024;
};
static_assert(SsdOutSmem::kBytes <= 113 * 1024, "two k_ssd_out CTAs per SM");

// grid (nch, nh, B), 256 threads.  Order: the int8 G operands and x codes
// are loaded; G = Cq Bq^T is issued as soon as they are in; the first half
// builds Ca from the int8 C tile while the second half builds X'; Y = Ca Hq^T
// is issued; once G is complete M is built (above-diagonal 32-column blocks
// are written as zeros without reading G); Y += M X'^T; epilogue.
__global__ void __launch_bounds__(kSsdOutThreads, 2) k_ssd_out(SsdArgs a) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  using L = SsdOutSmem;
  uint8_t *sC8 = sm + L::kC8, *sB8 = sm + L::kB8, *sM = sm + L::kM, *sCa = sm + L::kCa;
  uint8_t *sX = sm + L::kX, *sH = sm + L::kH;
  int8_t *Xt = reinterpret_cast<int8_t *>(sm + L::kXt);
  float *sdt = reinterpret_cast<float *>(sm + L::kDt);
  long long *sW = reinterpret_cast<long long *>(sm + L::kW);
  long long *wtot = reinterpret_cast<long long *>(sm + L::kWt);
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + L::kBar);
  uint32_t *slot = reinterpret_cast<uint32_t *>(sm + L::kSlot);

  const int t = threadIdx.x, warp = t >> 5;
  const int r = t & (kSsdQ - 1);  // token row (and TMEM lane) of this thread
  const int half = t >> 7;        // which half of the row's columns
  const int q = warp & 3;         // TMEM lane quarter: rows 32 q .. 32 q + 31
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int t0 = c * kSsdQ, nt = min(kSsdQ, a.T - t0);
  const long long row0 = (long long)b * a.T + t0;
  const long long bh = (long long)b * a.nh + h;

  // every scalar input, loaded up front (their latency overlaps the tile loads)
  const SsdDecayIn din = ssd_decay_in(a, b, h, t0, nt);
  const int s_y = *a.e_C + a.e_x[h] + *a.e_B - a.e_y[h];
  const int s_D = a.e_y[h] - a.e_D[h] - a.e_x[h];
  const long long Dq = a.D_q[h];
  if (t == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    tmem_alloc(slot, 256);  // G: columns 0..127 (int32), Y: 128..191 (fp32)
    tc_fence_before();
  }

  // the chunk's B and C rows (int8 operands of G) and x codes, zero past the
  // end: 16 threads per token row (the B | C bytes are contiguous), so each
  // warp load covers two whole 256-byte rows
#pragma unroll
  for (int i = t; i < kSsdQ * 16; i += kSsdOutThreads) {
    const int s = i >> 4, k = i & 15;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (s < nt) v = *reinterpret_cast<const uint4 *>(a.xbc + (row0 + s) * a.cc + a.di + k * 16);
    uint8_t *dst = k < 8 ? sB8 + sw128_off(s, k * 16, kSsdQ) : sC8 + sw128_off(s, (k - 8) * 16, kSsdQ);
    *reinterpret_cast<uint4 *>(dst) = v;
  }
#pragma unroll
  for (int i = t; i < kSsdQ * 4; i += kSsdOutThreads) {
    const int s = i >> 2, k = i & 3;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (s < nt)
      v = *reinterpret_cast<const uint4 *>(a.xbc + (row0 + s) * a.cc + (long long)h * kSsdHd + k * 16);
    *reinterpret_cast<uint4 *>(Xt + xt_off(s, k * 16)) = v;
  }
  fence_proxy_async_smem();  // the G tiles, for the tensor cores
  // (its CTA barrier makes the tiles, the barriers and the TMEM address
  // visible to every thread)
  const int dtq = ssd_chunk_decay(din, nt, sW, wtot);
  tc_fence_after();
  const uint32_t tmem = *slot;
  if (t == 0) {  // G = Cq Bq^T, exact int32 in TMEM columns 0..127
    constexpr uint32_t idesc = i8_idesc(128, 128);
    const uint64_t ad = sw128_desc(smem_u32(sC8)), bd = sw128_desc(smem_u32(sB8));
#pragma unroll
    for (int k = 0; k < 4; ++k) mma_i8(tmem, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), idesc, k > 0 ? 1u : 0u);
    mma_commit(&bar[0]);
  }
  if (half == 0) {
    sdt[r] = __fmul_rn(__int2float_rn(dtq), 1.0f / 65536.0f);
    // row r of Ca: bf16(2^W[r] Cq[r][n]), Cq read back from the int8 tile
    // (the MMA reads the same tile; neither writes it)
    const float a0 = pow2_q16(sW[r]);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint4 cv = *reinterpret_cast<const uint4 *>(sC8 + sw128_off(r, k * 16, kSsdQ));
      const uint32_t wv[4] = {cv.x, cv.y, cv.z, cv.w};
      uint32_t pk[8];
#pragma unroll
      for (int qq = 0; qq < 4; ++qq)
#pragma unroll
        for (int j = 0; j < 4; j += 2) {
          const float c0v = __fmul_rn(a0, (float)(int8_t)((wv[qq] >> (8 * j)) & 0xFF));
          const float c1v = __fmul_rn(a0, (float)(int8_t)((wv[qq] >> (8 * (j + 1))) & 0xFF));
          pk[qq * 2 + j / 2] = bf16_bits(c0v) | (bf16_bits(c1v) << 16);
        }
      // 16 int8 -> 16 bf16 = 32 bytes: two 16-byte pieces at bf16 columns 16k .. 16k+15
      *reinterpret_cast<uint4 *>(sCa + sw128_off(r, k * 32, kSsdQ)) =
          make_uint4(pk[0], pk[1], pk[2], pk[3]);
      *reinterpret_cast<uint4 *>(sCa + sw128_off(r, k * 32 + 16, kSsdQ)) =
          make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
  } else {
    // X': row p holds bf16 x[s][p] over s; thread r builds the 8-token
    // pieces i = r, r + 128, ... of the 16 x 64 grid (p = i mod 64: a warp
    // reads 32 consecutive bytes of each token row)
#pragma unroll 2
    for (int i = r; i < kSsdHd * (kSsdQ / 8); i += kSsdQ) {
      const int p = i & (kSsdHd - 1), s = (i >> 6) * 8;
      uint32_t pk[4];
#pragma unroll
      for (int j = 0; j < 8; j += 2)
        pk[j / 2] = bf16_bits((float)Xt[xt_off(s + j, p)]) |
                    (bf16_bits((float)Xt[xt_off(s + j + 1, p)]) << 16);
      *reinterpret_cast<uint4 *>(sX + sw128_off(p, s * 2, kSsdHd)) =
          make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
  }
  {  // the bf16 state entering the chunk, rows p: 64 x 256 bytes
    const uint4 *src = reinterpret_cast<const uint4 *>(a.Hin + (bh * a.nch + c) * (kSsdHd * kSsdDs));
#pragma unroll
    for (int i = t; i < kSsdHd * 16; i += kSsdOutThreads) {
      const int p = i >> 4, j = i & 15;  // 16-byte piece j of row p
      *reinterpret_cast<uint4 *>(sH + sw128_off(p, j * 16, kSsdHd)) = src[i];
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();  // Ca, X', H, sdt, sW complete
  tc_fence_after();
  constexpr uint32_t idesc_y = bf16_idesc(128, 64);
  const uint32_t dY = tmem + 128;
  if (t == 0) {  // Y = Ca Hq^T, fp32 in TMEM columns 128..191
#pragma unroll
    for (int k = 0; k < kSsdDs / 16; ++k) {
      const int atom = k >> 2, kk = k & 3;
      const uint64_t ad = sw128_desc(smem_u32(sCa + atom * kSsdQ * 128)) + (uint64_t)(2 * kk);
      const uint64_t bd = sw128_desc(smem_u32(sH + atom * kSsdHd * 128)) + (uint64_t)(2 * kk);
      mma_bf16(dY, ad, bd, idesc_y, k > 0 ? 1u : 0u);
    }
  }
  bool ok = mbar_drain(&bar[0], 0);
  tc_fence_after();
  {  // row r of M: bf16(G[r][s] * fl32(2^(W[r]-W[s]) dt[s])) for s <= r, else 0;
     // this thread takes the 32-column blocks half, half + 2
    const long long Wr = sW[r];
#pragma unroll 1
    for (int s0 = half * 32; s0 < kSsdQ; s0 += 64) {
      if (s0 <= 32 * q + 31) {  // the warp's rows reach this block (warp-uniform)
        uint32_t g[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)s0, g);
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
          uint32_t pk[4];
#pragma unroll
          for (int qq = 0; qq < 8; qq += 2) {
            float m2[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int s = s0 + j + qq + e;
              float m = 0.0f;
              if (s <= r) {  // |G| <= 128 * 127^2 < 2^22: exact without the conversion unit
                const float ad = __fmul_rn(pow2_q16_decay(Wr - sW[s]), sdt[s]);
                m = __fmul_rn(small_i2f((int)g[j + qq + e]), ad);
              }
              m2[e] = m;
            }
            pk[qq / 2] = bf16_bits(m2[0]) | (bf16_bits(m2[1]) << 16);
          }
          *reinterpret_cast<uint4 *>(sM + sw128_off(r, (s0 + j) * 2, kSsdQ)) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; j += 8)
          *reinterpret_cast<uint4 *>(sM + sw128_off(r, (s0 + j) * 2, kSsdQ)) =
              make_uint4(0u, 0u, 0u, 0u);
      }
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (t == 0) {  // Y += M X'^T
#pragma unroll
    for (int k = 0; k < kSsdQ / 16; ++k) {
      const int atom = k >> 2, kk = k & 3;
      const uint64_t ad = sw128_desc(smem_u32(sM + atom * kSsdQ * 128)) + (uint64_t)(2 * kk);
      const uint64_t bd = sw128_desc(smem_u32(sX + atom * kSsdHd * 128)) + (uint64_t)(2 * kk);
      mma_bf16(dY, ad, bd, idesc_y, 1u);
    }
    mma_commit(&bar[1]);
  }
  ok = mbar_drain(&bar[1], 0) && ok;
  tc_fence_after();
  // the y tile is staged in shared memory (M and Ca are dead once the MMAs
  // that read them have completed; rows padded to 68 words) and written out
  // in whole rows
  constexpr int kYStride = kSsdHd + 4;
  int32_t *sY = reinterpret_cast<int32_t *>(sm + L::kC8);
  static_assert(kSsdQ * kYStride * 4 <= L::kX - L::kC8, "the y tile fits over M and Ca");
  {  // y codes of token r, columns 32 half ..: rint(Y 2^(e_C+e_x+e_B-e_y)) + rshr(D_q x, s_D), saturated
    const float scale = pow2f(s_y);
    const int c0 = half * 32;
    uint32_t yv[32];
    tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(128 + c0), yv);
    // this row's 32 x codes (two 16-byte pieces)
    const uint4 xa = *reinterpret_cast<const uint4 *>(Xt + xt_off(r, c0));
    const uint4 xb = *reinterpret_cast<const uint4 *>(Xt + xt_off(r, c0 + 16));
    const uint32_t xw[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      int v4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        // rint of a float is an integer; the int64 conversion is exact
        const long long yc = __float2ll_rn(rintf(__fmul_rn(__uint_as_float(yv[j + e]), scale)));
        const int xc = (int)(int8_t)((xw[(j + e) >> 2] >> (8 * ((j + e) & 3))) & 0xFFu);
        const long long skip = rshr64(Dq * (long long)xc, s_D);
        long long v = yc + skip;
        v = v < -2147483647LL ? -2147483647LL : (v > 2147483647LL ? 2147483647LL : v);
        v4[e] = (int)v;
      }
      *reinterpret_cast<int4 *>(sY + r * kYStride + c0 + j) = make_int4(v4[0], v4[1], v4[2], v4[3]);
    }
  }
  __syncthreads();
  if (ok) {  // 16 threads per token row of 64 int32
#pragma unroll
    for (int i = t; i < kSsdQ * 16; i += kSsdOutThreads) {
      const int s = i >> 4, k = i & 15;
      if (s < nt)
        *reinterpret_cast<int4 *>(a.y + (row0 + s) * a.di + (long long)h * kSsdHd + k * 4) =
            *reinterpret_cast<const int4 *>(sY + s * kYStride + k * 4);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace fm
