// k_gemm.cuh -- W8A8 GEMM on the 5th-generation tensor cores (tcgen05, kind::i8).
//
// acc[m, n] = sum_k A[m, k] W[n, k] in exact int32 (Hadamard-rotated int8
// operands; FastMamba, arXiv 2505.18975, pith.science review "What carries
// the argument": Y = (XH)(H^T W^T)), followed by the dequantisation
// fl(fl(float(acc) * s_x[m]) * s_w[n]) and either a plain fp32 store (+ an
// optional residual) or the in_proj split into z / xBC power-of-two codes /
// dt (Mamba2 column order).
//
// Two kernels share the pieces below.  k_gemm_i8_tc (small grids: one
// 128 x BN output tile per CTA, 6 warps, two CTAs per SM):
//   warp 0      TMA producer: 128-byte-swizzled A and W tiles (128 x 128 and
//               BN x 128 int8) into a STAGES-deep shared-memory ring;
//   warp 1      allocates TMEM (BN columns of int32) and one elected lane
//               issues tcgen05.mma (M=128, N=BN, K=32 per instruction);
//               tcgen05.commit frees each ring slot and finally signals the
//               accumulator;
//   warps 2..5  epilogue: tcgen05.ld 32 columns at a time from their TMEM
//               lane quarter, dequantise and store.
// k_gemm_i8_persist (large grids, further below): one CTA per SM walking the
// tiles, the accumulator double-buffered in TMEM, 8 epilogue warps writing
// through TMA stores.
// Every mbarrier wait is bounded by a wall-clock limit; on expiry the thread
// sets the device error word and the kernel runs to its end (TMEM is always
// released), so a broken pipeline can never hang the GPU.
#pragma once
#include <cuda.h>
#include "fm_common.cuh"

namespace fm {

constexpr int kGemmBM = 128;
constexpr int kGemmBK = 128;  // int8 elements = bytes per row per stage (one swizzle atom)
constexpr int kGemmThreads = 192;
constexpr unsigned long long kWaitLimitNs = 4000000000ull;  // 4 s

// Failure injection for the tests of the bounded-wait path (set by
// fm_set_fault_injection; both per device, zero-cost when unset):
//   g_wait_limit_ns  the limit of the pipeline waits (kWaitLimitNs by default)
//   g_test_stall     bit 0: the GEMM producers issue no loads; bit 1: the
//                    scan producer issues no copies -- the consumers then wait
//                    on a barrier nothing completes, with nothing in flight
// Drains (waits for work already issued) always use the fixed kWaitLimitNs.
__device__ unsigned long long g_wait_limit_ns = kWaitLimitNs;
__device__ int g_test_stall = 0;
constexpr int kStallGemm = 1, kStallScan = 2;

struct GemmEpilogue {
  int mode;  // 0: plain (Y, residual), 1: in_proj split
  long long M, N;
  const float *s_x, *s_w;
  const float *residual;
  float *Y;
  int32_t *acc_out;
  // in_proj split
  int di, cc, nh;
  const int32_t *e_u;
  float *z;
  int8_t *xbc;
  float *dt;
  // persistent kernel only: write the outputs through TMA stores (the tensor
  // maps passed beside this struct); 0 falls back to per-thread stores
  int tma_store;
  // split-K (small-grid kernel, gridDim.z > 1): each K slice adds its int32
  // partial sums into split_acc [M, N] (zeroed by the host); the dequantising
  // epilogue then runs once on the exact total (k_gemm_splitk_epilogue)
  int32_t *split_acc;
};

// ------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// bounded wait: false (and the error word set) if the phase does not
// complete within `limit` ns
__device__ __forceinline__ bool mbar_wait_for(uint64_t *bar, uint32_t parity,
                                              unsigned long long limit) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer() - t0 > limit) {
      raise_error(kErrTimeout);
      return false;
    }
  }
}
// a pipeline wait (its limit can be lowered for the failure tests)
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_for(bar, parity, *(volatile unsigned long long *)&g_wait_limit_ns);
}
// a wait expected to be long (a producer waiting for its consumers, epilogue
// warps waiting out the whole main loop): the thread sleeps between polls, so
// it takes few issue slots from the warps doing the work
__device__ __forceinline__ bool mbar_wait_sleepy(uint64_t *bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long limit = *(volatile unsigned long long *)&g_wait_limit_ns;
  const unsigned long long t0 = globaltimer();
  while (true) {
    __nanosleep(128);
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer() - t0 > limit) {
      raise_error(kErrTimeout);
      return false;
    }
  }
}
// a drain: waits for work this CTA has already issued, at the fixed limit
__device__ __forceinline__ bool mbar_drain(uint64_t *bar, uint32_t parity) {
  return mbar_wait_for(bar, parity, kWaitLimitNs);
}
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *tm, int c0, int c1,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"((unsigned long long)tm), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}
// TMA store of a 2-D box from shared memory (bulk-group completion)
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *tm, int c0, int c1,
                                             const void *src) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
          (unsigned long long)tm),
      "r"(c0), "r"(c1), "r"(smem_u32(src))
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// the shared-memory sources of every committed store have been read
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// every committed store has completed
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Shared-memory matrix descriptor (sm_100 format): K-major operand whose rows
// are 128 bytes, 128-byte swizzle, 8-row groups 1024 bytes apart.
//   bits  0-13 start address >> 4      bits 16-29 leading byte offset >> 4 (1, unused)
//   bits 32-45 stride byte offset >> 4 (1024 >> 4)
//   bits 46-47 descriptor version (1)  bits 61-63 layout (2 = 128-byte swizzle)
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}
// Instruction descriptor, kind::i8: D = s32 (bits 4-5 = 2), A and B signed
// int8 (bits 7-9 = 1, 10-12 = 1), both K-major, N >> 3 at bits 17-22,
// M >> 4 at bits 24-28.
__host__ __device__ constexpr uint32_t i8_idesc(int M, int N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void mma_i8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ar: rows of A staged per stage (kGemmBM, or 64 for a decode batch)
__host__ __device__ constexpr int gemm_smem_bytes(int BN, int stages, int ar = kGemmBM) {
  return stages * (ar + BN) * kGemmBK + 1024 /*align slack*/ + 256 /*barriers*/ +
         2 * BN * 4 /*staged column scales*/;
}

// ------------------------------------------------------------ epilogue
__device__ __forceinline__ float pow2f(int e) {  // exact 2^e for e in [-126, 127]
  return __int_as_float((127 + e) << 23);
}

// One 32-column chunk of one output row.  colw / cole: this chunk's column
// scales s_w and (split mode) the PoT factors 2^-e_u staged in shared memory.
__device__ __forceinline__ void gemm_store_chunk(const GemmEpilogue &ep, long long row, float sx,
                                                 long long col0, uint32_t (&r)[32],
                                                 const float *colw, const float *cole) {
  if (row >= ep.M) return;
  const bool full = col0 + 32 <= ep.N;
  if (ep.acc_out) {
    int32_t *dst = ep.acc_out + row * ep.N + col0;
    for (int j = 0; j < 32; ++j)
      if (col0 + j < ep.N) dst[j] = (int32_t)r[j];
  }
  // dequantise in place (the accumulator registers become the fp32 values)
  float(&y)[32] = reinterpret_cast<float(&)[32]>(r);
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    const float4 sw = *reinterpret_cast<const float4 *>(colw + j);
    y[j] = __fmul_rn(__fmul_rn(__int2float_rn((int)r[j]), sx), sw.x);
    y[j + 1] = __fmul_rn(__fmul_rn(__int2float_rn((int)r[j + 1]), sx), sw.y);
    y[j + 2] = __fmul_rn(__fmul_rn(__int2float_rn((int)r[j + 2]), sx), sw.z);
    y[j + 3] = __fmul_rn(__fmul_rn(__int2float_rn((int)r[j + 3]), sx), sw.w);
  }
  if (ep.mode == 0) {
    float *dst = ep.Y + row * ep.N + col0;
    const float *res = ep.residual ? ep.residual + row * ep.N + col0 : nullptr;
    if (full && ((ep.N & 3) == 0)) {
      float4 rv[8];
      if (res) {
#pragma unroll
        for (int j = 0; j < 8; ++j) rv[j] = *reinterpret_cast<const float4 *>(res + 4 * j);
      }
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        float4 o = make_float4(y[j], y[j + 1], y[j + 2], y[j + 3]);
        if (res) {
          o.x = __fadd_rn(rv[j / 4].x, o.x);
          o.y = __fadd_rn(rv[j / 4].y, o.y);
          o.z = __fadd_rn(rv[j / 4].z, o.z);
          o.w = __fadd_rn(rv[j / 4].w, o.w);
        }
        *reinterpret_cast<float4 *>(dst + j) = o;
      }
    } else {
      for (int j = 0; j < 32; ++j) {
        if (col0 + j >= ep.N) break;
        dst[j] = res ? __fadd_rn(res[j], y[j]) : y[j];
      }
    }
    return;
  }
  // in_proj split: [0, di) z | [di, di+cc) xBC codes | [di+cc, N) dt
  const long long di = ep.di, cc = ep.cc;
  if (full && col0 + 32 <= di && (di & 3) == 0) {
    float *dst = ep.z + row * di + col0;
#pragma unroll
    for (int j = 0; j < 32; j += 4)
      *reinterpret_cast<float4 *>(dst + j) = make_float4(y[j], y[j + 1], y[j + 2], y[j + 3]);
    return;
  }
  if (full && col0 >= di && col0 + 32 <= di + cc && ((col0 - di) & 15) == 0 && (cc & 15) == 0) {
    const long long c0 = col0 - di;
    uint32_t packed[8];
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      const float4 es = *reinterpret_cast<const float4 *>(cole + j);
      const float e4[4] = {es.x, es.y, es.z, es.w};
      uint32_t w = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int code = quant127(__fmul_rn(y[j + b], e4[b]));
        w |= ((uint32_t)(code & 0xFF)) << (8 * b);
      }
      packed[j / 4] = w;
    }
    uint4 *dst = reinterpret_cast<uint4 *>(ep.xbc + row * cc + c0);
    dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
    return;
  }
  for (int j = 0; j < 32; ++j) {
    const long long c = col0 + j;
    if (c >= ep.N) break;
    if (c < di) {
      ep.z[row * di + c] = y[j];
    } else if (c < di + cc) {
      ep.xbc[row * cc + (c - di)] = (int8_t)quant127(__fmul_rn(y[j], cole[j]));
    } else {
      ep.dt[row * ep.nh + (c - di - cc)] = y[j];
    }
  }
}

// ------------------------------------------------------------ the kernel
// AR: rows of A staged per stage (128, or 64 when M <= 64: a decode batch,
// whose A box then has 64 rows).  The MMA always reads a 128-row A tile; with
// AR = 64 the tile's rows 64..127 are the next 8 KB of shared memory (the next
// stage's A rows, or for the last stage the start of the B ring: always inside
// the allocation), which only feed accumulator rows >= M that the epilogue
// never stores.  The L2 -> shared traffic of A and its ring space halve, so
// the ring can be deeper.
template <int BN, int STAGES, bool SPLIT = false, int AR = kGemmBM>
__global__ void __launch_bounds__(kGemmThreads, 2)
    k_gemm_i8_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 int num_k_blocks, int kb_per_split, GemmEpilogue ep) {
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN");
  static_assert(AR == kGemmBM || (AR == 64 && STAGES * BN >= 64),
                "a 64-row A stage reads 64 more rows, inside the ring");
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + STAGES * AR * kGemmBK;
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(sB + STAGES * BN * kGemmBK);
  uint64_t *empty_bar = full_bar + STAGES;
  uint64_t *accum_bar = empty_bar + STAGES;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(accum_bar + 1);
  // [BN] s_w of this tile, 16-byte aligned (read as float4)
  float *col_w = reinterpret_cast<float *>((reinterpret_cast<uintptr_t>(tmem_slot + 1) + 15) &
                                           ~static_cast<uintptr_t>(15));
  float *col_e = col_w + BN;                                // [BN] 2^-e_u (split mode)

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * kGemmBM;
  const int n0 = blockIdx.x * BN;
  // this CTA's K slice (SPLIT: the host launches only non-empty slices, so
  // kb_n >= 1; otherwise the whole K)
  const int kb0 = SPLIT ? (int)blockIdx.z * kb_per_split : 0;
  const int kb_n = SPLIT ? min(kb_per_split, num_k_blocks - kb0) : num_k_blocks;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(accum_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"((unsigned long long)&tmA) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"((unsigned long long)&tmB) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"((uint32_t)BN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The prologue above touches only this CTA's shared memory and TMEM.  Under
  // programmatic dependent launch (fm_set_pdl) the weights -- written long
  // before -- are fetched for the first stages while the previous kernel
  // drains; only the producer lane (before the activations) and the epilogue
  // warps (before the row scales and the residual) wait for it.
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      const int kb_issue = (g_test_stall & kStallGemm) ? 0 : kb_n;
      const int pre = kb_issue < STAGES ? kb_issue : STAGES;
      for (int kb = 0; kb < pre; ++kb) {  // fresh ring: no empty-slot wait
        mbar_arrive_expect_tx(&full_bar[kb], (uint32_t)((AR + BN) * kGemmBK));
        tma_load_2d(sB + kb * BN * kGemmBK, &tmB, (kb0 + kb) * kGemmBK, n0, &full_bar[kb]);
      }
      pdl_wait();
      for (int kb = 0; kb < pre; ++kb)
        tma_load_2d(sA + kb * AR * kGemmBK, &tmA, (kb0 + kb) * kGemmBK, m0, &full_bar[kb]);
      int issued = pre;
      for (int kb = pre; kb < kb_issue; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = (uint32_t)(kb / STAGES) & 1u;
        if (!mbar_wait(&empty_bar[s], ph ^ 1u)) break;
        mbar_arrive_expect_tx(&full_bar[s], (uint32_t)((AR + BN) * kGemmBK));
        tma_load_2d(sA + s * AR * kGemmBK, &tmA, (kb0 + kb) * kGemmBK, m0, &full_bar[s]);
        tma_load_2d(sB + s * BN * kGemmBK, &tmB, (kb0 + kb) * kGemmBK, n0, &full_bar[s]);
        ++issued;
      }
      // every copy issued must have landed before the CTA may exit (on the
      // normal path the MMA lane has consumed them all and these return at once)
      for (int j = issued > STAGES ? issued - STAGES : 0; j < issued; ++j)
        if (!mbar_drain(&full_bar[j % STAGES], (uint32_t)(j / STAGES) & 1u)) break;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = i8_idesc(kGemmBM, BN);
      for (int kb = 0; kb < kb_n; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = (uint32_t)(kb / STAGES) & 1u;
        if (!mbar_wait(&full_bar[s], ph)) break;
        tc_fence_after();
        const uint64_t ad = sw128_desc(smem_u32(sA + s * AR * kGemmBK));
        const uint64_t bd = sw128_desc(smem_u32(sB + s * BN * kGemmBK));
#pragma unroll
        for (int k = 0; k < kGemmBK / 32; ++k) {
          // advance the start address by 32 bytes (2 x 16 B) per K=32 slice
          mma_i8(tmem_base, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), idesc,
                 (kb > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(&empty_bar[s]);
      }
      mma_commit(accum_bar);
      // every MMA issued must have completed before TMEM is released
      mbar_drain(accum_bar, 0);
    }
  } else {
    pdl_wait();
    // while the main loop runs: stage this tile's column scales and the row scale
    const int et = threadIdx.x - 64;  // 0 .. 127
    for (int j = et; j < BN; j += 128) {
      const long long c = (long long)n0 + j;
      col_w[j] = c < ep.N ? ep.s_w[c] : 0.0f;
      float e = 0.0f;
      if (ep.mode == 1 && c >= ep.di && c < (long long)ep.di + ep.cc) e = pow2f(-ep.e_u[c - ep.di]);
      col_e[j] = e;
    }
    const int quarter = warp & 3;  // TMEM lanes [32*quarter, 32*quarter + 32)
    const long long row = (long long)m0 + quarter * 32 + lane;
    const float sx = row < ep.M ? ep.s_x[row] : 0.0f;
    asm volatile("bar.sync 1, 128;" ::: "memory");  // the 4 epilogue warps only
    // tcgen05.ld is warp-collective: the whole warp skips it after a failed wait
    const bool ok = __all_sync(0xffffffffu, mbar_wait_sleepy(accum_bar, 0));
    tc_fence_after();
#pragma unroll 1
    for (int c = 0; c < BN && ok; c += 32) {
      uint32_t r[32];
      tmem_ld32(tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)c, r);
      if (n0 + c >= ep.N) continue;
      if constexpr (SPLIT) {  // add this slice's exact partial sums
        if (row < ep.M) {
          int32_t *dst = ep.split_acc + row * ep.N + n0 + c;
          for (int j = 0; j < 32 && n0 + c + j < ep.N; ++j) atomicAdd(dst + j, (int)r[j]);
        }
      } else {
        gemm_store_chunk(ep, row, sx, (long long)n0 + c, r, col_w + c, col_e + c);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"((uint32_t)BN)
                 : "memory");
  }
}

// ------------------------------------------------------------ split K in a cluster
// A decode batch (M <= 64) whose output tiles are fewer than the SMs (the
// out_proj): each tile's K is split over the S CTAs of a thread-block cluster
// (cluster dims (1, 1, S), rank = the K slice), so every SM streams a share of
// the weights and of the activations.  Each CTA accumulates its slice's exact
// int32 partial sums in TMEM; ranks 1..S-1 copy theirs to their own shared
// memory, and after a cluster barrier rank 0 adds them (distributed shared
// memory loads) to its own and runs the unchanged epilogue, so the outputs
// are bit-identical to the unsplit kernel.  A second cluster barrier keeps
// every CTA's shared memory alive until rank 0 has read it.  Every thread of
// every CTA reaches both barriers: the kernel has no early exit and all its
// waits are bounded.  Plain TMA loads only (no multicast).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t dsmem_map(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
__device__ __forceinline__ uint4 dsmem_ld4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

constexpr int kClPad = 4;  // int32 words of padding per partial-sum row
__host__ __device__ constexpr int gemm_cl_smem_bytes(int BN, int stages) {
  return stages * (64 + BN) * kGemmBK + kGemmBM * (BN + kClPad) * 4 + 1024 /*align slack*/ +
         256 /*barriers*/ + 2 * BN * 4 /*staged column scales*/;
}

// grid (ceil(N / BN), 1, S), cluster (1, 1, S), kGemmThreads threads; the
// host gives every rank at least one K block (kb_per_rank * (S - 1) < nkb)
template <int BN, int STAGES, int S>
__global__ void __launch_bounds__(kGemmThreads)
    k_gemm_i8_cl(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 int num_k_blocks, int kb_per_rank, GemmEpilogue ep) {
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 128, "BN");
  static_assert(STAGES * BN >= 64, "a 64-row A stage reads 64 more rows, inside the ring");
  static_assert(S >= 2 && S <= 8, "portable cluster sizes");
  constexpr int AR = 64;
  constexpr int PSTR = BN + kClPad;  // partial-sum row stride (int32 words)
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + STAGES * AR * kGemmBK;
  int32_t *part = reinterpret_cast<int32_t *>(sB + STAGES * BN * kGemmBK);  // [128][PSTR]
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(part + kGemmBM * PSTR);
  uint64_t *empty_bar = full_bar + STAGES;
  uint64_t *accum_bar = empty_bar + STAGES;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(accum_bar + 1);
  float *col_w = reinterpret_cast<float *>((reinterpret_cast<uintptr_t>(tmem_slot + 1) + 15) &
                                           ~static_cast<uintptr_t>(15));
  float *col_e = col_w + BN;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN;
  const uint32_t rank = cluster_rank();
  const int kb0 = (int)rank * kb_per_rank;
  const int kb_n = max(0, min(kb_per_rank, num_k_blocks - kb0));

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(accum_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"((unsigned long long)&tmA) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"((unsigned long long)&tmB) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"((uint32_t)BN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_trigger();

  bool ok = true;  // this thread's accumulator wait (epilogue warps)
  if (warp == 0) {
    if (lane == 0) {
      const int kb_issue = (g_test_stall & kStallGemm) ? 0 : kb_n;
      const int pre = kb_issue < STAGES ? kb_issue : STAGES;
      for (int kb = 0; kb < pre; ++kb) {  // fresh ring: no empty-slot wait
        mbar_arrive_expect_tx(&full_bar[kb], (uint32_t)((AR + BN) * kGemmBK));
        tma_load_2d(sB + kb * BN * kGemmBK, &tmB, (kb0 + kb) * kGemmBK, n0, &full_bar[kb]);
      }
      pdl_wait();
      for (int kb = 0; kb < pre; ++kb)
        tma_load_2d(sA + kb * AR * kGemmBK, &tmA, (kb0 + kb) * kGemmBK, 0, &full_bar[kb]);
      int issued = pre;
      for (int kb = pre; kb < kb_issue; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = (uint32_t)(kb / STAGES) & 1u;
        if (!mbar_wait(&empty_bar[s], ph ^ 1u)) break;
        mbar_arrive_expect_tx(&full_bar[s], (uint32_t)((AR + BN) * kGemmBK));
        tma_load_2d(sA + s * AR * kGemmBK, &tmA, (kb0 + kb) * kGemmBK, 0, &full_bar[s]);
        tma_load_2d(sB + s * BN * kGemmBK, &tmB, (kb0 + kb) * kGemmBK, n0, &full_bar[s]);
        ++issued;
      }
      for (int j = issued > STAGES ? issued - STAGES : 0; j < issued; ++j)
        if (!mbar_drain(&full_bar[j % STAGES], (uint32_t)(j / STAGES) & 1u)) break;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = i8_idesc(kGemmBM, BN);
      for (int kb = 0; kb < kb_n; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = (uint32_t)(kb / STAGES) & 1u;
        if (!mbar_wait(&full_bar[s], ph)) break;
        tc_fence_after();
        const uint64_t ad = sw128_desc(smem_u32(sA + s * AR * kGemmBK));
        const uint64_t bd = sw128_desc(smem_u32(sB + s * BN * kGemmBK));
#pragma unroll
        for (int k = 0; k < kGemmBK / 32; ++k)
          mma_i8(tmem_base, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), idesc,
                 (kb > 0 || k > 0) ? 1u : 0u);
        mma_commit(&empty_bar[s]);
      }
      mma_commit(accum_bar);
      mbar_drain(accum_bar, 0);
    }
  } else {
    pdl_wait();
    const int et = threadIdx.x - 64;  // 0 .. 127
    if (rank == 0) {  // the tile's column scales (used after the first cluster barrier)
      for (int j = et; j < BN; j += 128) {
        const long long c = (long long)n0 + j;
        col_w[j] = c < ep.N ? ep.s_w[c] : 0.0f;
        float e = 0.0f;
        if (ep.mode == 1 && c >= ep.di && c < (long long)ep.di + ep.cc) e = pow2f(-ep.e_u[c - ep.di]);
        col_e[j] = e;
      }
    }
    ok = __all_sync(0xffffffffu, mbar_wait_sleepy(accum_bar, 0));
    tc_fence_after();
    if (rank != 0) {  // this slice's partial sums into shared memory, row by row
      const int quarter = warp & 3;
      const int row = quarter * 32 + lane;
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        uint32_t r[32];
        if (ok) tmem_ld32(tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)c, r);
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          *reinterpret_cast<uint4 *>(part + row * PSTR + c + j) =
              ok ? make_uint4(r[j], r[j + 1], r[j + 2], r[j + 3]) : make_uint4(0u, 0u, 0u, 0u);
      }
    }
  }
  tc_fence_before();
  cluster_sync_all();  // every slice's partial sums written and visible
  tc_fence_after();
  if (rank == 0 && warp >= 2 && ok) {
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const float sx = row < ep.M ? ep.s_x[row] : 0.0f;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      uint32_t r[32];
      tmem_ld32(tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)c, r);
      if (n0 + c >= ep.N) continue;
      const uint32_t local = smem_u32(part + row * PSTR + c);
#pragma unroll 1
      for (int q = 1; q < S; ++q) {  // exact int32 sums, any order
        const uint32_t remote = dsmem_map(local, (uint32_t)q);
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const uint4 v = dsmem_ld4(remote + 4u * (uint32_t)j);
          r[j] += v.x;
          r[j + 1] += v.y;
          r[j + 2] += v.z;
          r[j + 3] += v.w;
        }
      }
      gemm_store_chunk(ep, row, sx, (long long)n0 + c, r, col_w + c, col_e + c);
    }
  }
  cluster_sync_all();  // rank 0 has read every slice: the CTAs may leave
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"((uint32_t)BN)
                 : "memory");
  }
}

// The dequantising epilogue of a split-K GEMM: one thread per (row, 32-column
// chunk) reads the exact int32 totals and runs the same gemm_store_chunk as
// the unsplit kernels, so the outputs are bit-identical to theirs.
__global__ void __launch_bounds__(128) k_gemm_splitk_epilogue(GemmEpilogue ep) {
  pdl_wait();
  pdl_trigger();
  const long long nchunk = (ep.N + 31) / 32;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= ep.M * nchunk) return;
  const long long row = i / nchunk, col0 = (i % nchunk) * 32;
  uint32_t r[32];
  __align__(16) float colw[32];
  __align__(16) float cole[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const long long c = col0 + j;
    const bool in = c < ep.N;
    r[j] = in ? (uint32_t)ep.split_acc[row * ep.N + c] : 0u;
    colw[j] = in ? ep.s_w[c] : 0.0f;
    float e = 0.0f;
    if (in && ep.mode == 1 && c >= ep.di && c < (long long)ep.di + ep.cc) e = pow2f(-ep.e_u[c - ep.di]);
    cole[j] = e;
  }
  gemm_store_chunk(ep, row, ep.s_x[row], col0, r, colw, cole);
}

// ------------------------------------------------------------ the persistent kernel
// One CTA per SM walks the output tiles (tile t = m_blk * n_tiles + n_blk,
// strided by the grid), so the set/teardown cost is paid once and the
// epilogue of tile i overlaps the main loop of tile i + 1: the accumulator is
// double-buffered in TMEM (2 x BN int32 columns).
//   warp 0          TMA producer (the smem ring runs across tile boundaries)
//   warp 1          TMEM allocation; one lane issues tcgen05.mma, commits each
//                   ring slot back to the producer and each finished
//                   accumulator to the epilogue
//   warps 2..2+EW   epilogue: EW / 4 warps per TMEM lane quarter, each taking
//                   BN / (EW / 4) columns; the accumulator is handed back to
//                   the MMA warp as soon as its last tcgen05.ld has completed
// Barriers: full[s] / empty[s] for the ring, tfull[a] / tempty[a] for the two
// accumulators.  Every wait is bounded; after a failed wait a thread stops
// waiting (it still meets its named barriers), the MMA lane drains its
// outstanding MMAs and the producer its outstanding copies before TMEM is
// released, so the kernel always ends.
template <int BN, int STAGES, int EW>
struct PersistSmem {
  static constexpr int kA = kGemmBM * kGemmBK;  // bytes per A stage
  static constexpr int kB = BN * kGemmBK;       // bytes per B stage
  static constexpr int kStage = 4096;           // per epilogue warp: 32 rows x 128 bytes
  static constexpr int kBytes = 1024 /*align slack*/ + STAGES * (kA + kB) + EW * kStage +
                                (2 * STAGES + 5) * 8 /*barriers*/ + 16 /*tmem slot*/ +
                                4 * BN * 4 /*column scales, double-buffered*/;
};

// One 32 x 32 chunk of the tile (rows: this warp's TMEM lane quarter, lane =
// row; 32 columns from col0) written by TMA: the lanes put their rows into
// the warp's staging buffer (128-byte rows, 16-byte pieces swizzled by row so
// the writes avoid bank conflicts; the store's tensor map uses the same 128B
// swizzle), then lane 0 issues the store.  The buffer is reused only after the
// warp's previous store has read it.  Rows past M and columns past N are
// clipped by the TMA unit.
__device__ __forceinline__ void tma_chunk_f32(const CUtensorMap *tm, int x, int y0,
                                              const float (&v)[32], uint8_t *stage, int lane) {
  if (lane == 0) bulk_wait_read_all();
  __syncwarp();
  float4 *row = reinterpret_cast<float4 *>(stage + lane * 128);
#pragma unroll
  for (int q = 0; q < 8; ++q)
    row[q ^ (lane & 7)] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(tm, x, y0, stage);
    bulk_commit();
  }
}
__device__ __forceinline__ void tma_chunk_i8(const CUtensorMap *tm, int x, int y0,
                                             const uint32_t (&codes)[8], uint8_t *stage, int lane) {
  if (lane == 0) bulk_wait_read_all();
  __syncwarp();
  uint4 *row = reinterpret_cast<uint4 *>(stage + lane * 32);  // 32-byte rows, no swizzle
  row[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
  row[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(tm, x, y0, stage);
    bulk_commit();
  }
}

// The epilogue of one 32-column chunk through TMA stores: dequantise (same
// operations and order as gemm_store_chunk), add the residual (plain mode),
// and store the fp32 values -- or, in the in_proj split, the z / xBC-code / dt
// piece the chunk falls in (the split points are multiples of 32).
__device__ __forceinline__ void gemm_tma_chunk(const GemmEpilogue &ep, const CUtensorMap *tm0,
                                               const CUtensorMap *tm1, const CUtensorMap *tm2,
                                               long long row, int row0, float sx, int col0,
                                               uint32_t (&r)[32], const float *colw,
                                               const float *cole, uint8_t *stage, int lane) {
  float(&y)[32] = reinterpret_cast<float(&)[32]>(r);
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    const float4 sw = *reinterpret_cast<const float4 *>(colw + j);
    y[j] = __fmul_rn(__fmul_rn(__int2float_rn((int)r[j]), sx), sw.x);
    y[j + 1] = __fmul_rn(__fmul_rn(__int2float_rn((int)r[j + 1]), sx), sw.y);
    y[j + 2] = __fmul_rn(__fmul_rn(__int2float_rn((int)r[j + 2]), sx), sw.z);
    y[j + 3] = __fmul_rn(__fmul_rn(__int2float_rn((int)r[j + 3]), sx), sw.w);
  }
  if (ep.mode == 0) {
    if (ep.residual && row < ep.M) {
      const float *res = ep.residual + row * ep.N + col0;
      if (col0 + 32 <= ep.N) {
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const float4 rv = *reinterpret_cast<const float4 *>(res + j);
          y[j] = __fadd_rn(rv.x, y[j]);
          y[j + 1] = __fadd_rn(rv.y, y[j + 1]);
          y[j + 2] = __fadd_rn(rv.z, y[j + 2]);
          y[j + 3] = __fadd_rn(rv.w, y[j + 3]);
        }
      } else {
        for (int j = 0; j < 32 && col0 + j < ep.N; ++j) y[j] = __fadd_rn(res[j], y[j]);
      }
    }
    tma_chunk_f32(tm0, col0, row0, y, stage, lane);
    return;
  }
  const int di = ep.di, cc = ep.cc;
  if (col0 < di) {
    tma_chunk_f32(tm0, col0, row0, y, stage, lane);
  } else if (col0 < di + cc) {
    uint32_t packed[8];
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      const float4 es = *reinterpret_cast<const float4 *>(cole + j);
      const float e4[4] = {es.x, es.y, es.z, es.w};
      uint32_t w = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int code = quant127(__fmul_rn(y[j + b], e4[b]));
        w |= ((uint32_t)(code & 0xFF)) << (8 * b);
      }
      packed[j / 4] = w;
    }
    tma_chunk_i8(tm1, col0 - di, row0, packed, stage, lane);
  } else {
    tma_chunk_f32(tm2, col0 - di - cc, row0, y, stage, lane);
  }
}

template <int BN, int STAGES, int EW>
__global__ void __launch_bounds__(64 + 32 * EW, 1)
    k_gemm_i8_persist(const __grid_constant__ CUtensorMap tmA,
                      const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmO0,
                      const __grid_constant__ CUtensorMap tmO1,
                      const __grid_constant__ CUtensorMap tmO2, int num_k_blocks, int m_tiles,
                      int n_tiles, GemmEpilogue ep) {
  static_assert(BN % 32 == 0 && BN >= 64 && BN <= 256, "BN");
  static_assert(EW % 4 == 0 && (BN / (EW / 4)) % 32 == 0, "epilogue split");
  using Sm = PersistSmem<BN, STAGES, EW>;
  constexpr int kEpiThreads = 32 * EW;
  constexpr int kColsPerWarp = BN / (EW / 4);
  constexpr uint32_t kTmemCols = 2 * BN;  // a power of two >= 32 for BN in {64, 128, 256}
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + STAGES * Sm::kA;
  uint8_t *sOut = sB + STAGES * Sm::kB;  // [EW][4096], 1024-aligned
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(sOut + EW * Sm::kStage);
  uint64_t *empty_bar = full_bar + STAGES;
  uint64_t *tfull = empty_bar + STAGES;   // [2]
  uint64_t *tempty = tfull + 2;           // [2]
  uint64_t *drain_bar = tempty + 2;       // [1]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain_bar + 1);
  float *col_w = reinterpret_cast<float *>((reinterpret_cast<uintptr_t>(tmem_slot + 1) + 15) &
                                           ~static_cast<uintptr_t>(15));  // [2][BN]
  float *col_e = col_w + 2 * BN;                                          // [2][BN]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_tiles = m_tiles * n_tiles;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], EW);
    }
    mbar_init(drain_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"((unsigned long long)&tmA) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"((unsigned long long)&tmB) : "memory");
    if (ep.tma_store) {
      asm volatile("prefetch.tensormap [%0];" ::"l"((unsigned long long)&tmO0) : "memory");
      if (ep.mode == 1) {
        asm volatile("prefetch.tensormap [%0];" ::"l"((unsigned long long)&tmO1) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"((unsigned long long)&tmO2) : "memory");
      }
    }
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // As in k_gemm_i8_tc: under programmatic dependent launch the weights of
  // the first tile's first stages are fetched before the dependency wait;
  // the producer lane waits before the activations, the epilogue warps before
  // the row scales and the residual.
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      bool ok = !(g_test_stall & kStallGemm);
      const int pre = ok && (int)blockIdx.x < num_tiles
                          ? (num_k_blocks < STAGES ? num_k_blocks : STAGES) : 0;
      if (pre) {
        const int n0 = ((int)blockIdx.x % n_tiles) * BN;
        for (int kb = 0; kb < pre; ++kb) {  // fresh ring: no empty-slot wait
          mbar_arrive_expect_tx(&full_bar[kb], (uint32_t)(Sm::kA + Sm::kB));
          tma_load_2d(sB + kb * Sm::kB, &tmB, kb * kGemmBK, n0, &full_bar[kb]);
        }
      }
      pdl_wait();
      if (pre) {
        const int m0 = ((int)blockIdx.x / n_tiles) * kGemmBM;
        for (int kb = 0; kb < pre; ++kb)
          tma_load_2d(sA + kb * Sm::kA, &tmA, kb * kGemmBK, m0, &full_bar[kb]);
      }
      long long it = pre;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        const int m0 = (t / n_tiles) * kGemmBM, n0 = (t % n_tiles) * BN;
        for (int kb = t == (int)blockIdx.x ? pre : 0; kb < num_k_blocks; ++kb, ++it) {
          const int s = (int)(it % STAGES);
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait(&empty_bar[s], ph ^ 1u)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full_bar[s], (uint32_t)(Sm::kA + Sm::kB));
          tma_load_2d(sA + s * Sm::kA, &tmA, kb * kGemmBK, m0, &full_bar[s]);
          tma_load_2d(sB + s * Sm::kB, &tmB, kb * kGemmBK, n0, &full_bar[s]);
        }
      }
      // every copy issued must have landed before the CTA may exit (on the
      // normal path the MMA lane has consumed them all and these return at once)
      const long long first = it > STAGES ? it - STAGES : 0;
      for (long long j = first; j < it; ++j)
        if (!mbar_drain(&full_bar[j % STAGES], (uint32_t)(j / STAGES) & 1u)) break;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = i8_idesc(kGemmBM, BN);
      long long it = 0;
      int tl = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++tl) {
        const int acc = tl & 1;
        const uint32_t use = (uint32_t)(tl >> 1);
        if (!mbar_wait(&tempty[acc], (use & 1u) ^ 1u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < num_k_blocks; ++kb, ++it) {
          const int s = (int)(it % STAGES);
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait(&full_bar[s], ph)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sw128_desc(smem_u32(sA + s * Sm::kA));
          const uint64_t bd = sw128_desc(smem_u32(sB + s * Sm::kB));
#pragma unroll
          for (int k = 0; k < kGemmBK / 32; ++k)
            mma_i8(d, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), idesc,
                   (kb > 0 || k > 0) ? 1u : 0u);
          mma_commit(&empty_bar[s]);
        }
        if (ok) mma_commit(&tfull[acc]);
      }
      // wait for every MMA issued so far before TMEM can be released
      mma_commit(drain_bar);
      mbar_drain(drain_bar, 0);
    }
  } else {
    pdl_wait();
    const int e = warp - 2;                 // 0 .. EW-1
    const int quarter = warp & 3;           // TMEM lanes [32 quarter, 32 quarter + 32)
    const int part = e / 4;                 // which column slice of the tile
    const int et = threadIdx.x - 64;        // 0 .. kEpiThreads-1
    static_assert(BN <= kEpiThreads, "one staged column per epilogue thread");
    // the scales of a tile (column s_w and PoT factor, row s_x) are loaded one
    // tile ahead into registers, so no global latency sits between tiles
    auto load_scales = [&](int t, float &w, float &ev, float &sxv) {
      const int m0 = (t / n_tiles) * kGemmBM, n0 = (t % n_tiles) * BN;
      const long long c = (long long)n0 + et;
      w = (et < BN && c < ep.N) ? ep.s_w[c] : 0.0f;
      ev = 0.0f;
      if (et < BN && ep.mode == 1 && c >= ep.di && c < (long long)ep.di + ep.cc)
        ev = pow2f(-ep.e_u[c - ep.di]);
      const long long row = (long long)m0 + quarter * 32 + lane;
      sxv = row < ep.M ? ep.s_x[row] : 0.0f;
    };
    float nw = 0.0f, ne = 0.0f, nsx = 0.0f;
    if ((int)blockIdx.x < num_tiles) load_scales(blockIdx.x, nw, ne, nsx);
    int tl = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++tl) {
      const int acc = tl & 1;
      const uint32_t use = (uint32_t)(tl >> 1);
      const int m0 = (t / n_tiles) * kGemmBM, n0 = (t % n_tiles) * BN;
      float *cw = col_w + acc * BN, *ce = col_e + acc * BN;
      // stage this tile's column scales (buffer acc was last read two tiles
      // ago, before every epilogue warp passed the previous tile's barrier)
      if (et < BN) {
        cw[et] = nw;
        ce[et] = ne;
      }
      const float sx = nsx;
      if (t + (int)gridDim.x < num_tiles) load_scales(t + gridDim.x, nw, ne, nsx);
      const long long row = (long long)m0 + quarter * 32 + lane;
      asm volatile("bar.sync 1, %0;" ::"r"(kEpiThreads) : "memory");
      if (ok) ok = mbar_wait(&tfull[acc], use & 1u);
      ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
      tc_fence_after();
      const int c_begin = part * kColsPerWarp;
#pragma unroll 1
      for (int c = c_begin; c < c_begin + kColsPerWarp; c += 32) {
        uint32_t r[32];
        if (ok) {
          tmem_ld32(tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN + c), r);
          if (c + 32 >= c_begin + kColsPerWarp) {  // last load of this warp: hand the buffer back
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
          }
          if (n0 + c < ep.N) {
            if (ep.tma_store)
              gemm_tma_chunk(ep, &tmO0, &tmO1, &tmO2, row, m0 + quarter * 32, sx, n0 + c, r,
                             cw + c, ce + c, sOut + e * Sm::kStage, lane);
            else
              gemm_store_chunk(ep, row, sx, (long long)n0 + c, r, cw + c, ce + c);
          }
        }
      }
    }
    if (ep.tma_store && lane == 0) bulk_wait_all();  // stores done before the CTA exits
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kTmemCols)
                 : "memory");
  }
}

}  // namespace fm
