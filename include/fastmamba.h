/*
 * fastmamba.h -- C ABI of the quantised Mamba2 mixer library (libfastmamba.so).
 *
 * The method is FastMamba's quantisation scheme for a Mamba2 mixer layer
 * (arXiv 2505.18975; cited below by web page and section):
 *   - Hadamard-rotated 8-bit linear layers, Y = (XH)(H^T W^T) with H
 *     orthonormal after 1/sqrt(n) (pith.science review, "What carries the
 *     argument"; scales from the max of the rotated tensors: Referee Report,
 *     major comment 1, on Algorithm 1 and Fig. 6);
 *   - power-of-two (2^p, shift-only) fixed point for the causal conv1d and
 *     the SSM recurrence (same section; original abstract);
 *   - an 8-segment first-order linear approximation of 2^v, with
 *     e^x = 2^(x log2 e) and SoftPlus(x) = x + SoftPlus(-x) (same section;
 *     Referee minor comment 5 on Eq. (5): SoftPlus(x) ~ e^x for x <= 0).
 * The Mamba2 block structure (in_proj -> conv1d + SiLU -> selective scan ->
 * gate + RMSNorm -> out_proj; Figure 2 caption) is that of Mamba2, the
 * paper's reference [2].
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the
 *     library never allocates, frees or retains them.  Tensors are dense,
 *     row-major (last index fastest).  Pointers must be 16-byte aligned.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream).  Host-side validation happens before any
 *     launch; on error nothing is launched and a status is returned.
 *   - Kernels that wait (the GEMM's and the sequential scan's pipeline
 *     barriers) give up after a bounded time and set a device error word
 *     instead of hanging; fm_sync_status() reports it (FM_ERR_TIMEOUT), and
 *     the outputs of that call are then undefined.
 *   - Shapes: K of every linear layer and d_model, d_inner are multiples of
 *     256 (the Hadamard block); headdim = 64, d_state = 128, ngroups = 1,
 *     d_conv = 4 (the Mamba2-130M / 2.7B configuration); conv_ch and
 *     d_inner are multiples of 16.
 *   - Fixed-point conventions (rshr, satb, Q.16, exponent table) are
 *     described next to fm_exp_layout below.
 *   - No exceptions cross the ABI; no global mutable state except a
 *     per-device device error word, the per-process entry-point cache and
 *     the streams and events fm_stack_prefill keeps per CUDA context.
 */
#ifndef FASTMAMBA_H
#define FASTMAMBA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fm_status {
    FM_OK = 0,
    FM_ERR_INVALID_ARG = 1, /* null pointer, bad enum value */
    FM_ERR_SHAPE = 2,       /* unsupported or inconsistent sizes */
    FM_ERR_ALIGNMENT = 3,   /* pointer not 16-byte aligned */
    FM_ERR_WORKSPACE = 4,   /* workspace missing or too small */
    FM_ERR_NONFINITE = 5,   /* a NaN or Inf reached an int8 activation quantiser */
    FM_ERR_TIMEOUT = 6,     /* a bounded device-side wait gave up */
    FM_ERR_CUDA = 7,        /* a CUDA runtime/driver call failed */
    FM_ERR_UNSUPPORTED = 8  /* no sm_100 device, or driver entry point missing */
} fm_status;

enum { FM_DYNAMIC = 0, FM_STATIC = 1 };

typedef void *fm_stream; /* cudaStream_t */

/* Human-readable name of a status code (static string). */
const char *fm_status_string(fm_status s);
/* Detail of the last failed call on this host thread (static, thread-local). */
const char *fm_last_error(void);
/* Synchronises `stream`, then reads and clears the device error word of the
 * current device: FM_OK, FM_ERR_TIMEOUT (a bounded wait gave up; it takes
 * precedence; the outputs and the carried states -- ssm_state, conv_state --
 * of the calls since the last read are then undefined), FM_ERR_NONFINITE (an activation row entering an int8
 * quantiser -- fm_hadamard_quant, fm_gate_norm_quant and the layers that
 * call them -- held a NaN or Inf; that row's codes and scale are then
 * undefined) or FM_ERR_CUDA (the synchronisation itself failed).  The word
 * accumulates over every call on the device since it was last read. */
fm_status fm_sync_status(fm_stream stream);
/* Failure injection for tests of the bounded-wait path (the pages have no
 * counterpart).  On the current device, for every later launch until reset:
 *   stall_mask bit 0: the GEMM producers issue no loads; bit 1: the
 *   sequential scan's producer issues no copies.  The consumers then wait on
 *   a barrier that nothing completes, with no copy or MMA in flight, give up
 *   after wait_limit_ns, set the device error word (FM_ERR_TIMEOUT at the
 *   next fm_sync_status) and end; every kernel still frees its TMEM.
 *   wait_limit_ns: the pipeline waits' limit; 0 = the default (4 s).  Waits
 *   for work already issued (drains) always use the default.
 * fm_set_fault_injection(0, 0) restores normal operation.  Synchronous
 * (cudaMemcpyToSymbol); not for use while the device runs library kernels. */
fm_status fm_set_fault_injection(int stall_mask, uint64_t wait_limit_ns);
/* Tuning, process-wide (the pages have no counterpart): 1 (default) launches
 * the hot kernels with programmatic stream serialisation, so that each may be
 * scheduled while its predecessor in the stream drains.  Every such kernel
 * waits for its predecessor before it reads that kernel's outputs; before the
 * wait the GEMMs fetch their first weight stages and the single decode step
 * its state (the kernels that write a state end before any successor starts).
 * The sequential scan and the gate after it are always launched plainly (the
 * scan's CTA placement matters), and so is the first kernel after one of
 * fm_stack_prefill's waits on another stream.  0 launches every kernel
 * plainly.  Results
 * are the same bits either way.  FM_ERR_INVALID_ARG for other values. */
fm_status fm_set_pdl(int enable);
/* Library ABI version (major * 100 + minor). */
int fm_version(void);

/* ------------------------------------------------------------------ */
/* shapes and the exponent table                                       */
/* ------------------------------------------------------------------ */
typedef struct fm_shape {
    int d_model, d_inner, headdim, d_state, ngroups, d_conv;
} fm_shape;

/* Derived sizes: nheads = d_inner / headdim; conv_ch = d_inner + 2 d_state;
 * n_in = 2 d_inner + 2 d_state + nheads (in_proj columns z | x | B | C | dt). */

/* Power-of-two exponent table of one layer: one device int32 array.  A value
 * e means "the integer code times 2^e".  Layout (offsets in int32 elements):
 *   [0, cc)            e_u  conv input, per conv channel
 *   [cc, 2cc)          e_w  conv weights, per conv channel
 *   [2cc, 3cc)         e_o  conv output, per conv channel (x: its head's e_x; B: e_B; C: e_C)
 *   [3cc, 3cc+nh)      e_x  per head
 *   3cc+nh             e_B
 *   3cc+nh+1           e_C
 *   [3cc+nh+2, +nh)    e_h  state, per head
 *   [3cc+2nh+2, +nh)   e_y  scan output, per head
 *   [3cc+3nh+2, +nh)   e_D  skip parameter D, per head
 *   3cc+4nh+2          e_g  gate output
 * Size: 3cc + 4nh + 3. */
typedef struct fm_exp_layout {
    int e_u, e_w, e_o, e_x, e_B, e_C, e_h, e_y, e_D, e_g, size;
} fm_exp_layout;
fm_exp_layout fm_exp_table_layout(const fm_shape *shape);

/* ------------------------------------------------------------------ */
/* a0 + a1 / a10: (pre-RMSNorm) + Hadamard rotation + int8 quantisation */
/* ------------------------------------------------------------------ */
/* Source: Y = (XH)(H^T W^T) with H orthonormal after 1/sqrt(n) (pith.science review of FastMamba,
 * "What carries the argument"); the scale from the max of the rotated tensor
 * (Referee Report, major comment 1, on Algorithm 1 and Fig. 6); the stack's
 * pre-RMSNorm is Mamba2's (the paper's reference [10], Figure 2 caption).
 * x [M, K] fp32 -> q [M, K] int8 codes and s_x [M] fp32 scales, so that
 * dequant = q * s_x[row] approximates (RMSNorm(x) * prenorm_w) H_bd.
 *   prenorm_w  [K] or NULL: apply RMSNorm (eps 1e-5, fixed summation order)
 *              and this weight before rotating (stack layers).
 *   rotate     1: block-diagonal Sylvester Hadamard (block 256) / 16; 0: identity.
 *   mode       FM_DYNAMIC: per-row amax; FM_STATIC: *static_amax (device
 *              scalar) for every row, values beyond it clip to +-127.
 *   amax_row   [M] or NULL: receives each row's max |rotated value|.
 * K % 256 == 0, K <= 8192. */
fm_status fm_hadamard_quant(const float *x, int64_t M, int64_t K, const float *prenorm_w,
                            int rotate, int mode, const float *static_amax, int8_t *q,
                            float *s_x, float *amax_row, fm_stream stream);

/* Source: the pre-rotated weight H^T W^T of "What carries the argument" (pith.science review of FastMamba).
 * Offline: W [N, K] fp32 -> Wq [N, K] int8 and s_w [N] fp32 with
 * W' = W H_bd (fp64), s_w = max|W'[n,:]| / 127, Wq = rint(W' / s_w). */
fm_status fm_prepare_linear(const float *W, int64_t N, int64_t K, int rotate, int8_t *Wq,
                            float *s_w, fm_stream stream);

/* ------------------------------------------------------------------ */
/* a2 + a3 / a11: W8A8 GEMM on the tensor cores + dequantisation        */
/* ------------------------------------------------------------------ */
/* Source: the 8-bit linear layers, (XH)(H^T W^T) computed as an int8 product
 * and dequantised (pith.science review of FastMamba, "What carries the argument"; Referee
 * major comment 1 on Algorithm 1).
 * Y[m,n] = fl(fl(float(acc[m,n]) * s_x[m]) * s_w[n]) (+ residual[m,n]),
 * acc = sum_k A[m,k] Wq[n,k] (exact int32).
 *   A [M, K] int8, Wq [N, K] int8 (both K-major), residual [M, N] or NULL
 *   (may alias Y), acc_out [M, N] int32 or NULL (raw accumulators).
 * K % 128 == 0. */
fm_status fm_w8a8_gemm(const int8_t *A, const float *s_x, int64_t M, const int8_t *Wq,
                       const float *s_w, int64_t N, int64_t K, const float *residual, float *Y,
                       int32_t *acc_out, fm_stream stream);

/* Source: as fm_w8a8_gemm; the column split z | x | B | C | dt is Mamba2's
 * in_proj (the paper's reference [2]; Figure 2 caption), the xBC columns
 * quantised to the conv's power-of-two codes ("What carries the argument").
 * in_proj: the same GEMM (N = n_in, K = d_model) with the split epilogue:
 *   z   [M, d_inner] fp32   (columns [0, di))
 *   xbc [M, conv_ch] int8   (columns [di, di+cc)): satb(rint(y * 2^-e_u[c]), 8)
 *   dt  [M, nheads] fp32    (columns [di+cc, n_in))
 * e_u is the exponent table's first region (device). */
fm_status fm_in_proj(const int8_t *A, const float *s_x, int64_t M, const int8_t *Wq,
                     const float *s_w, const fm_shape *shape, const int32_t *exps, float *z,
                     int8_t *xbc, float *dt, fm_stream stream);

/* Tuning: the tile width (output columns per CTA tile) of the persistent GEMM
 * kernel for every later call in this process: 0 (default) chooses by the
 * grid, 128 or 256 forces it where the persistent kernel runs.  All widths
 * compute the same bits.  FM_ERR_INVALID_ARG for other values. */
fm_status fm_set_gemm_tile(int bn);

/* Workspace variants: the same results, bit for bit.  Given a device
 * workspace of fm_gemm_workspace_bytes(M, N, K) bytes (0 when the problem
 * would not split), a grid with fewer output tiles than the GPU has SMs
 * splits K across CTAs: each slice adds its exact int32 partial sums into the
 * workspace, and one epilogue pass dequantises the totals.  The layer entry
 * points (fm_mixer_prefill, fm_decode_step) do this from their own workspace.
 * ws may be NULL (no split) when fm_gemm_workspace_bytes returns 0. */
size_t fm_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);
/* Process-wide switch of the split-K path above: 0 (default) never splits
 * (fm_gemm_workspace_bytes then returns 0 and the layer workspaces hold no
 * partial sums), 1 splits small grids.  Set it before sizing workspaces and
 * keep it while they are in use.  FM_ERR_INVALID_ARG for other values. */
fm_status fm_set_gemm_splitk(int enable);
/* Process-wide: 1 runs a decode-size GEMM (M <= 64) whose 32-wide output
 * tiles are fewer than the SMs with K split over the 2..8 CTAs of a
 * thread-block cluster -- each CTA accumulates its slice's exact int32 partial
 * sums, rank 0 adds the others' through distributed shared memory and runs
 * the same epilogue, so the outputs are bit-identical; no workspace.  0
 * (default; measured faster) runs one CTA per tile.  Not used while
 * fm_set_gemm_splitk(1) splits through a workspace.  FM_ERR_INVALID_ARG for
 * other values.
 * Source: the W8A8 linear of the pith.science review of FastMamba, "What
 * carries the argument" (the split only changes the int32 summation order). */
fm_status fm_set_gemm_cluster(int enable);
fm_status fm_w8a8_gemm_ws(const int8_t *A, const float *s_x, int64_t M, const int8_t *Wq,
                          const float *s_w, int64_t N, int64_t K, const float *residual,
                          float *Y, int32_t *acc_out, void *ws, size_t ws_bytes,
                          fm_stream stream);
fm_status fm_in_proj_ws(const int8_t *A, const float *s_x, int64_t M, const int8_t *Wq,
                        const float *s_w, const fm_shape *shape, const int32_t *exps, float *z,
                        int8_t *xbc, float *dt, void *ws, size_t ws_bytes, fm_stream stream);

/* ------------------------------------------------------------------ */
/* a4: power-of-two causal depthwise conv1d (kernel 4) + SiLU           */
/* ------------------------------------------------------------------ */
/* Source: fine-grained power-of-two quantisation of the convolution (pith.science review of FastMamba,
 * "What carries the argument"; original abstract); SiLU through the shared
 * 2^v unit (Figure 7 caption: the nonlinear approximation unit).
 * u [B, T, cc] int8 codes at e_u -> out [B, T, cc] int8 codes at e_o:
 *   acc = bq[c] + sum_{k=0..3} wq[c,k] u[t-3+k, c]   (tap 3 = current token)
 *   x16 = satb(rshr(acc, -(e_w+e_u+16)), 32); s = SiLU_pwl(x16)
 *   out = satb(rshr(s, e_o + 16), 8)
 *   wq [cc, 4] int8, bq [cc] int32 (at e_w + e_u), exps = exponent table.
 *   conv_state [B, 3, cc] int8 or NULL: history (oldest first) read before
 *   the first token and replaced by the last three inputs. */
fm_status fm_conv1d_pot(const int8_t *u, int B, int T, const fm_shape *shape, const int8_t *wq,
                        const int32_t *bq, const int32_t *exps, int8_t *conv_state, int8_t *out,
                        fm_stream stream);

/* The same conv with per-token output exponents (see fm_set_xbc_exponents):
 * e_tok [B*T, nheads + 2] int32 receives each token's exponents of its heads'
 * x channels, of B and of C; the codes in `out` are at those exponents.
 * Independent of the process-wide setting. */
fm_status fm_conv1d_pot_tok(const int8_t *u, int B, int T, const fm_shape *shape,
                            const int8_t *wq, const int32_t *bq, const int32_t *exps,
                            int8_t *conv_state, int8_t *out, int32_t *e_tok, fm_stream stream);

/* ------------------------------------------------------------------ */
/* a5 - a8: selective scan in power-of-two fixed point                  */
/* ------------------------------------------------------------------ */
/* Tuning: selects the tile of the sequential scan kernel used by every later
 * call in this process -- npt state columns per thread, pc channels per CTA,
 * tch time steps per staged chunk.  Compiled variants: (4,0,32) (default:
 * pc chosen by the grid -- 8 where there are at least three 8-channel CTAs
 * per SM, else 4, with 16-step chunks for the runs of a pipelined
 * fm_stack_prefill), (4,4,32), (4,8,32), (4,4,16), (4,2,16), (4,8,16),
 * (8,4,16), (8,2,16), (8,8,16);
 * anything else returns FM_ERR_INVALID_ARG.  All variants compute the same
 * bits. */
fm_status fm_set_scan_tile(int npt, int pc, int tch);

/* Workspace bytes fm_ssm_scan_pot needs for B*T tokens (per-token dt/dA, the
 * dt*x factor and the skip term, B and C widened). */
size_t fm_scan_workspace_bytes(const fm_shape *shape, int B, int T);

/* Source: power-of-two fixed point for the SSM block and the 8-segment
 * first-order 2^v with e^x = 2^(x log2 e) and SoftPlus(x) = x + SoftPlus(-x)
 * (pith.science review of FastMamba, "What carries the argument"; Referee minor comment 5 on
 * Eq. (5)); the recurrence and C.h + D.x are Mamba2's SSM (Figure 2 and
 * Figure 7 captions; the paper's reference [2]).
 * xbc [B, T, cc] int8 conv output (x | B | C), dt_raw [B, T, nh] fp32.
 * Per token and head (Q.16): dt_q = SoftPlus_pwl(to_q16(dt_raw + dt_bias)),
 * dA_q = 2^(-rshr(dt_q * A_q, 12)).  Per (b, h, p, n), t in order:
 *   u = satb(rshr(dt_q x[p], e_h - e_B - e_x + 16), 24)
 *   h = clamp(rshr(dA_q h, 16) + u B[n], +-(2^30 - 1))
 *   y[p] = satb(rshr(sum_n C[n] h, e_y - e_C - e_h) + rshr(D_q x[p], e_y - e_D - e_x), 32)
 *   dt_bias [nh] fp32, A_q [nh] int32 (exp(A_log) log2(e) 2^12), D_q [nh] int32.
 *   state [B, nh, hd, ds] int32 or NULL (zeros): initial state in, final out;
 *   values must lie within +-(2^30 - 1), the range the recurrence produces.
 *   y [B, T, d_inner] int32 at e_y.
 *   ws: device workspace of at least fm_scan_workspace_bytes(shape, B, T). */
fm_status fm_ssm_scan_pot(const int8_t *xbc, const float *dt_raw, int B, int T,
                          const fm_shape *shape, const float *dt_bias, const int32_t *A_q,
                          const int32_t *D_q, const int32_t *exps, int32_t *state, int32_t *y,
                          void *ws, size_t ws_bytes, fm_stream stream);
/* The same scan on codes at per-token exponents (e_tok from fm_conv1d_pot_tok):
 * per token, s_h = e_h - e_B,t - e_x,t + 16, the output shift
 * e_y - e_C,t - e_h and the skip shift e_y - e_D - e_x,t.  Its workspace,
 * fm_scan_workspace_bytes_tok, also holds the per-token shifts. */
size_t fm_scan_workspace_bytes_tok(const fm_shape *shape, int B, int T);
fm_status fm_ssm_scan_pot_tok(const int8_t *xbc, const float *dt_raw, int B, int T,
                              const fm_shape *shape, const float *dt_bias, const int32_t *A_q,
                              const int32_t *D_q, const int32_t *exps, const int32_t *e_tok,
                              int32_t *state, int32_t *y, void *ws, size_t ws_bytes,
                              fm_stream stream);

/* ------------------------------------------------------------------ */
/* a9 + a10: gate, gated RMSNorm, rotation, int8 quantisation           */
/* ------------------------------------------------------------------ */
/* Source: Mamba2's gate and gated RMSNorm before out_proj (Figure 2 caption;
 * the paper's references [2], [10], [11]) with the SiLU through the 2^v unit,
 * then the out_proj input's rotation and int8 codes as fm_hadamard_quant.
 * y [M, di] int32 (at e_y per head), z [M, di] fp32 -> q [M, di] int8, s_x [M]:
 *   g = y SiLU_pwl(to_q16(z)); g_q = satb(rshr(g, e_g - e_y + 16), 16)
 *   rstd = 1/sqrt(sum g_q^2 2^(2 e_g) / di + 1e-5) (exact integer sum)
 *   o = g_q 2^e_g rstd norm_w, then as fm_hadamard_quant. */
fm_status fm_gate_norm_quant(const int32_t *y, const float *z, int64_t M, const fm_shape *shape,
                             const int32_t *exps, const float *norm_w, int rotate, int mode,
                             const float *static_amax, int8_t *q, float *s_x, float *amax_row,
                             fm_stream stream);

/* ------------------------------------------------------------------ */
/* the nonlinear approximation unit, element-wise (verification)        */
/* ------------------------------------------------------------------ */
/* The shared 8-segment first-order approximation of 2^v and the functions
 * built on it (pith.science review of FastMamba, "What carries the
 * argument"; Referee minor comment 5, Eq. (5)), evaluated element-wise over
 * a device int64 array -- the same device functions the conv, scan and gate
 * kernels use (SiLU in the form the conv and gate kernels evaluate: table in
 * shared memory, reciprocal-estimate division).  kind: 0 = 2^v (Q.16 in,
 * v <= 0), 1 = e^x, 2 = SoftPlus,
 * 3 = SiLU (in clamped to int32), 4 = to_q16 of the fp32 bit pattern held
 * in the low 32 bits.  in, out: [n] int64. */
fm_status fm_eval_pwl(int kind, const int64_t *in, int64_t n, int64_t *out, fm_stream stream);

/* ------------------------------------------------------------------ */
/* layers                                                               */
/* ------------------------------------------------------------------ */
/* A prepared layer: device pointers to quantised parameters (caller-owned). */
typedef struct fm_layer {
    fm_shape shape;
    int rotate;                 /* 1: Hadamard rotation in both linear layers */
    int mode;                   /* FM_DYNAMIC or FM_STATIC activation scales */
    const int8_t *w_in_q;       /* [n_in, d_model] */
    const float *w_in_s;        /* [n_in] */
    const int8_t *w_out_q;      /* [d_model, d_inner] */
    const float *w_out_s;       /* [d_model] */
    const float *prenorm_w;     /* [d_model] or NULL: stack layer pre-RMSNorm */
    const int8_t *conv_wq;      /* [conv_ch, 4] */
    const int32_t *conv_bq;     /* [conv_ch] */
    const float *dt_bias;       /* [nheads] */
    const int32_t *A_q;         /* [nheads] */
    const int32_t *D_q;         /* [nheads] */
    const float *norm_w;        /* [d_inner] gated-norm weight */
    const int32_t *exps;        /* exponent table (fm_exp_table_layout) */
    const float *static_amax;   /* [2]: in_proj input, out_proj input (FM_STATIC) */
} fm_layer;

/* Chunked (state-space-dual) scan mode: the same inputs and outputs as
 * fm_ssm_scan_pot, computed chunk by chunk (128 tokens) on the tensor cores as
 * in Mamba2's own algorithm (reference [2] of the FastMamba paper): exact
 * int8 C.B^T, bf16 operands elsewhere, fp32 sums, decays 2^(running sum of the
 * step's log2 decay) per chunk.  Not bit-identical to the sequential scan; its
 * error budget is that of bf16 operands (relative 2^-9 per rounded operand).
 * state (nullable): int32 at e_h in and out, interchangeable with the
 * sequential scan's.  ws: device workspace of fm_ssd_workspace_bytes. */
size_t fm_ssd_workspace_bytes(const fm_shape *shape, int B, int T);
/* Process-wide scan mode of the layer entry points (fm_mixer_prefill and
 * what calls it): 0 = the sequential fixed-point scan (default, the method),
 * 1 = the chunked mode above for calls of more than one token.  The mode in
 * force when fm_workspace_bytes is asked must also be in force for the call.
 * FM_ERR_INVALID_ARG for any other value. */
fm_status fm_set_scan_mode(int mode);
fm_status fm_ssd_scan(const int8_t *xbc, const float *dt_raw, int B, int T,
                      const fm_shape *shape, const float *dt_bias, const int32_t *A_q,
                      const int32_t *D_q, const int32_t *exps, int32_t *state, int32_t *y,
                      void *ws, size_t ws_bytes, fm_stream stream);
/* Source: the pages give the SSM block "fine-grained" power-of-two scales but
 * neither the state's word width nor the granularity (pith.science review of
 * FastMamba, "What carries the argument"); this selects between two readings.
 * Process-wide state spec of every scan entry point and of the calibration:
 * (31, 0), the default, is the method as built -- an int32 state clamped at
 * +-(2^30 - 1), the increment u B with u rounded first.  (16, 7) is the narrow
 * reading: the state clamps at +-32767 and is stored as int16 -- every
 * int32_t *state / ssm_state argument then points at an int16 [B, nh, hd, ds]
 * buffer -- and the increment is rshr(ug B, 7) with
 * ug = satb(rshr(dt_q x, s_h - 7), 24); the calibration leaves 2^14 of
 * headroom.  Switch it before calibrating and allocating states, and keep it
 * for the layer's life.  Anything else: FM_ERR_INVALID_ARG. */
fm_status fm_set_state_spec(int bits, int guard);
/* Source: as fm_set_state_spec (the granularity of the "fine-grained"
 * power-of-two scales is left open by the pages).
 * Process-wide granularity of the conv output's exponents in the layer entry
 * points (fm_mixer_prefill, fm_decode_step, fm_calibrate_layer): 0 (default)
 * the static exponents as built (e_x per head, e_B, e_C); 1 per token -- each
 * token's codes of a head's x channels, of B and of C are
 * satb(rshr(s, e + 16), 8) with e = max(E(max |s|, 127) - 16, static - 16),
 * s the Q.16 SiLU values, and the scan shifts u, its output and the skip
 * term by the token's exponents (state and output exponents stay static).
 * The layer workspace then holds the exponents ([B*T, nh + 2] int32) and the
 * scan's per-token shifts.  Set it before calibrating and sizing workspaces;
 * the chunked scan mode refuses it.  The standalone fm_conv1d_pot and
 * fm_ssm_scan_pot stay static.  FM_ERR_INVALID_ARG for other values. */
fm_status fm_set_xbc_exponents(int per_token);

/* Workspace bytes fm_mixer_prefill / fm_decode_step need for B*T tokens. */
size_t fm_workspace_bytes(const fm_shape *shape, int B, int T);

/* Source: the Mamba2 block of Figure 2's caption (in_proj -> conv1d + SiLU
 * -> SSM -> gate + RMSNorm -> out_proj) under the three pieces of "What
 * carries the argument" (pith.science review of FastMamba); a0-a11 in order.
 * One mixer layer on x [B, T, d_model] fp32 -> out [B, T, d_model] fp32.
 *   residual 1: out = x + mixer(x) (stack layer; out may alias x).
 *   conv_state [B, 3, conv_ch] int8 / ssm_state [B, nh, hd, ds] int32, or
 *   NULL: carried state in/out (prefill in chunks is bit-identical to one pass).
 *   ws: device workspace of at least fm_workspace_bytes(shape, B, T).
 *   Launch limits, checked before any kernel: B <= 65535 and
 *   B * T <= 65535 * 128 rows, else FM_ERR_SHAPE (fm_calibrate_layer too). */
fm_status fm_mixer_prefill(const fm_layer *L, const float *x, int B, int T, int residual,
                           int8_t *conv_state, int32_t *ssm_state, float *out, void *ws,
                           size_t ws_bytes, fm_stream stream);

/* Source: as fm_mixer_prefill, for the pre-normed residual stack the
 * review's workloads run (pith.science review of FastMamba, the 130M and
 * 2.7B models of Table III); the recurrence's state carries only forward in
 * time (Mamba2's recurrent form, the paper's reference [2]), which is what
 * makes the time-pipelined schedule below exact.
 * A stack of residual layers over one batch, in place on x [B, T, d_model]:
 * for l = 0 .. n_layers-1, x <- x + mixer_l(x), bit for bit the loop of
 * fm_mixer_prefill(layers[l], residual = 1, out = x) over the layers (with
 * the sequential scan a prefill split with carried states gives the one-pass
 * bits; in the chunked scan mode, whose state crosses a call boundary as
 * int32, the pipelined result is that loop applied run after run with
 * carried states).  All layers share d_model and d_inner (FM_ERR_SHAPE
 * otherwise).
 *   conv_states / ssm_states: NULL (every layer starts from zero states,
 *   none written back) or arrays of n_layers per-layer state buffers as
 *   fm_mixer_prefill takes them (read, then updated).
 *   n_chunks 1: the plain layer loop on `stream`.  n_chunks in [2, 64]: each
 *   sequence's tokens are cut into runs of ceil(T / n_chunks) tokens
 *   (rounded up to a multiple of 32), and every run walks the layers on one
 *   of up to 8 streams the library keeps per CUDA context, forked from and
 *   joined back to `stream` (work queued on `stream` before the call runs
 *   first; work queued after it waits for all of it).  Run k of a layer
 *   waits only for run k-1's conv and scan of that layer (the states it
 *   starts from), so successive runs' scans overlap each other and the other
 *   stages; runs of different sequences do not wait for each other.  The
 *   first pipelined call in a context creates the streams and events (make
 *   it outside stream capture); concurrent calls from several host threads
 *   are serialised on the host while they queue their work.
 *   ws: device workspace of fm_stack_workspace_bytes(shape, n_layers, B, T,
 *   n_chunks) bytes, 16-byte aligned (FM_ERR_WORKSPACE / FM_ERR_ALIGNMENT).
 *   With the scan tile left to the grid (fm_set_scan_tile's default), runs
 *   whose scan grid is too small for 8 channels per CTA stage 16-step chunks
 *   (half the shared memory), so that more of the neighbouring runs' kernels
 *   fit beside them; the bits are the same either way.
 *   Launch limits as fm_mixer_prefill; n_chunks outside [1, 64] or
 *   n_layers < 0: FM_ERR_INVALID_ARG. */
fm_status fm_stack_prefill(const fm_layer *const *layers, int n_layers, float *x, int B, int T,
                           int8_t *const *conv_states, int32_t *const *ssm_states, int n_chunks,
                           void *ws, size_t ws_bytes, fm_stream stream);
/* fm_stack_prefill with the batch in host memory: x_host [B, T, d_model] is
 * copied to the device rows x_dev (caller-owned, [B, T, d_model], 16-byte
 * aligned), the stack runs there, and the result is copied to out_host (may
 * equal x_host).  Pipelined, each run's input is copied on the run's stream
 * before its first layer and its output right after its last, so the copies
 * of one run overlap the other runs' kernels; with n_chunks 1 the two copies
 * bracket the layer loop on `stream`.  The call only queues the copies
 * (cudaMemcpyAsync): they overlap only if the host buffers are pinned, and
 * out_host holds the result once `stream` has been synchronised.  x_host and
 * out_host are required when B * T > 0 (FM_ERR_INVALID_ARG); n_layers 0 does
 * nothing.  Everything else as fm_stack_prefill, with the same workspace. */
fm_status fm_stack_prefill_host(const fm_layer *const *layers, int n_layers, const float *x_host,
                                float *out_host, float *x_dev, int B, int T,
                                int8_t *const *conv_states, int32_t *const *ssm_states,
                                int n_chunks, void *ws, size_t ws_bytes, fm_stream stream);
/* Workspace bytes of fm_stack_prefill (0 for an invalid shape or argument):
 * n_chunks 1 needs fm_workspace_bytes(shape, B, T); pipelined, one run's
 * workspace per internal stream plus zero-started states for every layer. */
size_t fm_stack_workspace_bytes(const fm_shape *shape, int n_layers, int B, int T, int n_chunks);

/* Source: the 2.7B decode figures of the review's Table III discussion
 * (pith.science review of FastMamba, "What carries the argument"); Mamba2's recurrent form
 * (the paper's reference [2]): a prefill of one token with states carried.
 * Single-token decode step for B sequences: x [B, d_model] -> out [B, d_model],
 * updating conv_state and ssm_state (both required). */
fm_status fm_decode_step(const fm_layer *L, const float *x, int B, int residual,
                         int8_t *conv_state, int32_t *ssm_state, float *out, void *ws,
                         size_t ws_bytes, fm_stream stream);

/* Decode step that allocates nothing and takes no workspace.
 *
 * The paper has no counterpart to this entry point: it exists for callers
 * that cannot call cudaMalloc -- for example a plugin running inside a host
 * framework that owns all device memory, or a serving loop whose memory
 * budget is fixed at start-up and must never reach the allocator.  Its
 * scratch (the intermediates fm_decode_step keeps in `ws`) lives in a
 * file-scope device array of FM_NOALLOC_SCRATCH_BYTES that every GPU which
 * loads the library holds until the process exits.
 *   - Same arguments and results as fm_decode_step, minus ws/ws_bytes.
 *   - Batches whose workspace (fm_workspace_bytes(shape, B, 1)) exceeds
 *     FM_NOALLOC_SCRATCH_BYTES are rejected with FM_ERR_WORKSPACE before
 *     any launch.
 *   - The first call in a CUDA context looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it under
 *     the context's unique id; make that first call before any stream
 *     capture.  After cudaDeviceReset the next call runs in a new context,
 *     so it looks the address up again (and is again a first call).
 *   - Every call on a device shares the one array and leaves the last
 *     call's intermediates in it.  What must start at zero (the split-K
 *     partial sums of a small-batch GEMM) is cleared by the call itself on
 *     its stream; everything else is written before it is read.  Calls that
 *     overlap on the GPU (different streams, or different host threads)
 *     race on the array: serialise them. */
#define FM_NOALLOC_SCRATCH_BYTES (16u << 20)
fm_status fm_decode_step_noalloc(const fm_layer *L, const float *x, int B, int residual,
                                 int8_t *conv_state, int32_t *ssm_state, float *out,
                                 fm_stream stream);

/* ------------------------------------------------------------------ */
/* FastMamba-LQ: W8A8 linears, exact fp32 conv, scan and gate            */
/* ------------------------------------------------------------------ */
/* The variant that quantises only the linear layers, which FastMamba's
 * Table II reports beside the full method (pith.science review of
 * arXiv 2505.18975, Desk Editor's Note: "FastMamba-LQ").  The two linears
 * are the method's (rotation, int8, the same GEMM kernels and scales); the
 * conv1d + SiLU, SoftPlus, exp, the selective scan and the gate are Mamba2's
 * own fp32 arithmetic (the paper's reference [2]; Figure 2 caption), with
 * CUDA's expf / log1pf and no power-of-two codes or PWL unit.
 * The fp32 parameters it needs beyond an fm_layer: */
typedef struct fm_lq_params {
    const float *conv_w;  /* [conv_ch, 4], tap 3 multiplies the current token */
    const float *conv_b;  /* [conv_ch] */
    const float *a_log;   /* [nheads]: A = -exp(a_log) */
    const float *D;       /* [nheads] */
} fm_lq_params;

/* Causal depthwise conv + SiLU in fp32:
 *   out[b,t,c] = SiLU(conv_b[c] + sum_k conv_w[c,k] u[b,t-3+k,c]).
 *   u: rows of stride ldu floats (>= conv_ch; the in_proj output's xBC
 *   columns can be read in place, u = Y + d_inner, ldu = n_in), no alignment
 *   requirement.  out [B, T, conv_ch].  conv_state [B, 3, conv_ch] fp32 or
 *   NULL: the 3 inputs before token 0 (oldest first), replaced by the last 3. */
fm_status fm_lq_conv1d(const float *u, int64_t ldu, int B, int T, const fm_shape *shape,
                       const float *conv_w, const float *conv_b, float *conv_state, float *out,
                       fm_stream stream);

/* Selective scan in fp32 (Mamba2's recurrence, one group):
 *   dt = SoftPlus(dt_raw[b,t,h] + dt_bias[h]), dA = exp(-dt exp(a_log[h]))
 *   h[p,n] = dA h[p,n] + (dt x[p]) B[n];  y[p] = sum_n C[n] h[p,n] + D[h] x[p]
 *   out = y SiLU(z) when z is given (the gate), else y.
 *   xo [B, T, conv_ch] fp32 conv output (x | B | C); dt_raw rows of stride
 *   ld_dt (column h), z rows of stride ld_z (NULL: no gate); out [B, T, d_inner].
 *   state [B, nheads, 64, 128] fp32 or NULL (zeros): initial in, final out. */
fm_status fm_lq_scan(const float *xo, const float *dt_raw, int64_t ld_dt, const float *z,
                     int64_t ld_z, int B, int T, const fm_shape *shape, const float *dt_bias,
                     const float *a_log, const float *D, float *state, float *out,
                     fm_stream stream);

/* Tuning: channels per warp of the fp32 scan (0: chosen by the grid; 1, 2 or
 * 4).  Results differ only in the order of the warp's fp32 C.h sum.
 * FM_ERR_INVALID_ARG for other values. */
fm_status fm_set_lq_scan_cpw(int cpw);

/* One LQ layer: fm_hadamard_quant (with L->prenorm_w) -> in_proj GEMM (fp32
 * output) -> fm_lq_conv1d -> fm_lq_scan with the gate -> gated RMSNorm
 * (eps 1e-5, L->norm_w) + rotation + int8 (fm_hadamard_quant with norm_w as
 * its pre-norm weight) -> out_proj GEMM (+ x when residual).  L supplies the
 * linears, dt_bias, norm weights, mode and static scales; its fixed-point
 * fields are not used.  conv_state [B, 3, conv_ch] fp32 and ssm_state
 * [B, nheads, 64, 128] fp32 may be NULL (zero history, not kept).  ws: device
 * workspace of fm_lq_workspace_bytes(shape, B, T). */
size_t fm_lq_workspace_bytes(const fm_shape *shape, int B, int T);
fm_status fm_lq_mixer_prefill(const fm_layer *L, const fm_lq_params *P, const float *x, int B,
                              int T, int residual, float *conv_state, float *ssm_state,
                              float *out, void *ws, size_t ws_bytes, fm_stream stream);

/* Source: power-of-two codes for the conv weights and the SSM parameters;
 * A folded with log2(e) for the shift-based e^Delta (pith.science review of
 * FastMamba, "What carries the argument"; the verdict record's supporting
 * citation [15]).
 * Offline, per layer: quantise conv taps (e_w, wq) and the SSM parameters
 * (A_q, D_q, e_D) from fp32 device tensors: conv_w [cc, 4], a_log [nh], D [nh].
 * Writes the e_w and e_D regions of `exps`. */
fm_status fm_prepare_mixer_params(const fm_shape *shape, const float *conv_w, const float *a_log,
                                  const float *D, int8_t *conv_wq, int32_t *A_q, int32_t *D_q,
                                  int32_t *exps, fm_stream stream);

/* Calibration workspace bytes for B*T calibration tokens. */
size_t fm_calib_workspace_bytes(const fm_shape *shape, int B, int T);

/* Source: the static scales the hardware applies as "x s_coe >> s_shift"
 * (pith.science review of FastMamba, Referee major comment 1 on Fig. 6); the
 * pages do not say how they are found, so each stage's exponent is taken from
 * that stage's maximum on the calibration tokens.
 * Stage-by-stage calibration of one prepared layer on xcal [B, T, d_model]:
 * fills the remaining regions of exps (e_u, e_o, e_x, e_B, e_C, e_h, e_y,
 * e_g), conv_bq (from conv_b [cc] fp32 at e_w + e_u) and static_amax[2],
 * and writes the layer's output on xcal to out (next layer's calibration
 * input).  L->exps / L->conv_bq / L->static_amax are written through the
 * non-const pointers given here (they must be the same arrays). */
fm_status fm_calibrate_layer(const fm_layer *L, const float *conv_b, int32_t *exps,
                             int32_t *conv_bq, float *static_amax, const float *xcal, int B,
                             int T, int residual, float *out, void *ws, size_t ws_bytes,
                             fm_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* FASTMAMBA_H */
