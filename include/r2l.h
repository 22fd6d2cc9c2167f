/*
 * r2l.h -- C ABI of the B200 (sm_100a) right-to-left selective-scan sidecar library (libr2l.so).
 *
 * The library implements the data-parallel hot path of the R2LM sidecar:
 *
 *   "Bifocal Diffusion Language Models", section 2 (Methodology, R2LM): the sidecar takes the
 *   causal backbone's hidden-state projections, reverses the token order, runs a Mamba
 *   selective scan, reverses back and adds the result to the hidden state as a residual
 *   correction scaled by a learnable scalar s that starts at zero; during parallel decoding
 *   the scan runs over the tokens of the generation block only.
 *
 *   "Training Hybrid Block Diffusion Language Models with Partial Bidirectionality",
 *   Methodology item 1: the forward Mamba direction resumes from a cached forward-only
 *   boundary state and the reverse direction is confined to the active block.
 *
 * The pages give no formulas for the scan; the standard Mamba-1 (S6) recurrence is used:
 *   delta_t = softplus(dt_t + dt_bias)              per (batch, token, channel)
 *   Abar    = exp(delta_t * A[d][n]),  Bbar x = delta_t * B_t[n] * u_t
 *   reverse: h_t = Abar_t * h_(t+1) + Bbar_t x_t    (h = 0 to the right of each block)
 *   forward: h_t = Abar_t * h_(t-1) + Bbar_t x_t    (h_(-1) = h0)
 *   y_t = sum_n C_t[n] h_t[n] + D[d] * u_t,  then y_t *= SiLU(z_t)
 * where u is x, or SiLU(conv_b + causal depthwise conv of x) when conv_width == 4 (the
 * convolution is causal in scan order and sees zeros outside the scanned range).
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library allocates no
 *    device memory and never frees caller memory.  Layouts are dense row-major (C order).
 *  - Work is enqueued asynchronously on `stream`; the return value reports host-side
 *    argument validation and launch errors only.  Device-side failures (a bounded wait that
 *    ran out) set a library-global device status word that r2l_device_status() reads.
 *  - Sizes of zero (batch, seqlen, d_inner, M, d_model) are valid and enqueue nothing.
 *  - There is no CPU fallback: without a usable sm_100 device every compute call returns
 *    R2L_ERR_CUDA.
 *  - Entry points are thread-safe; concurrent calls on different streams are independent
 *    except that they share the device status word.
 */
#ifndef R2L_H
#define R2L_H

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define R2L_API __attribute__((visibility("default")))
#else
#define R2L_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    R2L_OK = 0,
    R2L_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, negative or inconsistent size      */
    R2L_ERR_UNSUPPORTED = 2,  /* valid but not built: d_state != 16, conv_width not in {0,4}  */
    R2L_ERR_CUDA = 3,         /* a CUDA runtime/driver call or kernel launch failed           */
    R2L_ERR_TIMEOUT = 4       /* a device-side bounded wait ran out (see r2l_device_status)   */
} r2l_status;

typedef enum { R2L_F32 = 0, R2L_BF16 = 1 } r2l_dtype;

/*
 * One direction of a selective scan.
 *   x, dt, z : [batch][seqlen][d_inner] of in_dtype.  z may be NULL (no output gate).
 *   B, C     : [batch][seqlen][d_state] of in_dtype (one group, shared by all channels).
 *   A        : [d_inner][d_state] fp32, negative (A = -exp(A_log)).
 *   D, dt_bias: [d_inner] fp32.
 *   conv_w   : [d_inner][conv_width] fp32, conv_b: [d_inner] fp32; both NULL iff conv_width == 0.
 *   block_len: reverse scans restart from a zero state at the right edge of every block of
 *              block_len tokens; block_len must divide seqlen.  Ignored by forward scans.
 *   conv_state, conv_state_out: forward scans with conv_width 4 only (NULL otherwise).
 *              [batch][d_inner][conv_width - 1] fp32: the x values of the tokens just before the
 *              first one (index 0 = one token back), NULL = zeros; and the same for the tokens
 *              ending the scanned range, written on exit (NULL = not written).  They carry the
 *              convolution across calls the way h0/h_last carry the state, so a cached prefix
 *              continues exactly ("Training Hybrid Block Diffusion Language Models with Partial
 *              Bidirectionality", Methodology item 1).  conv_state_out may alias conv_state.
 *              4-byte aligned.  A call with seqlen == 0 writes neither (nor h_last).
 * Requirements: d_state == 16; conv_width in {0, 4}; d_inner a multiple of 8 (bf16) or
 * 4 (fp32); x, dt, z, B, C, A and conv_w 16-byte aligned.
 */
typedef struct {
    int batch, seqlen, block_len;
    int d_inner, d_state, conv_width;
    r2l_dtype in_dtype;
    const void *x, *dt, *B, *C, *z;
    const float *A, *D, *dt_bias;
    const float *conv_w, *conv_b;
    const float *conv_state;
    float *conv_state_out;
} r2l_scan_args;

/*
 * Right-to-left selective scan over each block of a->block_len tokens ("Bifocal Diffusion
 * Language Models", section 2: reverse, scan, reverse back; scan on generation-block tokens
 * only).  The reversal is done by index arithmetic; nothing is copied.
 *   y : [batch][seqlen][d_inner] of y_dtype, device, written at the original token index.
 *       Must not overlap any input.  16-byte aligned.
 * The kernel and its launch shape depend on the problem size (one lane per two channels, a
 * balanced 16-warp launch, chunked long blocks, or four lanes per channel for launches under one
 * warp per SM); a row's outputs are bit-identical whichever of the first, second and last runs it.
 */
R2L_API r2l_status r2l_scan_block(const r2l_scan_args *a, void *y, r2l_dtype y_dtype, cudaStream_t stream);

/*
 * Forward selective scan resumed from a cached boundary state, optionally fused with the
 * block-confined reverse scan of the partial-bidirectional mixer ("Training Hybrid Block
 * Diffusion Language Models with Partial Bidirectionality", Methodology item 1).
 *   fwd    : forward direction over fwd->seqlen tokens (block_len ignored); its z is the gate.
 *   rev    : NULL, or the reverse direction over the same batch/seqlen/d_inner.  x and z must
 *            be the same pointers as fwd's; dt, B, C, A, D, dt_bias, conv are its own.
 *            rev->block_len must divide seqlen and be at most 64.
 *   h0     : [batch][d_inner][d_state] fp32 cached forward state; NULL = zeros.
 *   h_last : [batch][d_inner][d_state] fp32 forward state after the last token; NULL = not
 *            written.  May alias h0 (each state row is read completely before it is written).
 *   y      : [batch][seqlen][d_inner] of y_dtype = (y_fwd [+ y_rev]) * SiLU(z) (gate applied
 *            once to the sum; no gate if fwd->z is NULL).
 * Split points are exact: scanning a prefix, passing its h_last as h0 and scanning the rest
 * reproduces the one-shot forward scan bit for bit.
 */
R2L_API r2l_status fwd_scan_from_state(const r2l_scan_args *fwd, const r2l_scan_args *rev,
                               const float *h0, float *h_last, void *y, r2l_dtype y_dtype,
                               cudaStream_t stream);

/*
 * Gradient of r2l_scan_block (gate and width-4 convolution front-end optional), for training the
 * sidecar as a plug-in ("Bifocal Diffusion Language Models", section 2).  Given dy = dL/dy
 * ([batch][seqlen][d_inner], dy_dtype), writes fp32
 *   dx, ddt, dz [batch][seqlen][d_inner]  (dz NULL iff a->z is NULL; dx is the gradient of the
 *                                          raw x, through the convolution when there is one),
 *   dB, dC      [batch][seqlen][d_state]  (summed over channels),
 *   dA          [d_inner][d_state], dD and ddt_bias [d_inner]  (summed over rows and tokens),
 *   dconv_w     [d_inner][4], dconv_b [d_inner]  (summed over rows and tokens; both NULL iff
 *                                          a->conv_width == 0).
 * Every output is overwritten (the sums are zeroed first on `stream`).  Requirements beyond
 * r2l_scan_block's: block_len <= 64, d_inner a multiple of 16, batch * seqlen / block_len <= 65535
 * (R2L_ERR_UNSUPPORTED otherwise).  The channel and token sums use atomic adds, so their last bits
 * may differ between runs.
 */
R2L_API r2l_status r2l_scan_block_bwd(const r2l_scan_args *a, const void *dy, r2l_dtype dy_dtype, float *dx,
                                      float *ddt, float *dB, float *dC, float *dz, float *dA, float *dD,
                                      float *ddt_bias, float *dconv_w, float *dconv_b, cudaStream_t stream);

/*
 * Bidirectional scan for any reverse block length, up to the whole window:
 *   y = (y_f + y_r) * SiLU(z)
 * with y_f the forward scan of `fwd` from h0 (writing h_last, and the convolution state when
 * fwd carries one) and y_r the reverse scan of `rev` restarted at the right edge of every block of
 * rev->block_len tokens.  rev->block_len = seqlen gives the fully bidirectional scan of earlier
 * hybrids whose reverse pass covers the whole denoising window ("Training Hybrid Block Diffusion
 * Language Models with Partial Bidirectionality", Problem statement); block_len = the active block
 * gives the partial-bidirectional mixer of fwd_scan_from_state (Methodology item 1) without its
 * 64-token limit.  x and z are shared as in fwd_scan_from_state.
 * Runs as two ungated fp32 scans into `workspace` (caller-owned, >= r2l_bidir_scan_workspace_size
 * bytes, 256-byte aligned) and one elementwise pass.  Results agree with fwd_scan_from_state
 * within rounding (not bit for bit: the two paths round differently).
 */
R2L_API size_t r2l_bidir_scan_workspace_size(const r2l_scan_args *fwd);
R2L_API r2l_status r2l_bidir_scan(const r2l_scan_args *fwd, const r2l_scan_args *rev, const float *h0,
                                  float *h_last, void *y, r2l_dtype y_dtype, void *workspace,
                                  size_t workspace_bytes, cudaStream_t stream);

/*
 * Residual correction: hidden <- hidden + s * (y . W_out^T) ("Bifocal Diffusion Language
 * Models", section 2: residual correction signal gated by the scalar s).
 *   hidden : [M][d_model] of dtype, updated in place.
 *   y      : [M][d_inner] of dtype;  W_out: [d_model][d_inner] of dtype.
 *   dtype  : R2L_BF16 -> tcgen05 tensor-core GEMM, fp32 accumulation, fp32 epilogue,
 *            result rounded to bf16 (RNE).  R2L_F32 -> fp32 FMA kernel.
 *            With M <= 64 and d_inner a multiple of 64 the bf16 GEMM splits d_inner over a
 *            cluster of up to 8 CTAs and sums the partial products in a fixed order: the result
 *            is the same from run to run (the split depends only on M, d_model and d_inner).
 *   s == 0 returns immediately and leaves hidden bit-identical (identity at initialisation).
 * Requirements: d_inner a multiple of 8 (bf16) / 4 (fp32); d_model a multiple of 8 for bf16;
 * pointers 16-byte aligned; y and W_out must not overlap hidden.
 */
R2L_API r2l_status r2l_residual_apply(void *hidden, const void *y, const void *W_out, float s, int M,
                              int d_model, int d_inner, r2l_dtype dtype, cudaStream_t stream);

/*
 * One R2LM decode step of the sidecar from its scan operands ("Bifocal Diffusion Language
 * Models", section 2: the right-to-left scan over each generation block, then the residual
 * correction gated by s): r2l_scan_block(a, y, dtype) followed by r2l_residual_apply(hidden, y,
 * W_out, s, a->batch * a->seqlen, d_model, a->d_inner, dtype), with the same results bit for bit.
 * While the scan runs, its CTAs pull W_out and hidden into L2 (bulk prefetches, a hint that moves
 * no data into the kernel), so that the residual GEMM finds its operands there; neither depends
 * on the scan.
 *   a      : as for r2l_scan_block; y [batch][seqlen][d_inner] of dtype, written, then read by
 *            the residual.
 *   hidden : [batch * seqlen][d_model] of dtype, updated in place;  W_out: [d_model][d_inner].
 *   s == 0 or d_model == 0: the scan runs, hidden is not touched (hidden and W_out may be NULL).
 * Requirements: those of both calls; hidden, W_out and y must not overlap one another or the
 * scan's inputs.  Errors are those of the two calls; an argument error launches nothing.
 */
R2L_API r2l_status r2l_decode_step(const r2l_scan_args *a, void *y, void *hidden, const void *W_out, float s,
                                   int d_model, r2l_dtype dtype, cudaStream_t stream);

/*
 * ---------------------------------------------------------------------------------------------
 * Sidecar front-end: from hidden states to the operands of the right-to-left scan.
 *
 * "Bifocal Diffusion Language Models", section 2 (R2LM mechanism): the sidecar runs a Mamba
 * selective scan on projections of the backbone's hidden states and projects its output back.
 * The pages do not spell the projections out; those of the standard Mamba-1 block are used
 * (expand = d_inner / d_model, dt_rank = ceil(d_model / 16) in the usual sizing):
 *   [x | z]            = hidden . W_in^T            W_in  [2 d_inner][d_model]  (x rows first)
 *   u                  = SiLU(conv(x))              right to left inside each block of block_len
 *                                                   tokens: u_t = SiLU(conv_b + sum_k
 *                                                   conv_w[k] x_(t+3-k)), zero past the block end
 *   [dt_low | B | C]   = u . W_x^T                  W_x   [dt_rank + 2 d_state][d_inner]
 *   dt                 = dt_low . W_dt^T            W_dt  [d_inner][dt_rank]   (dt_bias is added
 *                                                   inside the scan's softplus)
 * All tensors are bf16 row-major device buffers; the products accumulate in fp32 on the tensor
 * cores and round once to bf16.  Token rows are (batch, token) pairs, M = batch * seqlen.
 * ---------------------------------------------------------------------------------------------
 */

/*
 * in_proj with the convolution fused: u, z [M][d_inner] from hidden [M][d_model].
 * conv_w [d_inner][4] / conv_b [d_inner] fp32, both NULL for no convolution (then u = x and
 * block_len is ignored).  Requirements: d_model % 8 == 0, d_inner % 64 == 0, block_len > 0
 * dividing seqlen (with the convolution); all pointers 16-byte aligned.  M == 0 enqueues nothing.
 */
R2L_API r2l_status r2l_in_proj(const void *hidden, const void *W_in, const float *conv_w, const float *conv_b,
                               int batch, int seqlen, int block_len, int d_model, int d_inner, void *u, void *z,
                               cudaStream_t stream);

/* Bytes of device workspace r2l_x_proj needs (fp32 partial sums of its split reduction). */
R2L_API size_t r2l_x_proj_workspace_size(int M, int d_inner, int dt_rank, int d_state);

/*
 * x_proj: dt_low [M][dt_rank], B, C [M][d_state] (bf16) from u [M][d_inner].  The reduction over
 * d_inner is split across CTAs; the partial sums land in `workspace` (caller-owned, at least
 * r2l_x_proj_workspace_size bytes, 16-byte aligned) and are added in a fixed order, so results
 * are deterministic.  Requirements: d_inner % 8 == 0, dt_rank % 16 == 0, d_state % 8 == 0,
 * dt_rank + 2 d_state <= 256; pointers 16-byte aligned.
 */
R2L_API r2l_status r2l_x_proj(const void *u, const void *W_x, int M, int d_inner, int dt_rank, int d_state,
                              void *dt_low, void *B, void *C, void *workspace, size_t workspace_bytes,
                              cudaStream_t stream);

/*
 * r2l_x_proj without a caller workspace: the same computation and results as r2l_x_proj (bit for
 * bit), with the partial sums in a 16 MiB scratch array that the library holds in each device's
 * memory (a module global; nothing is allocated at call time).  Inputs whose split reduction needs
 * more than that scratch return R2L_ERR_UNSUPPORTED (the decode step, 2048 tokens at N = 160,
 * needs 10.5 MB).  Because the scratch is shared, calls on one device must be ordered (one stream,
 * or streams synchronised with each other); concurrent calls on unordered streams would race.
 */
R2L_API r2l_status r2l_x_proj_noalloc(const void *u, const void *W_x, int M, int d_inner, int dt_rank, int d_state,
                                      void *dt_low, void *B, void *C, cudaStream_t stream);

/*
 * dt_proj: dt [M][d_inner] (bf16) = dt_low [M][dt_rank] . W_dt^T.  Requirements: dt_rank % 8 == 0,
 * d_inner % 8 == 0; pointers 16-byte aligned.
 */
R2L_API r2l_status r2l_dt_proj(const void *dt_low, const void *W_dt, int M, int dt_rank, int d_inner, void *dt,
                               cudaStream_t stream);

/* Weights of one sidecar (all device pointers, bf16 unless marked fp32). */
typedef struct {
    int d_model, d_inner, d_state, dt_rank, conv_width; /* d_state == 16, conv_width in {0, 4} */
    const void *W_in;                                   /* [2 d_inner][d_model]                  */
    const float *conv_w, *conv_b;                       /* fp32 [d_inner][4], [d_inner]; or NULL */
    const void *W_x;                                    /* [dt_rank + 2 d_state][d_inner]        */
    const void *W_dt;                                   /* [d_inner][dt_rank]                    */
    const float *A, *D, *dt_bias;                       /* fp32 [d_inner][d_state], [d_inner] x2 */
    const void *W_out;                                  /* [d_model][d_inner]                    */
} r2l_sidecar_weights;

/* Bytes of device workspace r2l_sidecar_forward needs for batch x seqlen tokens. */
R2L_API size_t r2l_sidecar_workspace_size(const r2l_sidecar_weights *w, int batch, int seqlen);

/*
 * The whole sidecar on the active tokens, hidden -> hidden, in place:
 *   hidden += s * out_proj( RightToLeftScan(u, dt, B, C, z) )      (bf16 hidden [M][d_model])
 * = r2l_in_proj, r2l_x_proj, r2l_dt_proj, r2l_scan_block (block_len, no further convolution)
 * and r2l_residual_apply, enqueued back to back on `stream` with the intermediates in
 * `workspace` (caller-owned, >= r2l_sidecar_workspace_size bytes, 256-byte aligned).
 * s == 0 leaves hidden bit-identical and enqueues nothing ("Bifocal Diffusion Language Models",
 * section 2: s starts at zero so the sidecar starts as the identity).
 */
R2L_API r2l_status r2l_sidecar_forward(const r2l_sidecar_weights *w, int batch, int seqlen, int block_len, float s,
                                       void *hidden, void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* Human-readable name of a status code (static string, never NULL). */
R2L_API const char *r2l_status_string(r2l_status status);

/*
 * Synchronises `stream`, then reads and clears the library's device status word.
 * Returns R2L_OK, R2L_ERR_TIMEOUT if a kernel gave up a bounded wait since the last call,
 * or R2L_ERR_CUDA if the synchronisation itself failed.
 */
R2L_API r2l_status r2l_device_status(cudaStream_t stream);

/*
 * Description of the last CUDA failure seen by a library call on the calling thread (the
 * call that returned R2L_ERR_CUDA): the failing runtime/driver call and CUDA's error name.
 * Static thread-local storage; empty string if none.
 */
R2L_API const char *r2l_last_error(void);

/*
 * Failure-path self-test: enqueues one CTA whose mbarrier wait can never complete.  Like every wait
 * in the library's kernels it is bounded (2 s of %globaltimer); when it runs out it sets the
 * device status word and the kernel returns, leaving the context usable.  A following
 * r2l_device_status(stream) returns R2L_ERR_TIMEOUT (and clears the word).  For tests of the
 * failure detection; no fault, trap or hang is involved.
 */
R2L_API r2l_status r2l_wait_selftest(cudaStream_t stream);

/* ABI version of this header (major * 100 + minor): 102. */
R2L_API int r2l_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* R2L_H */
