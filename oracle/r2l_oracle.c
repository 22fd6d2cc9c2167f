/*
 * r2l_oracle.c -- plain fp64 CPU oracle of the right-to-left selective-scan sidecar.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark load this file.  The GPU library neither links nor calls it, and it
 * shares no code, header, table or constant with the GPU path.
 *
 * What is computed, and where it comes from:
 *
 *  - "Bifocal Diffusion Language Models" (technical summary, section 2 "Methodology",
 *    R2LM mechanism): the sidecar takes the backbone's hidden-state projections,
 *    reverses the sequence, applies a Mamba selective scan and reverses the result
 *    back; its output is a residual correction gated by a learnable scalar s that is
 *    initialised to zero.  Reversing, scanning forward and reversing back is the same
 *    as scanning with the time index running downwards, which is how it is written
 *    here (no copy).
 *  - Same page, "Inference": during parallel decoding the R2L scan runs on the tokens
 *    of the generation block only, so the reverse state starts from zero at the right
 *    edge of every block.
 *  - "Training Hybrid Block Diffusion Language Models with Partial Bidirectionality",
 *    "Methodology" item 1: finished prefix blocks are stored as forward-only Mamba
 *    boundary (recurrent) states, and the reverse scan is confined to the active
 *    block.  The forward direction therefore resumes from a cached state h0 and emits
 *    the state after its last token.
 *  - The pages print no scan formulas.  The S6 recurrence used is the standard
 *    Mamba-1 one: delta = softplus(dt + dt_bias), Abar = exp(delta*A),
 *    Bbar*x = delta*B*x, h_t = Abar_t*h_(t+-1) + Bbar_t*x_t, y_t = C_t.h_t + D*x_t,
 *    then y *= SiLU(z).  The state is inclusive: y_t sees x_t through h_t.
 *  - Optional depthwise convolution of width W before the scan (standard Mamba-1
 *    front-end): causal in the scan's own direction, zero outside the scanned range
 *    (right block edge for the reverse scan, sequence start for the forward scan),
 *    followed by SiLU.  The D skip uses the post-convolution value.
 *  - A forward scan that resumes a cached prefix also needs the prefix's last W-1
 *    inputs for that convolution (the standard Mamba-1 decode cache holds the
 *    convolution window beside the recurrent state).  conv_state supplies them in
 *    place of the zero padding before the first token, and conv_state_out returns
 *    the W-1 inputs that end the scanned range, so chaining calls reproduces one
 *    long scan.
 *
 * Everything is evaluated in double precision in the order written above.
 */
#include <math.h>
#include <stddef.h>

/* softplus(v) = log(1 + e^v); for v > 20 the correction is below 2e-9 relative. */
static double softplus(double v) { return v > 20.0 ? v : log1p(exp(v)); }

/* SiLU(v) = v * sigmoid(v) */
static double silu(double v) { return v / (1.0 + exp(-v)); }

/*
 * Selective scan over x[batch][seqlen][d_inner].
 *   reverse != 0 : right-to-left; the state is zero at the right edge of every
 *                  block of block_len tokens (block_len divides seqlen); h0 and
 *                  h_last must be NULL (the reverse pass emits no state).
 *   reverse == 0 : left-to-right over the whole sequence, starting from h0
 *                  ([batch][d_inner][d_state], NULL = zeros) and writing the state
 *                  after the last token to h_last (NULL = not wanted).
 *                  conv_state ([batch][d_inner][conv_width-1], NULL = zeros):
 *                  the convolution's inputs before the first token, index j = the
 *                  input j+1 tokens before it.  conv_state_out (same layout, NULL =
 *                  not wanted): the inputs that end the scan, index j = the input
 *                  j tokens back from the last one.  Reverse scans take NULL.
 * B, C: [batch][seqlen][d_state] shared by all channels.  z: NULL = no gate.
 * A: [d_inner][d_state]; D, dt_bias: [d_inner]; conv_w: [d_inner][conv_width],
 * conv_b: [d_inner] (both NULL iff conv_width == 0).  y: [batch][seqlen][d_inner].
 * Returns 0 on success, -1 on bad arguments.
 */
int r2l_oracle_scan(int reverse, long batch, long seqlen, long block_len, long d_inner,
                    long d_state, long conv_width,
                    const double *x, const double *dt, const double *Bm, const double *Cm,
                    const double *z, const double *A, const double *Dskip,
                    const double *dt_bias, const double *conv_w, const double *conv_b,
                    const double *h0, double *h_last, const double *conv_state,
                    double *conv_state_out, double *y)
{
    enum { MAX_STATE = 256, MAX_CONV = 64 };
    double h[MAX_STATE];
    double cs_new[MAX_CONV];
    if (batch < 0 || seqlen < 0 || d_inner < 0 || d_state <= 0 || d_state > MAX_STATE) return -1;
    if (conv_width < 0 || conv_width > MAX_CONV || (conv_width > 0 && (!conv_w || !conv_b))) return -1;
    if ((conv_state || conv_state_out) && (reverse || conv_width < 2)) return -1;
    if (!x || !dt || !Bm || !Cm || !A || !Dskip || !dt_bias || !y) return -1;
    if (reverse) {
        if (block_len <= 0 || (seqlen % block_len) != 0 || h0 || h_last) return -1;
    } else {
        block_len = seqlen;
    }
    if (seqlen == 0) block_len = 1;

    for (long b = 0; b < batch; ++b) {
        for (long d = 0; d < d_inner; ++d) {
            for (long blk = 0; blk * block_len < seqlen; ++blk) {
                const long s0 = blk * block_len, s1 = s0 + block_len; /* [s0, s1) */
                for (long n = 0; n < d_state; ++n)
                    h[n] = (!reverse && h0) ? h0[(b * d_inner + d) * d_state + n] : 0.0;
                for (long i = 0; i < block_len; ++i) {
                    const long t = reverse ? (s1 - 1 - i) : (s0 + i);
                    const long row = b * seqlen + t;
                    double u = x[row * d_inner + d];
                    if (conv_width > 0) {
                        /* Causal in scan order: tap k looks (W-1-k) tokens back along the
                         * scan, i.e. towards larger t for the reverse scan. */
                        double acc = conv_b[d];
                        for (long k = 0; k < conv_width; ++k) {
                            const long back = conv_width - 1 - k;
                            const long tt = reverse ? (t + back) : (t - back);
                            double xv = 0.0;
                            if (tt >= s0 && tt < s1)
                                xv = x[(b * seqlen + tt) * d_inner + d];
                            else if (conv_state && tt < s0) /* the cached prefix inputs */
                                xv = conv_state[(b * d_inner + d) * (conv_width - 1) + (s0 - 1 - tt)];
                            acc += conv_w[d * conv_width + k] * xv;
                        }
                        u = silu(acc);
                    }
                    const double delta = softplus(dt[row * d_inner + d] + dt_bias[d]);
                    double acc_y = 0.0;
                    for (long n = 0; n < d_state; ++n) {
                        const double abar = exp(delta * A[d * d_state + n]);
                        h[n] = abar * h[n] + delta * Bm[row * d_state + n] * u;
                        acc_y += Cm[row * d_state + n] * h[n];
                    }
                    double yv = acc_y + Dskip[d] * u;
                    if (z) yv *= silu(z[row * d_inner + d]);
                    y[row * d_inner + d] = yv;
                }
                if (!reverse && h_last)
                    for (long n = 0; n < d_state; ++n)
                        h_last[(b * d_inner + d) * d_state + n] = h[n];
                if (conv_state_out) {
                    /* input j tokens back from the last one, reaching into the cached
                     * prefix when the range is shorter than the window; buffered so
                     * that conv_state_out may alias conv_state */
                    for (long j = 0; j < conv_width - 1; ++j) {
                        const long tt = s1 - 1 - j;
                        if (tt >= s0)
                            cs_new[j] = x[(b * seqlen + tt) * d_inner + d];
                        else
                            cs_new[j] = conv_state ? conv_state[(b * d_inner + d) * (conv_width - 1) + (s0 - 1 - tt)] : 0.0;
                    }
                    for (long j = 0; j < conv_width - 1; ++j)
                        conv_state_out[(b * d_inner + d) * (conv_width - 1) + j] = cs_new[j];
                }
            }
        }
    }
    return 0;
}

/*
 * Residual correction (R2LM "Integration"): out = hidden + s * (y . W_out^T).
 * hidden, out: [M][d_model]; y: [M][d_inner]; W_out: [d_model][d_inner].
 */
int r2l_oracle_residual(long M, long d_model, long d_inner, const double *hidden,
                        const double *y, const double *W_out, double s, double *out)
{
    if (M < 0 || d_model < 0 || d_inner < 0 || !hidden || !y || !W_out || !out) return -1;
    for (long m = 0; m < M; ++m) {
        for (long j = 0; j < d_model; ++j) {
            double acc = 0.0;
            for (long k = 0; k < d_inner; ++k) acc += y[m * d_inner + k] * W_out[j * d_inner + k];
            out[m * d_model + j] = hidden[m * d_model + j] + s * acc;
        }
    }
    return 0;
}

/*
 * Dense projection out = X . W^T (no bias), the building block of the sidecar's input
 * projections (standard Mamba-1 in_proj, x_proj and dt_proj; the pages only say that the
 * sidecar applies a Mamba selective scan to projections of the hidden states).
 * X: [M][K]; W: [N][K]; out: [M][N].
 */
int r2l_oracle_linear(long M, long N, long K, const double *X, const double *W, double *out)
{
    if (M < 0 || N < 0 || K < 0 || !X || !W || !out) return -1;
    for (long m = 0; m < M; ++m)
        for (long n = 0; n < N; ++n) {
            double acc = 0.0;
            for (long k = 0; k < K; ++k) acc += X[m * K + k] * W[n * K + k];
            out[m * N + n] = acc;
        }
    return 0;
}

/*
 * The scan's convolution front-end on its own: u = SiLU(conv_b + depthwise convolution of x),
 * causal in scan order and zero outside the scanned range, exactly as inside r2l_oracle_scan
 * (reverse: inside each block of block_len tokens, taps reaching right of the block read zero).
 * x, u: [batch][seqlen][d_inner]; conv_w: [d_inner][conv_width]; conv_b: [d_inner].
 */
int r2l_oracle_conv_silu(int reverse, long batch, long seqlen, long block_len, long d_inner,
                         long conv_width, const double *x, const double *conv_w,
                         const double *conv_b, double *u)
{
    if (batch < 0 || seqlen < 0 || d_inner < 0 || conv_width <= 0) return -1;
    if (!x || !conv_w || !conv_b || !u) return -1;
    if (reverse) {
        if (block_len <= 0 || (seqlen % block_len) != 0) return -1;
    } else {
        block_len = seqlen;
    }
    for (long b = 0; b < batch; ++b)
        for (long t = 0; t < seqlen; ++t) {
            const long s0 = (t / block_len) * block_len, s1 = s0 + block_len;
            for (long d = 0; d < d_inner; ++d) {
                double acc = conv_b[d];
                for (long k = 0; k < conv_width; ++k) {
                    const long lag = conv_width - 1 - k; /* tokens back along the scan */
                    const long tsrc = reverse ? t + lag : t - lag;
                    const double xv = (tsrc >= s0 && tsrc < s1) ? x[(b * seqlen + tsrc) * d_inner + d] : 0.0;
                    acc += conv_w[d * conv_width + k] * xv;
                }
                u[(b * seqlen + t) * d_inner + d] = silu(acc);
            }
        }
    return 0;
}

/*
 * Gradient of the right-to-left block scan (gate and convolution front-end optional), for training
 * the sidecar as a plug-in ("Bifocal Diffusion Language Models", section 2: the sidecar is the only
 * trained part in the plug-in setting).  Reverse-mode differentiation of the recurrence in
 * r2l_oracle_scan, written out:
 *   front-end:   u_t = x_t, or with the convolution of width W (causal in the reverse scan's
 *                order, zero past the block's right edge)
 *                c_t = conv_b + sum_k conv_w[k] x_(t+W-1-k),  u_t = SiLU(c_t)
 *   forward, t = s1-1 .. s0:  delta_t = softplus(dt_t + bias),  a_tn = exp(delta_t A_n),
 *                             h_tn = a_tn h_(t+1)n + delta_t B_tn u_t  (h_(s1) = 0),
 *                             p_t = sum_n C_tn h_tn + D u_t,  y_t = p_t SiLU(z_t)
 *   adjoint,  t = s0 .. s1-1: dp_t = dy_t SiLU(z_t)
 *                             G_tn = dp_t C_tn + a_(t-1)n G_(t-1)n   (dL/dh_tn; no second term at s0)
 *   then   dz_t = dy_t p_t SiLU'(z_t),   dD += dp_t u_t,   dC_tn += dp_t h_tn,
 *          da_tn = G_tn h_(t+1)n,  ddelta_t = sum_n (da_tn a_tn A_n + G_tn B_tn u_t),
 *          dA_n += da_tn a_tn delta_t,  dB_tn += G_tn delta_t u_t,
 *          du_t = dp_t D + sum_n G_tn delta_t B_tn,
 *          ddt_t = ddelta_t sigmoid(dt_t + bias),  dbias += ddt_t,
 *   and through the front-end: without the convolution dx_t = du_t; with it
 *          dc_t = du_t SiLU'(c_t),  dx_s = sum_k conv_w[k] dc_(s-(W-1-k)) (terms inside the block),
 *          dconv_w[k] += dc_t x_(t+W-1-k),  dconv_b += dc_t.
 * B and C are shared by all channels, so dB and dC sum over channels; dA, dD, dbias, dconv_w and
 * dconv_b sum over batch rows and tokens.  All outputs are overwritten.  dz may be NULL when z is
 * NULL; conv_w, conv_b, dconv_w ([d_inner][W]) and dconv_b ([d_inner]) are NULL iff W == 0.
 * Returns 0 on success, -1 on bad arguments.
 */
int r2l_oracle_scan_bwd(long batch, long seqlen, long block_len, long d_inner, long d_state, long conv_width,
                        const double *x, const double *dt, const double *Bm, const double *Cm,
                        const double *z, const double *A, const double *Dskip, const double *dt_bias,
                        const double *conv_w, const double *conv_b, const double *dy,
                        double *dx, double *ddt, double *dB, double *dC, double *dz,
                        double *dA, double *dD, double *ddt_bias, double *dconv_w, double *dconv_b)
{
    enum { MAX_STATE = 256, MAX_BLOCK = 4096, MAX_CONV = 64 };
    static double hs[MAX_BLOCK + 1][MAX_STATE]; /* h_t of the current block, hs[i] = h at s0 + i */
    static double ub[MAX_BLOCK], cb[MAX_BLOCK], dub[MAX_BLOCK]; /* u_t, c_t and du_t of the block */
    double G[MAX_STATE];
    const long W = conv_width;
    if (batch < 0 || seqlen < 0 || d_inner < 0 || d_state <= 0 || d_state > MAX_STATE) return -1;
    if (block_len <= 0 || block_len > MAX_BLOCK || (seqlen % block_len) != 0) return -1;
    if (W < 0 || W > MAX_CONV) return -1;
    if ((W > 0) != (conv_w && conv_b && dconv_w && dconv_b)) return -1;
    if (W == 0 && (conv_w || conv_b || dconv_w || dconv_b)) return -1;
    if (!x || !dt || !Bm || !Cm || !A || !Dskip || !dt_bias || !dy) return -1;
    if (!dx || !ddt || !dB || !dC || !dA || !dD || !ddt_bias || (z && !dz)) return -1;
    for (long i = 0; i < batch * seqlen * d_inner; ++i) { dx[i] = 0.0; ddt[i] = 0.0; if (dz) dz[i] = 0.0; }
    for (long i = 0; i < batch * seqlen * d_state; ++i) { dB[i] = 0.0; dC[i] = 0.0; }
    for (long i = 0; i < d_inner * d_state; ++i) dA[i] = 0.0;
    for (long d = 0; d < d_inner; ++d) { dD[d] = 0.0; ddt_bias[d] = 0.0; }
    for (long i = 0; i < d_inner * W; ++i) dconv_w[i] = 0.0;
    for (long d = 0; W > 0 && d < d_inner; ++d) dconv_b[d] = 0.0;

    for (long b = 0; b < batch; ++b) {
        for (long d = 0; d < d_inner; ++d) {
            for (long s0 = 0; s0 < seqlen; s0 += block_len) {
                const long s1 = s0 + block_len;
                /* the front-end's outputs u_t (and pre-activations c_t) of the block */
                for (long t = s0; t < s1; ++t) {
                    const double xv = x[(b * seqlen + t) * d_inner + d];
                    if (W == 0) {
                        ub[t - s0] = xv;
                        continue;
                    }
                    double acc = conv_b[d];
                    for (long k = 0; k < W; ++k) {
                        const long tt = t + (W - 1 - k);
                        if (tt < s1) acc += conv_w[d * W + k] * x[(b * seqlen + tt) * d_inner + d];
                    }
                    cb[t - s0] = acc;
                    ub[t - s0] = silu(acc);
                }
                /* forward states, right to left */
                for (long n = 0; n < d_state; ++n) hs[block_len][n] = 0.0;
                for (long t = s1 - 1; t >= s0; --t) {
                    const long row = b * seqlen + t;
                    const double u = ub[t - s0];
                    const double delta = softplus(dt[row * d_inner + d] + dt_bias[d]);
                    for (long n = 0; n < d_state; ++n) {
                        const double a = exp(delta * A[d * d_state + n]);
                        hs[t - s0][n] = a * hs[t - s0 + 1][n] + delta * Bm[row * d_state + n] * u;
                    }
                }
                /* adjoint, left to right */
                for (long t = s0; t < s1; ++t) {
                    const long row = b * seqlen + t;
                    const double u = ub[t - s0];
                    const double v = dt[row * d_inner + d] + dt_bias[d];
                    const double delta = softplus(v);
                    double p = Dskip[d] * u;
                    for (long n = 0; n < d_state; ++n) p += Cm[row * d_state + n] * hs[t - s0][n];
                    double g = 1.0, dg = 0.0;
                    if (z) {
                        const double zz = z[row * d_inner + d];
                        const double sg = 1.0 / (1.0 + exp(-zz));
                        g = zz * sg;
                        dg = sg * (1.0 + zz * (1.0 - sg));
                    }
                    const double dp = dy[row * d_inner + d] * g;
                    if (z) dz[row * d_inner + d] = dy[row * d_inner + d] * p * dg;
                    dD[d] += dp * u;
                    double ddelta = 0.0, du = dp * Dskip[d];
                    double delta_prev = 0.0;
                    if (t > s0) delta_prev = softplus(dt[(row - 1) * d_inner + d] + dt_bias[d]);
                    for (long n = 0; n < d_state; ++n) {
                        const double An = A[d * d_state + n];
                        const double Gprev = (t > s0) ? exp(delta_prev * An) * G[n] : 0.0;
                        G[n] = dp * Cm[row * d_state + n] + Gprev;
                        const double a = exp(delta * An);
                        const double da = G[n] * hs[t - s0 + 1][n];
                        dC[row * d_state + n] += dp * hs[t - s0][n];
                        ddelta += da * a * An + G[n] * Bm[row * d_state + n] * u;
                        dA[d * d_state + n] += da * a * delta;
                        dB[row * d_state + n] += G[n] * delta * u;
                        du += G[n] * delta * Bm[row * d_state + n];
                    }
                    const double ddt_t = ddelta / (1.0 + exp(-v)); /* softplus' = sigmoid */
                    ddt[row * d_inner + d] = ddt_t;
                    ddt_bias[d] += ddt_t;
                    dub[t - s0] = du;
                }
                /* back through the front-end */
                for (long t = s0; t < s1; ++t) {
                    const long row = b * seqlen + t;
                    if (W == 0) {
                        dx[row * d_inner + d] = dub[t - s0];
                        continue;
                    }
                    const double c = cb[t - s0];
                    const double sg = 1.0 / (1.0 + exp(-c));
                    const double dc = dub[t - s0] * sg * (1.0 + c * (1.0 - sg)); /* SiLU'(c) */
                    dconv_b[d] += dc;
                    for (long k = 0; k < W; ++k) {
                        const long tt = t + (W - 1 - k);
                        if (tt >= s1) continue;
                        dconv_w[d * W + k] += dc * x[(b * seqlen + tt) * d_inner + d];
                        dx[(b * seqlen + tt) * d_inner + d] += conv_w[d * W + k] * dc;
                    }
                }
            }
        }
    }
    return 0;
}
