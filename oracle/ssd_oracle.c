/*
 * Bidirectional Mamba-2 SSD mixer: plain sequential fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the reference that the sm_100a
 * kernels are checked against. Only the tests, the smoke check and the
 * CPU-baseline leg of the benchmark may load it; the library never does.
 * It shares no code, header or constant with the CUDA path.
 *
 * What it computes (per batch b, head h, direction d; head h reads the B/C
 * group g = h / (H/G)):
 *
 *   forward  (t = 0 .. L-1):   h_t  = exp(dt_t*A) * h_{t-1}  + dt_t * B_t x_t^T
 *                              yf_t = C_t^T h_t
 *   reverse  (t = L-1 .. 0):   h'_t = exp(dt'_t*A') * h'_{t+1} + dt'_t * B'_t x_t^T
 *                              yb_t = C'_t^T h'_t
 *   output:                    y_t  = yf_t + yb_t + (D_f + D_b) * x_t
 *
 * h is an N x P matrix (d_state x head_dim) that starts at zero (or at a
 * given initial state for the prefix-state call). There is no chunking,
 * no blocking and no reordering: one token after the other, in double
 * precision, with exp() from libm.
 *
 * Sources:
 *  - "DiffuMamba: High-Throughput Diffusion LMs with Mamba Backbone"
 *    (gist.science, 2511.15927), Technical Summary, 2. Methodology, Core
 *    Architecture: one Mamba-2 layer runs over the sequence forward, one
 *    backward, and the two results are added.
 *  - "DiffMamba - Checkpoints" model card, Model details: the backward
 *    layer is Mamba-2 applied to the flipped sequence.
 *  - The pages name Mamba-2 but do not print its recurrence; the scalar-
 *    decay-per-head selective SSM above is the standard Mamba-2 (SSD) form
 *    and is taken as the definition.
 *  - "Training Hybrid Block Diffusion Language Models with Partial
 *    Bidirectionality", Abstract and Methodology: in block diffusion the
 *    reverse scan is confined to the active block, so the cached state of
 *    the prefix is forward-only and reused exactly.
 *
 * Memory layouts (row-major, natural token order, all double):
 *   x     (batch, L, H, P)
 *   dt    (2, batch, L, H)        [0] = forward, [1] = reverse
 *   A     (2, H)
 *   B, C  (2, batch, L, G, N)
 *   D     (2, H)
 *   out   (batch, L, H, P)
 *   state (batch, H, P, N)        the forward state h, stored transposed
 *                                 (P rows of N) as the library stores it.
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* One direction of the recurrence for one (batch, head) unit.
 * reverse = 0 walks t = 0..L-1, reverse = 1 walks t = L-1..0.
 * h (N*P, row n holds the P values h[n][.]) holds the starting state and is
 * left holding the final state. y (L*P) receives C_t^T h_t for every t and is
 * accumulated into (y += ...), so both directions can share one buffer.
 * Strides are in elements: x_ts = stride between tokens of x, bc_ts = stride
 * between tokens of B/C, dt_ts = stride between tokens of dt. */
static void scan_one_direction(int reverse, int L, int P, int N,
                               const double *x, ptrdiff_t x_ts,
                               const double *dt, ptrdiff_t dt_ts, double A,
                               const double *Bm, const double *Cm, ptrdiff_t bc_ts,
                               double *h, double *y /* L*P, may be NULL */)
{
    for (int step = 0; step < L; ++step) {
        int t = reverse ? (L - 1 - step) : step;
        const double *xt = x + (ptrdiff_t)t * x_ts;
        const double *Bt = Bm + (ptrdiff_t)t * bc_ts;
        const double dtt = dt[(ptrdiff_t)t * dt_ts];
        const double decay = exp(dtt * A);
        for (int n = 0; n < N; ++n) {
            const double bn = dtt * Bt[n];
            double *hn = h + (size_t)n * P;
            for (int p = 0; p < P; ++p)
                hn[p] = decay * hn[p] + bn * xt[p];
        }
        if (y) {
            const double *Ct = Cm + (ptrdiff_t)t * bc_ts;
            double *yt = y + (size_t)t * P;
            for (int p = 0; p < P; ++p) {
                double acc = 0.0;
                for (int n = 0; n < N; ++n)
                    acc += Ct[n] * h[(size_t)n * P + p];
                yt[p] += acc;
            }
        }
    }
}

static int set_threads(int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
    return omp_get_max_threads();
#else
    (void)nthreads;
    return 1;
#endif
}

int ssd_oracle_threads(int nthreads) { return set_threads(nthreads); }

/* Full bidirectional mixer over whole sequences.
 * units: optional list of n_units (b, h) pairs packed as b*H + h; when NULL
 * every unit is computed. Outputs of units not in the list are left as they
 * are, so a caller can check a sample of a large problem. */
int ssd_oracle_bidir(const double *x, const double *dt, const double *A,
                     const double *Bm, const double *Cm, const double *D,
                     double *out, int batch, int L, int H, int P, int N, int G,
                     const int *units, int n_units, int nthreads)
{
    if (batch < 0 || L < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || H % G) return -1;
    set_threads(nthreads);
    const int total = units ? n_units : batch * H;
    const int hpg = H / G;
    const ptrdiff_t x_ts = (ptrdiff_t)H * P, dt_ts = H, bc_ts = (ptrdiff_t)G * N;
    const size_t dt_dir = (size_t)batch * L * H;          /* dt direction stride */
    const size_t bc_dir = (size_t)batch * L * G * N;      /* B/C direction stride */
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int i = 0; i < total; ++i) {
        const int u = units ? units[i] : i;
        const int b = u / H, hh = u % H, g = hh / hpg;
        if (b < 0 || b >= batch) { bad |= 1; continue; }
        double *h = (double *)calloc((size_t)N * P, sizeof(double));
        double *y = (double *)calloc((size_t)L * P + 1, sizeof(double));
        if (!h || !y) { free(h); free(y); bad |= 1; continue; }
        const double *xu = x + ((size_t)b * L * H + hh) * P;
        for (int d = 0; d < 2; ++d) {
            memset(h, 0, sizeof(double) * (size_t)N * P);
            const double *dtu = dt + d * dt_dir + (size_t)b * L * H + hh;
            const double *Bu = Bm + d * bc_dir + ((size_t)b * L * G + g) * N;
            const double *Cu = Cm + d * bc_dir + ((size_t)b * L * G + g) * N;
            scan_one_direction(d, L, P, N, xu, x_ts, dtu, dt_ts, A[d * H + hh], Bu, Cu, bc_ts, h, y);
        }
        const double dsum = D[hh] + D[H + hh];
        for (int t = 0; t < L; ++t) {
            double *o = out + ((size_t)b * L * H + (size_t)t * H + hh) * P;
            const double *xt = xu + (size_t)t * x_ts;
            for (int p = 0; p < P; ++p) o[p] = y[(size_t)t * P + p] + dsum * xt[p];
        }
        free(h);
        free(y);
    }
    return bad ? -1 : 0;
}

/* Forward-only state after the last token of each sequence.
 * dt (batch, L, H), A (H), B (batch, L, G, N) are the forward direction's.
 * init (batch, H, P, N) may be NULL (zero start). state_out (batch, H, P, N). */
int ssd_oracle_prefix_state(const double *x, const double *dt, const double *A,
                            const double *Bm, const double *init, double *state_out,
                            int batch, int L, int H, int P, int N, int G, int nthreads)
{
    if (batch < 0 || L < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || H % G) return -1;
    set_threads(nthreads);
    const int hpg = H / G;
    const ptrdiff_t x_ts = (ptrdiff_t)H * P, dt_ts = H, bc_ts = (ptrdiff_t)G * N;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int u = 0; u < batch * H; ++u) {
        const int b = u / H, hh = u % H, g = hh / hpg;
        double *h = (double *)malloc(sizeof(double) * (size_t)N * P);
        if (!h) { bad |= 1; continue; }
        double *so = state_out + (size_t)u * P * N;
        for (int n = 0; n < N; ++n)
            for (int p = 0; p < P; ++p)
                h[(size_t)n * P + p] = init ? init[(size_t)u * P * N + (size_t)p * N + n] : 0.0;
        scan_one_direction(0, L, P, N, x + ((size_t)b * L * H + hh) * P, x_ts,
                           dt + (size_t)b * L * H + hh, dt_ts, A[hh],
                           Bm + ((size_t)b * L * G + g) * N, NULL, bc_ts, h, NULL);
        for (int n = 0; n < N; ++n)
            for (int p = 0; p < P; ++p) so[(size_t)p * N + n] = h[(size_t)n * P + p];
        free(h);
    }
    return bad ? -1 : 0;
}

/* One denoising step on the active block of T tokens: the forward scan starts
 * from the cached prefix state, the reverse scan starts from zero at the
 * block's right end and sees only the block; then the D terms.
 * Layouts as for ssd_oracle_bidir with L = T; prefix (batch, H, P, N) is
 * only read. */
int ssd_oracle_block_step(const double *x, const double *dt, const double *A,
                          const double *Bm, const double *Cm, const double *D,
                          const double *prefix, double *out,
                          int batch, int T, int H, int P, int N, int G, int nthreads)
{
    if (batch < 0 || T < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || H % G) return -1;
    set_threads(nthreads);
    const int hpg = H / G;
    const ptrdiff_t x_ts = (ptrdiff_t)H * P, dt_ts = H, bc_ts = (ptrdiff_t)G * N;
    const size_t dt_dir = (size_t)batch * T * H;
    const size_t bc_dir = (size_t)batch * T * G * N;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int u = 0; u < batch * H; ++u) {
        const int b = u / H, hh = u % H, g = hh / hpg;
        double *h = (double *)malloc(sizeof(double) * (size_t)N * P);
        double *y = (double *)calloc((size_t)T * P + 1, sizeof(double));
        if (!h || !y) { free(h); free(y); bad |= 1; continue; }
        const double *xu = x + ((size_t)b * T * H + hh) * P;
        for (int d = 0; d < 2; ++d) {
            for (int n = 0; n < N; ++n)
                for (int p = 0; p < P; ++p)
                    h[(size_t)n * P + p] = (d == 0 && prefix) ? prefix[(size_t)u * P * N + (size_t)p * N + n] : 0.0;
            scan_one_direction(d, T, P, N, xu, x_ts, dt + d * dt_dir + (size_t)b * T * H + hh, dt_ts,
                               A[d * H + hh], Bm + d * bc_dir + ((size_t)b * T * G + g) * N,
                               Cm + d * bc_dir + ((size_t)b * T * G + g) * N, bc_ts, h, y);
        }
        const double dsum = D[hh] + D[H + hh];
        for (int t = 0; t < T; ++t) {
            double *o = out + ((size_t)b * T * H + (size_t)t * H + hh) * P;
            const double *xt = xu + (size_t)t * x_ts;
            for (int p = 0; p < P; ++p) o[p] = y[(size_t)t * P + p] + dsum * xt[p];
        }
        free(h);
        free(y);
    }
    return bad ? -1 : 0;
}

/* Both scans over a sequence with given starting states: the forward scan
 * from `prefix` (the forward state before the first token), the reverse scan
 * from `suffix` (the reverse state after the last token); then the D terms.
 * This is the mixer over one segment of a longer sequence when prefix and
 * suffix are the states the tokens outside the segment leave: the recurrence
 * is the same one as in ssd_oracle_bidir, only its starting states differ.
 * Layouts as for ssd_oracle_bidir; prefix and suffix (batch, H, P, N), each
 * may be NULL (zero). */
int ssd_oracle_bidir_seeded(const double *x, const double *dt, const double *A,
                            const double *Bm, const double *Cm, const double *D,
                            const double *prefix, const double *suffix, double *out,
                            int batch, int L, int H, int P, int N, int G, int nthreads)
{
    if (batch < 0 || L < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || H % G) return -1;
    set_threads(nthreads);
    const int hpg = H / G;
    const ptrdiff_t x_ts = (ptrdiff_t)H * P, dt_ts = H, bc_ts = (ptrdiff_t)G * N;
    const size_t dt_dir = (size_t)batch * L * H;
    const size_t bc_dir = (size_t)batch * L * G * N;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int u = 0; u < batch * H; ++u) {
        const int b = u / H, hh = u % H, g = hh / hpg;
        double *h = (double *)malloc(sizeof(double) * (size_t)N * P);
        double *y = (double *)calloc((size_t)L * P + 1, sizeof(double));
        if (!h || !y) { free(h); free(y); bad |= 1; continue; }
        const double *xu = x + ((size_t)b * L * H + hh) * P;
        for (int d = 0; d < 2; ++d) {
            const double *start = d == 0 ? prefix : suffix;
            for (int n = 0; n < N; ++n)
                for (int p = 0; p < P; ++p)
                    h[(size_t)n * P + p] = start ? start[(size_t)u * P * N + (size_t)p * N + n] : 0.0;
            scan_one_direction(d, L, P, N, xu, x_ts, dt + d * dt_dir + (size_t)b * L * H + hh, dt_ts,
                               A[d * H + hh], Bm + d * bc_dir + ((size_t)b * L * G + g) * N,
                               Cm + d * bc_dir + ((size_t)b * L * G + g) * N, bc_ts, h, y);
        }
        const double dsum = D[hh] + D[H + hh];
        for (int t = 0; t < L; ++t) {
            double *o = out + ((size_t)b * L * H + (size_t)t * H + hh) * P;
            const double *xt = xu + (size_t)t * x_ts;
            for (int p = 0; p < P; ++p) o[p] = y[(size_t)t * P + p] + dsum * xt[p];
        }
        free(h);
        free(y);
    }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------ gradients
 * Gradients of the scalar sum_t <dy_t, y_t> over the bidirectional mixer's
 * inputs (the backward pass a training step of the mixer runs; "Training
 * Hybrid Block Diffusion Language Models with Partial Bidirectionality", Key
 * Results and Technical Contribution: the models are trained through the
 * mixer with a full-block objective).
 *
 * Written from the recurrence above by reverse-mode differentiation, one
 * token after the other in the opposite order of each direction's scan. With
 * a_t = exp(dt_t A), h_t = a_t h_{t-1} + dt_t B_t x_t^T, y_t = C_t^T h_t, and
 * g_t the adjoint of h_t (the derivative of the scalar with respect to h_t,
 * all later tokens included):
 *   g_t        = C_t dy_t^T + a_{t+1} g_{t+1}            (N x P)
 *   dC_t[n]   += sum_p h_t[n][p] dy_t[p]
 *   dx_t[p]   += dt_t sum_n B_t[n] g_t[n][p]
 *   dB_t[n]   += dt_t sum_p g_t[n][p] x_t[p]
 *   ddt_t     += sum_{n,p} g_t[n][p] B_t[n] x_t[p] + A a_t <g_t, h_{t-1}>
 *   dA        += dt_t a_t <g_t, h_{t-1}>
 * and from the skip term y_t += (D_f + D_b) x_t: dx_t += (D_f + D_b) dy_t,
 * dD_f = dD_b = sum_t <dy_t, x_t>. "Later" means later in the direction's
 * own order (t + 1 forward, t - 1 reverse). Every forward state is kept (L + 1
 * states of N x P doubles per unit), so this is for small problems and
 * sampled units.
 *
 * Layouts as for ssd_oracle_bidir; dy and dx (batch, L, H, P); ddt (2, batch,
 * L, H); dA, dD (2, H); dB, dC (2, batch, L, G, N). Every output is
 * overwritten. Heads of a B/C group add into the same dB, dC entries, so the
 * work is split by (batch, group) with the group's heads in order.
 *
 * ssd_oracle_bidir_bwd_seeded is the same for ssd_oracle_bidir_seeded's
 * scans: the forward one starts from `prefix`, the reverse one from `suffix`
 * ((batch, H, P, N) each, NULL for zero), which enter as the state before
 * each direction's first token; the gradients with respect to them,
 * dprefix and dsuffix (NULL to skip), are the adjoint of that state:
 * a_first g_first, the first token's decay times its state's adjoint. With
 * suffix NULL this is the backward pass of the block step. */
int ssd_oracle_bidir_bwd_seeded(const double *x, const double *dt, const double *A,
                                const double *Bm, const double *Cm, const double *D,
                                const double *prefix, const double *suffix,
                                const double *dy, double *dx, double *ddt, double *dA,
                                double *dB, double *dC, double *dD, double *dprefix, double *dsuffix,
                                int batch, int L, int H, int P, int N, int G, int nthreads)
{
    if (batch < 0 || L < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || H % G) return -1;
    set_threads(nthreads);
    const int hpg = H / G;
    const ptrdiff_t x_ts = (ptrdiff_t)H * P, dt_ts = H, bc_ts = (ptrdiff_t)G * N;
    const size_t dt_dir = (size_t)batch * L * H;
    const size_t bc_dir = (size_t)batch * L * G * N;
    memset(dx, 0, sizeof(double) * (size_t)batch * L * H * P);
    memset(ddt, 0, sizeof(double) * 2 * dt_dir);
    memset(dB, 0, sizeof(double) * 2 * bc_dir);
    memset(dC, 0, sizeof(double) * 2 * bc_dir);
    /* per batch element, summed in order afterwards */
    double *dA_b = (double *)calloc((size_t)batch * 2 * H + 1, sizeof(double));
    double *dD_b = (double *)calloc((size_t)batch * H + 1, sizeof(double));
    if (!dA_b || !dD_b) { free(dA_b); free(dD_b); return -1; }
    const size_t SN = (size_t)N * P;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int bg = 0; bg < batch * G; ++bg) {
        const int b = bg / G, g = bg % G;
        double *hs = (double *)malloc(sizeof(double) * SN * ((size_t)L + 1));
        double *gadj = (double *)malloc(sizeof(double) * SN);
        if (!hs || !gadj) { free(hs); free(gadj); bad |= 1; continue; }
        for (int hh = g * hpg; hh < (g + 1) * hpg; ++hh) {
            const double *xu = x + ((size_t)b * L * H + hh) * P;
            const double *dyu = dy + ((size_t)b * L * H + hh) * P;
            double *dxu = dx + ((size_t)b * L * H + hh) * P;
            for (int d = 0; d < 2; ++d) {
                const double Ad = A[d * H + hh];
                const double *dtu = dt + d * dt_dir + (size_t)b * L * H + hh;
                double *ddtu = ddt + d * dt_dir + (size_t)b * L * H + hh;
                const double *Bu = Bm + d * bc_dir + ((size_t)b * L * G + g) * N;
                const double *Cu = Cm + d * bc_dir + ((size_t)b * L * G + g) * N;
                double *dBu = dB + d * bc_dir + ((size_t)b * L * G + g) * N;
                double *dCu = dC + d * bc_dir + ((size_t)b * L * G + g) * N;
                /* forward through the direction's order: hs[k] is the state after k tokens,
                   hs[0] the given start state (its (P, N) layout transposed) or zero */
                const double *init = d ? suffix : prefix;
                if (init) {
                    const double *iu = init + ((size_t)b * H + hh) * P * N;
                    for (int n = 0; n < N; ++n)
                        for (int p = 0; p < P; ++p) hs[(size_t)n * P + p] = iu[(size_t)p * N + n];
                } else {
                    memset(hs, 0, sizeof(double) * SN);
                }
                for (int k = 0; k < L; ++k) {
                    const int t = d ? (L - 1 - k) : k;
                    const double dtt = dtu[(ptrdiff_t)t * dt_ts];
                    const double a = exp(dtt * Ad);
                    const double *Bt = Bu + (ptrdiff_t)t * bc_ts;
                    const double *xt = xu + (ptrdiff_t)t * x_ts;
                    const double *hp = hs + (size_t)k * SN;
                    double *hn = hs + (size_t)(k + 1) * SN;
                    for (int n = 0; n < N; ++n)
                        for (int p = 0; p < P; ++p)
                            hn[(size_t)n * P + p] = a * hp[(size_t)n * P + p] + dtt * Bt[n] * xt[p];
                }
                /* adjoint, in the opposite order */
                memset(gadj, 0, sizeof(double) * SN);
                double dA_acc = 0.0;
                for (int k = L - 1; k >= 0; --k) {
                    const int t = d ? (L - 1 - k) : k;
                    const double dtt = dtu[(ptrdiff_t)t * dt_ts];
                    const double a = exp(dtt * Ad);
                    const double *Bt = Bu + (ptrdiff_t)t * bc_ts;
                    const double *Ct = Cu + (ptrdiff_t)t * bc_ts;
                    const double *xt = xu + (ptrdiff_t)t * x_ts;
                    const double *dyt = dyu + (ptrdiff_t)t * x_ts;
                    const double *ht = hs + (size_t)(k + 1) * SN;
                    const double *hp = hs + (size_t)k * SN;
                    double *dxt = dxu + (ptrdiff_t)t * x_ts;
                    /* g_t = C_t dy_t^T + (the decayed adjoint of the later token) */
                    for (int n = 0; n < N; ++n)
                        for (int p = 0; p < P; ++p) gadj[(size_t)n * P + p] += Ct[n] * dyt[p];
                    for (int n = 0; n < N; ++n) {
                        double s = 0.0;
                        for (int p = 0; p < P; ++p) s += ht[(size_t)n * P + p] * dyt[p];
                        dCu[(ptrdiff_t)t * bc_ts + n] += s;
                    }
                    for (int p = 0; p < P; ++p) {
                        double s = 0.0;
                        for (int n = 0; n < N; ++n) s += Bt[n] * gadj[(size_t)n * P + p];
                        dxt[p] += dtt * s;
                    }
                    double gbx = 0.0, ghp = 0.0;
                    for (int n = 0; n < N; ++n) {
                        double s = 0.0;
                        for (int p = 0; p < P; ++p) {
                            s += gadj[(size_t)n * P + p] * xt[p];
                            ghp += gadj[(size_t)n * P + p] * hp[(size_t)n * P + p];
                        }
                        dBu[(ptrdiff_t)t * bc_ts + n] += dtt * s;
                        gbx += Bt[n] * s;
                    }
                    ddtu[(ptrdiff_t)t * dt_ts] = gbx + Ad * a * ghp;
                    dA_acc += dtt * a * ghp;
                    for (size_t q = 0; q < SN; ++q) gadj[q] *= a;   /* adjoint of h_{t-1}'s share */
                }
                dA_b[(size_t)b * 2 * H + d * H + hh] = dA_acc;
                /* the start state's adjoint: what is left after the first token */
                double *dinit = d ? dsuffix : dprefix;
                if (dinit) {
                    double *du = dinit + ((size_t)b * H + hh) * P * N;
                    for (int n = 0; n < N; ++n)
                        for (int p = 0; p < P; ++p) du[(size_t)p * N + n] = L > 0 ? gadj[(size_t)n * P + p] : 0.0;
                }
            }
            /* skip term */
            const double dsum = D[hh] + D[H + hh];
            double xdy = 0.0;
            for (int t = 0; t < L; ++t)
                for (int p = 0; p < P; ++p) {
                    dxu[(ptrdiff_t)t * x_ts + p] += dsum * dyu[(ptrdiff_t)t * x_ts + p];
                    xdy += xu[(ptrdiff_t)t * x_ts + p] * dyu[(ptrdiff_t)t * x_ts + p];
                }
            dD_b[(size_t)b * H + hh] = xdy;
        }
        free(hs);
        free(gadj);
    }
    for (int d = 0; d < 2; ++d)
        for (int hh = 0; hh < H; ++hh) {
            double sa = 0.0, sd = 0.0;
            for (int b = 0; b < batch; ++b) {
                sa += dA_b[(size_t)b * 2 * H + d * H + hh];
                sd += dD_b[(size_t)b * H + hh];
            }
            dA[d * H + hh] = sa;
            dD[d * H + hh] = sd;
        }
    free(dA_b);
    free(dD_b);
    return bad ? -1 : 0;
}

int ssd_oracle_bidir_bwd(const double *x, const double *dt, const double *A,
                         const double *Bm, const double *Cm, const double *D,
                         const double *dy, double *dx, double *ddt, double *dA,
                         double *dB, double *dC, double *dD,
                         int batch, int L, int H, int P, int N, int G, int nthreads)
{
    return ssd_oracle_bidir_bwd_seeded(x, dt, A, Bm, Cm, D, NULL, NULL, dy, dx, ddt, dA, dB, dC, dD, NULL, NULL,
                                       batch, L, H, P, N, G, nthreads);
}
