/*
 * oracle.c -- plain, slow CPU oracle for the element-wise recurrence scans.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path (the
 * CUDA library under scan_gated_rnns_b200/) never links, loads or calls it, and
 * the two share no code: no headers, no helpers, no constants.
 *
 * Everything here is written for a reader to check by eye against the method:
 *   - minGRU (the layer profiled on the page "Mingru Pytorch", sections
 *     "Requirements & limits" and "Install and apply the minGRU layer"): a
 *     gated recurrence over the time axis of a (B, T, D) tensor,
 *         z_t       = sigmoid(k_t)
 *         htilde_t  = g(hx_t),   g(x) = x + 0.5 for x >= 0, sigmoid(x) otherwise
 *         h_t       = (1 - z_t) * h_{t-1} + z_t * htilde_t,
 *     with an optional carried state h_0 (absent => h_0 = 0).  The page states
 *     that the implementation is the "log-space" numerically stable version;
 *     that version evaluates the same h_t as
 *         h_t = exp( a*_t + logcumsumexp_{s<=t}( log z_s + log htilde_s - a*_s ) ),
 *         a*_t = cumsum_{r<=t}( -softplus(k_r) ),
 *     where a carried h_0 > 0 joins the logcumsumexp as an s = 0 term log h_0
 *     with a*_0 = 0.  Two oracles are provided, one per formulation, so that
 *     each pins the other.
 *   - the MinMax neuron (page "MinMax Recurrent Neural Cascades", section
 *     "The model", item 3):  x_{t+1} = max(min(r_t, x_t), s_t), element-wise.
 *
 * Conventions (the pages are silent on them; these are the plainest readings):
 *   - layout (B, T, D) row-major, D fastest, like the page's torch.randn(2, 1024, 512);
 *   - output index t holds the state after consuming token t (T outputs; the
 *     carried initial state is not echoed);
 *   - optional initial states are (B, D) with a batch stride in elements;
 *   - all arithmetic is IEEE binary64; inputs given in fp32/bf16 are widened
 *     exactly by the caller.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>

/* ---------------------------------------------------------------- helpers */

/* logistic sigmoid, evaluated on the side where exp() cannot overflow */
static double sigmoid(double x)
{
    if (x >= 0.0) {
        return 1.0 / (1.0 + exp(-x));
    }
    double e = exp(x);
    return e / (1.0 + e);
}

/* minGRU candidate activation g */
static double g_act(double x)
{
    return (x >= 0.0) ? x + 0.5 : sigmoid(x);
}

/* softplus(x) = log(1 + e^x), without overflow */
static double softplus(double x)
{
    return fmax(x, 0.0) + log1p(exp(-fabs(x)));
}

/* --------------------------------------------------------- minGRU, linear */

/*
 * The recurrence h_t = (1 - z_t) h_{t-1} + z_t g(hx_t), sequentially in t,
 * for every channel (b, d); the state h_{t-1} is the previous output row.
 * 1 - z_t is written as sigmoid(-k_t), which is the same number without the
 * cancellation of 1 - sigmoid(k_t) when z_t is near 1.
 */
int oracle_mingru_linear(const double *k, const double *hx,
                         const double *h0, int64_t h0_bs,
                         double *h, int64_t B, int64_t T, int64_t D)
{
    if (B < 0 || T < 0 || D < 0) return 1;
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t t = 0; t < T; ++t) {
            for (int64_t d = 0; d < D; ++d) {
                int64_t i = (b * T + t) * D + d;
                double prev;
                if (t > 0) {
                    prev = h[i - D];
                } else {
                    prev = h0 ? h0[b * h0_bs + d] : 0.0;
                }
                double z = sigmoid(k[i]);
                double one_minus_z = sigmoid(-k[i]);
                h[i] = one_minus_z * prev + z * g_act(hx[i]);
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------ minGRU, log space */

/*
 * The log-space formula, term by term:
 *   log(1 - z_t)   = -softplus(k_t)           (accumulated into a*_t)
 *   log z_t        = -softplus(-k_t)
 *   log htilde_t   = log(hx_t + 0.5) if hx_t >= 0, else -softplus(-hx_t)
 *   v_s            = log z_s + log htilde_s - a*_s
 *   h_t            = exp(a*_t + logcumsumexp_{s<=t} v_s)
 * The running logcumsumexp is kept as (m, acc) with value m + log(acc), m the
 * running maximum, which is the usual overflow-free way to add exponentials.
 * A carried h0 contributes v_0 = log h0 (a*_0 = 0); it must be > 0.  Finite k
 * only: k = +-inf makes a*_t infinite and the formula undefined.
 * Per-channel running values (a*, m, acc) live in arrays over d so that the
 * loops walk the (B, T, D) arrays row by row.
 */
int oracle_mingru_log(const double *k, const double *hx,
                      const double *h0, int64_t h0_bs,
                      double *h, int64_t B, int64_t T, int64_t D)
{
    if (B < 0 || T < 0 || D < 0) return 1;
    if (D == 0) return 0;
    double *a_star = malloc(sizeof(double) * (size_t)D);
    double *m = malloc(sizeof(double) * (size_t)D);    /* running max of v_s */
    double *acc = malloc(sizeof(double) * (size_t)D);  /* sum of exp(v_s - m) */
    if (!a_star || !m || !acc) {
        free(a_star); free(m); free(acc);
        return 2;
    }
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t d = 0; d < D; ++d) {
            a_star[d] = 0.0;
            m[d] = -INFINITY;
            acc[d] = 0.0;
            if (h0) {
                m[d] = log(h0[b * h0_bs + d]);
                acc[d] = 1.0;
            }
        }
        for (int64_t t = 0; t < T; ++t) {
            for (int64_t d = 0; d < D; ++d) {
                int64_t i = (b * T + t) * D + d;
                a_star[d] += -softplus(k[i]);
                double log_z = -softplus(-k[i]);
                double x = hx[i];
                double log_ht = (x >= 0.0) ? log(x + 0.5) : -softplus(-x);
                double v = log_z + log_ht - a_star[d];
                if (v > m[d]) {
                    acc[d] = acc[d] * exp(m[d] - v) + 1.0;
                    m[d] = v;
                } else {
                    acc[d] += exp(v - m[d]);
                }
                h[i] = exp(a_star[d] + m[d] + log(acc[d]));
            }
        }
    }
    free(a_star); free(m); free(acc);
    return 0;
}

/* ------------------------------------------------------------- MinMax */

/*
 * x_{t+1} = max(min(r_t, x_t), s_t), sequentially in t, for every channel;
 * out[t] = x_{t+1} and the state x_t is the previous output row.  x0 absent
 * => +0.  min/max only select one of their operands, so the result is
 * exactly one of the input values whatever the working precision.
 */
int oracle_minmax(const double *r, const double *s,
                  const double *x0, int64_t x0_bs,
                  double *x, int64_t B, int64_t T, int64_t D)
{
    if (B < 0 || T < 0 || D < 0) return 1;
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t t = 0; t < T; ++t) {
            for (int64_t d = 0; d < D; ++d) {
                int64_t i = (b * T + t) * D + d;
                double state;
                if (t > 0) {
                    state = x[i - D];
                } else {
                    state = x0 ? x0[b * x0_bs + d] : 0.0;
                }
                x[i] = fmax(fmin(r[i], state), s[i]);
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------ gradients */

/*
 * Reverse mode through the same recurrences, for a loss L whose gradient
 * with respect to every output row is given: gy[b, t, d] = dL/d out[b, t, d].
 * The pages name training with bounded gradients as a property of the
 * MinMax model (page "MinMax Recurrent Neural Cascades", Key properties) and
 * show the minGRU layer as a trainable torch module (page "Mingru
 * Pytorch"); neither prints the derivative, so it is taken here from the
 * chain rule through the sequential loop, channel by channel:
 *   lam       = dL/d state_t flowing back from steps after t (0 after the last)
 *   delta_t   = gy_t + lam                           (total dL/d out_t)
 *   d input_t = delta_t * d out_t / d input_t
 *   lam       = delta_t * d out_t / d state_{t-1}     (moves one step back)
 * and after t = 0, lam is the gradient with respect to the initial state.
 * The forward states are recomputed here in fp64; dinit may be NULL.
 */

/*
 * minGRU: out_t = h_t = (1 - z_t) h_{t-1} + z_t g(hx_t), z_t = sigmoid(k_t).
 *   dh_t/dk_t     = z_t (1 - z_t) (g(hx_t) - h_{t-1})
 *                   (d sigmoid(k)/dk = z (1 - z), d (1 - z)/dk = -z (1 - z))
 *   dh_t/dhx_t    = z_t g'(hx_t),  g'(x) = 1 (x >= 0), sigmoid(x) sigmoid(-x) (x < 0)
 *   dh_t/dh_{t-1} = 1 - z_t
 */
int oracle_mingru_backward(const double *k, const double *hx,
                           const double *h0, int64_t h0_bs, const double *gy,
                           double *dk, double *dhx, double *dh0,
                           int64_t B, int64_t T, int64_t D)
{
    if (B < 0 || T < 0 || D < 0) return 1;
    double *h = malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    if (!h) return 2;
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t d = 0; d < D; ++d) {
            double init = h0 ? h0[b * h0_bs + d] : 0.0;
            /* forward, this channel only */
            double prev = init;
            for (int64_t t = 0; t < T; ++t) {
                int64_t i = (b * T + t) * D + d;
                prev = sigmoid(-k[i]) * prev + sigmoid(k[i]) * g_act(hx[i]);
                h[t] = prev;
            }
            /* backward */
            double lam = 0.0;
            for (int64_t t = T - 1; t >= 0; --t) {
                int64_t i = (b * T + t) * D + d;
                double delta = gy[i] + lam;
                double hprev = (t > 0) ? h[t - 1] : init;
                double z = sigmoid(k[i]);
                double one_minus_z = sigmoid(-k[i]);
                double x = hx[i];
                double g = g_act(x);
                double gprime = (x >= 0.0) ? 1.0 : sigmoid(x) * sigmoid(-x);
                dk[i] = delta * z * one_minus_z * (g - hprev);
                dhx[i] = delta * z * gprime;
                lam = delta * one_minus_z;
            }
            if (dh0) dh0[b * D + d] = lam;
        }
    }
    free(h);
    return 0;
}

/*
 * MinMax: out_t = x_{t+1} = max(m_t, s_t), m_t = min(r_t, x_t).  min and max
 * are differentiated the way PyTorch's elementwise minimum/maximum are: the
 * selected operand gets the whole gradient and equal operands share it
 * evenly (the plainest reading for a model trained with autograd; the pages
 * do not state a rule for ties).
 *   dm/dr = 1 if r < x, 1/2 if r == x, 0 if r > x;   dm/dx = 1 - dm/dr
 *   dout/dm = 1 if m > s, 1/2 if m == s, 0 if m < s;  dout/ds = 1 - dout/dm
 */
int oracle_minmax_backward(const double *r, const double *s,
                           const double *x0, int64_t x0_bs, const double *gy,
                           double *dr, double *ds, double *dx0,
                           int64_t B, int64_t T, int64_t D)
{
    if (B < 0 || T < 0 || D < 0) return 1;
    double *x = malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    if (!x) return 2;
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t d = 0; d < D; ++d) {
            double init = x0 ? x0[b * x0_bs + d] : 0.0;
            double state = init;
            for (int64_t t = 0; t < T; ++t) {
                int64_t i = (b * T + t) * D + d;
                state = fmax(fmin(r[i], state), s[i]);
                x[t] = state;
            }
            double lam = 0.0;
            for (int64_t t = T - 1; t >= 0; --t) {
                int64_t i = (b * T + t) * D + d;
                double delta = gy[i] + lam;
                double xprev = (t > 0) ? x[t - 1] : init;
                double m = fmin(r[i], xprev);
                double dm_dr = (r[i] < xprev) ? 1.0 : ((r[i] == xprev) ? 0.5 : 0.0);
                double dm_dx = 1.0 - dm_dr;
                double dout_dm = (m > s[i]) ? 1.0 : ((m == s[i]) ? 0.5 : 0.0);
                double dout_ds = 1.0 - dout_dm;
                dr[i] = delta * dout_dm * dm_dr;
                ds[i] = delta * dout_ds;
                lam = delta * dout_dm * dm_dx;
            }
            if (dx0) dx0[b * D + d] = lam;
        }
    }
    free(x);
    return 0;
}

/* ------------------------------------------------------ minGRU, time decay */

/*
 * Time decay (page "Your first delta model", Step 5: the decay contract every
 * mixer accepts): the carried state is gated once per token, at the token
 * boundary, before that token's own write lands undecayed,
 *     h <- gamma_t h,   gamma_t = exp(-lambda_d * u_{b,t}),
 * with u the gap preceding the token (delta_t), or log1p(delta_t) when gaps
 * are compressed (log1p_delta).  delta_t = 0 gives gamma = exp(0) = 1, no
 * decay.  A gap with lambda * u > 1e4 wipes the state completely (the page's
 * clamp; gamma = 0 exactly, with zero derivative).  For the minGRU's vector
 * state this reads
 *     h_t = (1 - z_t) gamma_t h_{t-1} + z_t g(hx_t).
 * delta_t is (B, T) with batch stride dt_bs; lambda is (D,), >= 0.
 */
static double decay_gate(double lam, double gap, int log1p_delta)
{
    double u = log1p_delta ? log1p(gap) : gap;
    double x = lam * u;
    return (x > 1e4) ? 0.0 : exp(-x);
}

/* d gamma / d lambda = -u gamma (0 where the clamp holds gamma at 0) */
static double decay_gate_dlam(double lam, double gap, int log1p_delta)
{
    double u = log1p_delta ? log1p(gap) : gap;
    double x = lam * u;
    return (x > 1e4) ? 0.0 : -u * exp(-x);
}

int oracle_mingru_decay(const double *k, const double *hx,
                        const double *h0, int64_t h0_bs,
                        const double *dt, int64_t dt_bs, const double *lam, int log1p_delta,
                        double *h, int64_t B, int64_t T, int64_t D)
{
    if (B < 0 || T < 0 || D < 0) return 1;
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t t = 0; t < T; ++t) {
            for (int64_t d = 0; d < D; ++d) {
                int64_t i = (b * T + t) * D + d;
                double prev;
                if (t > 0) {
                    prev = h[i - D];
                } else {
                    prev = h0 ? h0[b * h0_bs + d] : 0.0;
                }
                double gamma = decay_gate(lam[d], dt[b * dt_bs + t], log1p_delta);
                h[i] = sigmoid(-k[i]) * (gamma * prev) + sigmoid(k[i]) * g_act(hx[i]);
            }
        }
    }
    return 0;
}

/*
 * Gradients of the decayed recurrence for dL/dh = gy, as oracle_mingru_backward
 * plus the decay:
 *   dh_t/dk_t      = z (1 - z) (g - gamma h_{t-1})
 *   dh_t/dh_{t-1}  = (1 - z) gamma
 *   dL/dlambda_d   = sum over b, t of delta_t (1 - z_t) h_{t-1} dgamma_t/dlambda
 * dlam (D,) is overwritten with the sum over the whole batch; dh0, dlam may be NULL.
 */
int oracle_mingru_decay_backward(const double *k, const double *hx,
                                 const double *h0, int64_t h0_bs,
                                 const double *dt, int64_t dt_bs, const double *lam, int log1p_delta,
                                 const double *gy, double *dk, double *dhx, double *dh0, double *dlam,
                                 int64_t B, int64_t T, int64_t D)
{
    if (B < 0 || T < 0 || D < 0) return 1;
    double *h = malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    if (!h) return 2;
    if (dlam) {
        for (int64_t d = 0; d < D; ++d) dlam[d] = 0.0;
    }
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t d = 0; d < D; ++d) {
            double init = h0 ? h0[b * h0_bs + d] : 0.0;
            double prev = init;
            for (int64_t t = 0; t < T; ++t) {
                int64_t i = (b * T + t) * D + d;
                double gamma = decay_gate(lam[d], dt[b * dt_bs + t], log1p_delta);
                prev = sigmoid(-k[i]) * (gamma * prev) + sigmoid(k[i]) * g_act(hx[i]);
                h[t] = prev;
            }
            double back = 0.0;
            for (int64_t t = T - 1; t >= 0; --t) {
                int64_t i = (b * T + t) * D + d;
                double delta = gy[i] + back;
                double hprev = (t > 0) ? h[t - 1] : init;
                double gap = dt[b * dt_bs + t];
                double gamma = decay_gate(lam[d], gap, log1p_delta);
                double z = sigmoid(k[i]);
                double one_minus_z = sigmoid(-k[i]);
                double x = hx[i];
                double g = g_act(x);
                double gprime = (x >= 0.0) ? 1.0 : sigmoid(x) * sigmoid(-x);
                dk[i] = delta * z * one_minus_z * (g - gamma * hprev);
                dhx[i] = delta * z * gprime;
                if (dlam) dlam[d] += delta * one_minus_z * hprev * decay_gate_dlam(lam[d], gap, log1p_delta);
                back = delta * one_minus_z * gamma;
            }
            if (dh0) dh0[b * D + d] = back;
        }
    }
    free(h);
    return 0;
}
