/*
 * kda_oracle.c -- plain fp64 CPU oracle of the recurrent Kimi Delta Attention
 * (KDA) decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test suite, the smoke check of the package entry
 * file and the CPU-baseline leg of the benchmark use it.  It shares no code,
 * header, table or helper with the CUDA library; the two meet only through
 * the seeded input generators.
 *
 * What it computes (one value head h of one sequence n, tokens t = 0..T-1,
 * state S[K][V] held in double):
 *
 *   S      <- Diag(exp(g_t)) S                  per-key-channel decay
 *   u      <- beta_t (v_t - S^T k_t)            delta-rule correction
 *   S      <- S + k_t u^T                       rank-1 write
 *   o_t    <- scale S^T q_t                     readout from the updated S
 *   [gated variant]
 *   y_t    <- o_t / sqrt(mean_v(o_t^2) + eps) * w * sigmoid(z_t)
 *
 * Sources (pages by title; none of them prints the recurrence as a formula,
 * so the order above is the plainest reading consistent with all of them):
 *  - vLLM #57585 "Tune recurrent KDA launch configuration on SM90",
 *    section "Microbenchmark and earlier serving limits": BF16 q/k/v, FP32
 *    recurrent state, K = V = 128.
 *  - FlashInfer #4562 "feat(cake_kda): add optimized H12 packed decode across
 *    SM100 family", sequence diagram ("update state and write output"), the
 *    binding's kernel launch (slot table `state_indices`, scale literal
 *    0.08838834764831845 = 1/sqrt(128)) and the PR description (inactive
 *    graph-padding rows, indexed recurrent state).
 *  - b12x #249 "feat(gdn): add direct single-token KDA decode", sequence
 *    diagram: the KDA kernel updates the recurrent state and decodes the
 *    token, then an RMSNorm kernel normalises and gates the decoded output
 *    with z.
 *
 * Readings where the pages are silent:
 *  - decay is applied before the delta correction, and the correction uses
 *    the decayed state; the readout uses the state after the rank-1 write;
 *  - the RMS norm runs over V per (n, t, h) with eps inside the square root,
 *    weight w[V] is shared by all heads, the gate is sigmoid(z);
 *  - a negative slot index marks an inactive (graph-padding) row: its output
 *    is zero and the pool is not read or written;
 *  - bf16 inputs are widened exactly (bits << 16) and every step runs in
 *    double; outputs are left unrounded;
 *  - a bf16 state pool (FlashInfer #4562 keeps the recurrent state in bf16)
 *    is widened exactly on entry, the steps run in double as above, and the
 *    state is rounded to bf16 (nearest, ties to even) once, when the call
 *    writes it back.
 *
 * The oracle is written as loops in the order of the steps above.  It uses
 * no blocking, no fusion and no algebraic shortcut (in particular it computes
 * S^T q from the updated state, not through an identity).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* Exact bf16 -> double: a bf16 value is the top half of an IEEE binary32. */
static double bf16_to_double(uint16_t bits)
{
    uint32_t w = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

/*
 * One (n, h) unit.  Arguments point at the unit's data:
 *   q, k   : bf16 rows for token t at q + t*q_tstride (K entries each)
 *   v      : bf16 rows at v + t*v_tstride (V entries)
 *   g      : log-decay rows at g + t*g_tstride (K entries)
 *   beta   : scalars at beta + t*beta_tstride
 *   z      : bf16 gate rows (gated variant only, else NULL)
 *   w      : bf16 norm weight [V] (gated variant only, else NULL)
 *   S      : double state [K][V], row-major, updated in place (NULL = inactive)
 *   out    : double rows at out + t*out_tstride (V entries)
 */
static void kda_oracle_unit(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                            const double *g, const double *beta, const uint16_t *z,
                            const uint16_t *w, double *S, double *out,
                            int64_t T, int64_t K, int64_t V,
                            int64_t q_tstride, int64_t v_tstride, int64_t g_tstride,
                            int64_t beta_tstride, int64_t out_tstride,
                            double scale, double eps, double *rk, double *u)
{
    for (int64_t t = 0; t < T; ++t) {
        const uint16_t *qt = q + t * q_tstride;
        const uint16_t *kt = k + t * q_tstride;
        const uint16_t *vt = v + t * v_tstride;
        const double *gt = g + t * g_tstride;
        const double bt = beta[t * beta_tstride];
        double *ot = out + t * out_tstride;

        if (S == NULL) { /* inactive row */
            for (int64_t j = 0; j < V; ++j) ot[j] = 0.0;
            continue;
        }

        /* 1. decay: S[i][j] *= exp(g[i]) */
        for (int64_t i = 0; i < K; ++i) {
            const double d = exp(gt[i]);
            for (int64_t j = 0; j < V; ++j) S[i * V + j] *= d;
        }
        /* 2. rk = S^T k */
        for (int64_t j = 0; j < V; ++j) {
            double acc = 0.0;
            for (int64_t i = 0; i < K; ++i) acc += S[i * V + j] * bf16_to_double(kt[i]);
            rk[j] = acc;
        }
        /* 3. u = beta (v - rk) */
        for (int64_t j = 0; j < V; ++j) u[j] = bt * (bf16_to_double(vt[j]) - rk[j]);
        /* 4. S += k u^T */
        for (int64_t i = 0; i < K; ++i) {
            const double ki = bf16_to_double(kt[i]);
            for (int64_t j = 0; j < V; ++j) S[i * V + j] += ki * u[j];
        }
        /* 5. o = scale S^T q, from the updated state */
        for (int64_t j = 0; j < V; ++j) {
            double acc = 0.0;
            for (int64_t i = 0; i < K; ++i) acc += S[i * V + j] * bf16_to_double(qt[i]);
            ot[j] = scale * acc;
        }
        /* 6. optional gated RMS norm over V */
        if (z != NULL) {
            const uint16_t *zt = z + t * v_tstride;
            double ss = 0.0;
            for (int64_t j = 0; j < V; ++j) ss += ot[j] * ot[j];
            const double inv_rms = 1.0 / sqrt(ss / (double)V + eps);
            for (int64_t j = 0; j < V; ++j) {
                const double gate = 1.0 / (1.0 + exp(-bf16_to_double(zt[j])));
                ot[j] = ot[j] * inv_rms * bf16_to_double(w[j]) * gate;
            }
        }
    }
}

/*
 * Whole-call oracle over the units u = n*HV + h with unit_begin <= u < unit_end.
 *
 * Layouts (all contiguous, row-major):
 *   q, k  bf16 bits [N, T, HV, K]      v, z  bf16 bits [N, T, HV, V]
 *   g     double    [N, T, HV, K]      beta  double    [N, T, HV]
 *   state double    [num_slots, HV, K, V] (updated in place)
 *   slot_idx int32  [N]               out   double    [N, T, HV, V]
 *   w     bf16 bits [V]
 * z and w are NULL for the plain decode, both non-NULL for the gated one.
 * rk_scratch and u_scratch hold V doubles each, private to the caller.
 *
 * Returns 0 on success, -1 if an active slot index is >= num_slots or a size
 * is negative.  Units of rows whose slot is negative get zero output.
 */
int kda_oracle_decode_units(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                            const double *g, const double *beta, const uint16_t *z,
                            const uint16_t *w, double *state, int64_t num_slots,
                            const int32_t *slot_idx, double *out,
                            int64_t N, int64_t T, int64_t HV, int64_t K, int64_t V,
                            double scale, double eps, int64_t unit_begin, int64_t unit_end,
                            double *rk_scratch, double *u_scratch)
{
    if (N < 0 || T < 0 || HV <= 0 || K <= 0 || V <= 0) return -1;
    if (unit_begin < 0) unit_begin = 0;
    if (unit_end > N * HV) unit_end = N * HV;
    for (int64_t unit = unit_begin; unit < unit_end; ++unit) {
        const int64_t n = unit / HV;
        const int64_t h = unit % HV;
        const int32_t slot = slot_idx[n];
        if (slot >= num_slots) return -1;
        double *S = slot < 0 ? NULL : state + (((int64_t)slot * HV + h) * K * V);
        kda_oracle_unit(q + (n * T * HV + h) * K, k + (n * T * HV + h) * K,
                        v + (n * T * HV + h) * V, g + (n * T * HV + h) * K,
                        beta + (n * T * HV + h), z ? z + (n * T * HV + h) * V : NULL, w, S,
                        out + (n * T * HV + h) * V, T, K, V,
                        /*q_tstride=*/HV * K, /*v_tstride=*/HV * V, /*g_tstride=*/HV * K,
                        /*beta_tstride=*/HV, /*out_tstride=*/HV * V, scale, eps,
                        rk_scratch, u_scratch);
    }
    return 0;
}

/*
 * Round doubles to bf16 (round to nearest, ties to even), as the bf16-state
 * variant does when it writes the state back at the end of a call.  Returns
 * the bf16 bit patterns.  Written from the format's definition: 8 significant
 * bits, exponent range of binary32 (normal down to 2^-126, subnormal steps of
 * 2^-133), overflow to infinity past the largest finite value.
 */
static uint16_t double_to_bf16_rne(double x)
{
    if (isnan(x)) return 0x7fc0;
    const uint16_t sign = signbit(x) ? 0x8000 : 0;
    const double a = fabs(x);
    if (a == 0.0) return sign;
    int e;
    const double m = frexp(a, &e); /* a = m 2^e, m in [0.5, 1): leading bit has weight 2^(e-1) */
    int lsb = (e - 1) - 7;         /* weight of the last kept bit for a normal bf16 */
    if (lsb < -133) lsb = -133;    /* subnormal spacing */
    const double q = nearbyint(ldexp(a, -lsb)); /* current rounding mode: to nearest, ties to even */
    const double y = ldexp(q, lsb);
    if (y > 3.38953138925153547590470800371487866880e38) return sign | 0x7f80; /* overflow */
    const float f = (float)y; /* exact: at most 8 significant bits inside the binary32 range */
    uint32_t w;
    memcpy(&w, &f, sizeof w);
    return sign | (uint16_t)(w >> 16);
}

void kda_oracle_round_bf16(const double *in, uint16_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = double_to_bf16_rne(in[i]);
}

/*
 * Gate and beta activations of the serving input form (raw bf16 gate and
 * beta, per-head A_log, per-head per-key-channel dt_bias):
 *   g[n,t,h,i]  = -exp(A_log[h]) * softplus(raw_gate[n,t,h,i] + dt_bias[h,i])
 *   beta[n,t,h] = sigmoid(raw_beta[n,t,h])
 * FlashInfer #4562's kernel launch takes raw_gate, raw_beta, A_log and
 * dt_bias and b12x #249 takes raw_g and raw_beta, but neither page prints the
 * activation: this formula is a reading (the usual one for KDA's gate), not
 * something the pages fix -- parity unpinned by the sources (the tests pin
 * only properties any softplus-style gate and logistic beta share).
 * softplus(x) = log(1 + e^x), evaluated as x + log1p(e^-x) for x > 0 so that
 * it neither overflows nor cancels.
 * Layouts: raw_gate bf16 [N*T, HV*K], raw_beta bf16 [N*T, HV] (dense),
 * A_log [HV], dt_bias [HV*K]; outputs g [N*T, HV*K], beta [N*T, HV].
 */
static double softplus(double x) { return x > 0.0 ? x + log1p(exp(-x)) : log1p(exp(x)); }

void kda_oracle_activate(const uint16_t *raw_gate, const float *A_log, const float *dt_bias,
                         const uint16_t *raw_beta, double *g, double *beta, int64_t rows,
                         int64_t HV, int64_t K)
{
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t h = 0; h < HV; ++h) {
            const double a = exp((double)A_log[h]);
            for (int64_t i = 0; i < K; ++i) {
                const int64_t e = (r * HV + h) * K + i;
                g[e] = -a * softplus(bf16_to_double(raw_gate[e]) + (double)dt_bias[h * K + i]);
            }
            beta[r * HV + h] = 1.0 / (1.0 + exp(-bf16_to_double(raw_beta[r * HV + h])));
        }
    }
}
