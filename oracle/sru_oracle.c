/*
 * sru_oracle.c -- plain, slow, fp64 CPU oracle of the Simple Recurrent Unit layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may load this file or
 * its shared library: only the tests, the smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header, table or helper with the CUDA
 * library; it is built by its own gcc command (oracle/__init__.py).
 *
 * What it computes, and where the method is stated:
 *   "When Attention Meets Fast Recurrence: Training Language Models with Reduced
 *   Compute" (T. Lei), background section on SRU:
 *     - the unnumbered SRU cell (forget gate f, reset gate r, state c, highway
 *       output h) and its two code-level optimisations;
 *     - Eq. (1): the three input projections of all time steps grouped into one
 *       matrix product U^T = [W; W'; W''] X^T;
 *     - Eqs. (2)-(5): the element-wise recurrence driven by U, independent per
 *       hidden channel (and per batch row).
 *   The backward pass is not printed on the page; it is the plain reverse-mode
 *   derivative of Eqs. (2)-(5), taken step by step in reverse time order.
 *
 * Readings where the page is silent (all shared with the CUDA library's ABI):
 *   - gate blocks of U per token and direction are ordered [candidate | forget |
 *     reset] (the projection is written with [W; W_f; W_r], candidate first);
 *   - U is laid out (L, B, n_dir, 3, d), time-major, last index fastest;
 *   - a scalar alpha multiplies the highway input x in Eq. (5) (alpha = 1 is the
 *     page's form);
 *   - a padded position (mask = 1) leaves the state unchanged, writes h = 0 and
 *     receives zero gradient; the state gradient passes through it unchanged;
 *   - direction 1 of a bidirectional layer walks t = L-1 ... 0 with its own
 *     gate block of U, its own v, b and c0; both directions read the same x and
 *     the input gradient dx is the sum of both directions' highway terms.
 *
 * Every routine walks one (direction, batch row, channel) stream at a time, in
 * the order the equations are written, with no blocking, fusion or reordering.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* logistic sigma(z) = 1 / (1 + exp(-z)), the gate non-linearity of Eqs. (2)-(3). */
static double sigma(double z) { return 1.0 / (1.0 + exp(-z)); }

/* Flat index helpers for the layouts listed above. */
static int64_t ix_u(int64_t t, int64_t b, int64_t dir, int64_t g, int64_t j,
                    int64_t B, int64_t n_dir, int64_t d) {
    return (((t * B + b) * n_dir + dir) * 3 + g) * d + j;
}
static int64_t ix_h(int64_t t, int64_t b, int64_t dir, int64_t j,
                    int64_t B, int64_t n_dir, int64_t d) {
    return ((t * B + b) * n_dir + dir) * d + j;
}
static int64_t ix_x(int64_t t, int64_t b, int64_t j, int64_t B, int64_t d) {
    return (t * B + b) * d + j;
}
static int64_t ix_state(int64_t b, int64_t dir, int64_t j, int64_t n_dir, int64_t d) {
    return (b * n_dir + dir) * d + j;
}
/* v and b are (n_dir, 2, d): row 0 = forget-gate vector, row 1 = reset-gate vector. */
static int64_t ix_vec(int64_t dir, int64_t which, int64_t j, int64_t d) {
    return (dir * 2 + which) * d + j;
}

/* time index of processing step s in direction dir */
static int64_t step_time(int64_t s, int64_t dir, int64_t L) {
    return dir == 0 ? s : L - 1 - s;
}

/*
 * Forward, Eqs. (2)-(5).
 *   U    (L, B, n_dir, 3, d)   x (L, B, d)     v, bias (n_dir, 2, d)
 *   c0   (B, n_dir, d) or NULL (zero initial state)
 *   mask (L, B) bytes or NULL; 1 = padded position
 * Outputs: h (L, B, n_dir, d), cT (B, n_dir, d) = state after the last step.
 * Returns 0, or -1 on a bad size.
 */
int sru_oracle_forward(int64_t L, int64_t B, int64_t d, int64_t n_dir, double alpha,
                       const double* U, const double* x, const double* v,
                       const double* bias, const double* c0, const uint8_t* mask,
                       double* h, double* cT) {
    if (L < 0 || B < 0 || d < 0 || (n_dir != 1 && n_dir != 2)) return -1;
    for (int64_t dir = 0; dir < n_dir; ++dir)
        for (int64_t b = 0; b < B; ++b)
            for (int64_t j = 0; j < d; ++j) {
                const double vf = v[ix_vec(dir, 0, j, d)], vr = v[ix_vec(dir, 1, j, d)];
                const double bf = bias[ix_vec(dir, 0, j, d)], br = bias[ix_vec(dir, 1, j, d)];
                double c = c0 ? c0[ix_state(b, dir, j, n_dir, d)] : 0.0;
                for (int64_t s = 0; s < L; ++s) {
                    const int64_t t = step_time(s, dir, L);
                    const int64_t ho = ix_h(t, b, dir, j, B, n_dir, d);
                    if (mask && mask[t * B + b]) { h[ho] = 0.0; continue; }
                    const double u_c = U[ix_u(t, b, dir, 0, j, B, n_dir, d)];
                    const double u_f = U[ix_u(t, b, dir, 1, j, B, n_dir, d)];
                    const double u_r = U[ix_u(t, b, dir, 2, j, B, n_dir, d)];
                    const double f = sigma(u_f + vf * c + bf);            /* Eq. (2) */
                    const double r = sigma(u_r + vr * c + br);            /* Eq. (3) */
                    const double c_new = f * c + (1.0 - f) * u_c;         /* Eq. (4) */
                    h[ho] = r * c_new + (1.0 - r) * alpha * x[ix_x(t, b, j, B, d)]; /* Eq. (5) */
                    c = c_new;
                }
                cT[ix_state(b, dir, j, n_dir, d)] = c;
            }
    return 0;
}

/*
 * Backward: reverse-mode derivative of the forward above for the loss
 *   Loss = sum(dh * h) + sum(dcT * cT).
 * Inputs as the forward, plus dh (L, B, n_dir, d) and dcT (B, n_dir, d) or NULL.
 * Outputs (all overwritten):
 *   dU  (L, B, n_dir, 3, d)    gradient w.r.t. U (zero at padded positions)
 *   dx  (L, B, d)              highway part of dLoss/dx, summed over directions
 *   dv, dbias (n_dir, 2, d)    summed over t and b
 *   dc0 (B, n_dir, d)
 * Returns 0, -1 on a bad size, -2 if scratch memory cannot be allocated.
 */
int sru_oracle_backward(int64_t L, int64_t B, int64_t d, int64_t n_dir, double alpha,
                        const double* U, const double* x, const double* v,
                        const double* bias, const double* c0, const uint8_t* mask,
                        const double* dh, const double* dcT,
                        double* dU, double* dx, double* dv, double* dbias, double* dc0) {
    if (L < 0 || B < 0 || d < 0 || (n_dir != 1 && n_dir != 2)) return -1;
    double* c_prev = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double* c_now = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double* fs = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double* rs = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    if (!c_prev || !c_now || !fs || !rs) {
        free(c_prev); free(c_now); free(fs); free(rs);
        return -2;
    }
    for (int64_t i = 0; i < L * B * d; ++i) dx[i] = 0.0;
    for (int64_t i = 0; i < n_dir * 2 * d; ++i) { dv[i] = 0.0; dbias[i] = 0.0; }

    for (int64_t dir = 0; dir < n_dir; ++dir)
        for (int64_t b = 0; b < B; ++b)
            for (int64_t j = 0; j < d; ++j) {
                const double vf = v[ix_vec(dir, 0, j, d)], vr = v[ix_vec(dir, 1, j, d)];
                const double bf = bias[ix_vec(dir, 0, j, d)], br = bias[ix_vec(dir, 1, j, d)];
                /* forward again, keeping what the derivative needs */
                double c = c0 ? c0[ix_state(b, dir, j, n_dir, d)] : 0.0;
                for (int64_t s = 0; s < L; ++s) {
                    const int64_t t = step_time(s, dir, L);
                    c_prev[s] = c;
                    if (mask && mask[t * B + b]) { c_now[s] = c; fs[s] = rs[s] = 0.0; continue; }
                    const double u_c = U[ix_u(t, b, dir, 0, j, B, n_dir, d)];
                    const double u_f = U[ix_u(t, b, dir, 1, j, B, n_dir, d)];
                    const double u_r = U[ix_u(t, b, dir, 2, j, B, n_dir, d)];
                    fs[s] = sigma(u_f + vf * c + bf);
                    rs[s] = sigma(u_r + vr * c + br);
                    c = fs[s] * c + (1.0 - fs[s]) * u_c;
                    c_now[s] = c;
                }
                /* reverse time: g is dLoss/dc of the state leaving step s */
                double g = dcT ? dcT[ix_state(b, dir, j, n_dir, d)] : 0.0;
                double dvf = 0.0, dvr = 0.0, dbf = 0.0, dbr = 0.0;
                for (int64_t s = L - 1; s >= 0; --s) {
                    const int64_t t = step_time(s, dir, L);
                    const int64_t u0 = ix_u(t, b, dir, 0, j, B, n_dir, d);
                    const int64_t u1 = ix_u(t, b, dir, 1, j, B, n_dir, d);
                    const int64_t u2 = ix_u(t, b, dir, 2, j, B, n_dir, d);
                    if (mask && mask[t * B + b]) { dU[u0] = dU[u1] = dU[u2] = 0.0; continue; }
                    const double f = fs[s], r = rs[s], cp = c_prev[s], cn = c_now[s];
                    const double u_c = U[u0];
                    const double xv = x[ix_x(t, b, j, B, d)];
                    const double dhv = dh[ix_h(t, b, dir, j, B, n_dir, d)];
                    /* h = r*c + (1-r)*alpha*x */
                    const double G = g + dhv * r;                  /* total dLoss/dc[t] */
                    const double d_r = dhv * (cn - alpha * xv);
                    dx[ix_x(t, b, j, B, d)] += dhv * (1.0 - r) * alpha;
                    /* c = f*cp + (1-f)*u_c */
                    const double d_zf = G * (cp - u_c) * f * (1.0 - f);
                    const double d_zr = d_r * r * (1.0 - r);
                    dU[u0] = G * (1.0 - f);
                    dU[u1] = d_zf;
                    dU[u2] = d_zr;
                    dvf += d_zf * cp; dvr += d_zr * cp;
                    dbf += d_zf;      dbr += d_zr;
                    /* cp reaches the loss through f*cp and through both peepholes */
                    g = G * f + d_zf * vf + d_zr * vr;
                }
                dc0[ix_state(b, dir, j, n_dir, d)] = g;
                dv[ix_vec(dir, 0, j, d)] += dvf;    dv[ix_vec(dir, 1, j, d)] += dvr;
                dbias[ix_vec(dir, 0, j, d)] += dbf; dbias[ix_vec(dir, 1, j, d)] += dbr;
            }
    free(c_prev); free(c_now); free(fs); free(rs);
    return 0;
}

/* ---------------------------------------------------------------------------
 * Matrix products of Eq. (1) and of its gradients, as plain sums.
 *
 * out[r, c] = sum_k A(r, k) * Bm(c, k), where A(r, k) = A[r*a_rs + k*a_ks] and
 * Bm(c, k) = Bm[c*b_rs + k*b_ks].  Operands are read in their storage type and
 * widened exactly to double: dtype 0 = fp32, 1 = bf16 (the upper 16 bits of an
 * fp32 word), 2 = fp64.  With A = X (M x K) and Bm = W_cat (N x K) this is
 * U = X W_cat^T of Eq. (1); with other strides it is dX = dU W_cat and
 * dW_cat = dU^T X, the gradients of that product.
 * ------------------------------------------------------------------------- */
static double load_elem(const void* p, int dtype, int64_t i) {
    if (dtype == 0) return (double)((const float*)p)[i];
    if (dtype == 1) {
        uint32_t w = ((uint32_t)((const uint16_t*)p)[i]) << 16;
        float f;
        memcpy(&f, &w, sizeof f);
        return (double)f;
    }
    return ((const double*)p)[i];
}

int sru_oracle_gemm(int64_t R, int64_t C, int64_t K,
                    const void* A, int a_dtype, int64_t a_rs, int64_t a_ks,
                    const void* Bm, int b_dtype, int64_t b_rs, int64_t b_ks,
                    double* out) {
    if (R < 0 || C < 0 || K < 0) return -1;
    for (int64_t r = 0; r < R; ++r)
        for (int64_t c = 0; c < C; ++c) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += load_elem(A, a_dtype, r * a_rs + k * a_ks) *
                       load_elem(Bm, b_dtype, c * b_rs + k * b_ks);
            out[r * C + c] = acc;
        }
    return 0;
}

/* The same sum for a list of n (row, col) entries: out[i] = sum_k A(rows[i], k) * Bm(cols[i], k). */
int sru_oracle_gemm_entries(int64_t n, const int64_t* rows, const int64_t* cols, int64_t K,
                            const void* A, int a_dtype, int64_t a_rs, int64_t a_ks,
                            const void* Bm, int b_dtype, int64_t b_rs, int64_t b_ks,
                            double* out) {
    if (n < 0 || K < 0) return -1;
    for (int64_t i = 0; i < n; ++i) {
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k)
            acc += load_elem(A, a_dtype, rows[i] * a_rs + k * a_ks) *
                   load_elem(Bm, b_dtype, cols[i] * b_rs + k * b_ks);
        out[i] = acc;
    }
    return 0;
}
