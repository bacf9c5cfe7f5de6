/*
 * Float64 CPU oracle for block-causal ReLU linear attention with 3D RoPE.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the tests, the smoke check and the benchmark's CPU
 * baseline use it.  It shares no code, header or table with the CUDA path.
 *
 * What it computes (sources are the SANA-Video pages):
 *   - "SANA-Video ... Block Linear Diffusion Transformer [ICLR 2026, Oral]"
 *     talk transcript, passage reviewing the linear-attention state: the state
 *     is a d x d matrix whatever the sequence length; each block adds its own
 *     contribution K^T V to the cached state of the previous blocks; block b
 *     sees its own block and all earlier blocks; 3D RoPE is applied inside
 *     linear attention.
 *   - "四库全闻快报：NVIDIA团队重磅突破 ..." news article, paragraph on the
 *     positional encoding: RoPE stays in the numerator and is removed from the
 *     denominator for numerical stability.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   phi = ReLU; tokens ordered t-major, then y, then x; RoPE rotates
 *   interleaved pairs (2j, 2j+1) inside each axis section, sections ordered
 *   t, y, x, angle p_a * theta^(-2j/d_a); q and k are both rotated in the
 *   numerator, neither in the denominator; eps is added after the
 *   denominator's dot product; no 1/sqrt(d) scale; block of a frame is
 *   floor(t_abs / F); attention is full inside a block.
 *
 * Inputs arrive as float32 arrays holding the exact values handed to the GPU
 * (bf16 values widen exactly); every sum and product here is in double.
 *
 * Parity pins: the test suite checks this file against brute-force
 * enumeration, the non-causal textbook case, a library RoPE, closed forms and
 * invariants.  The RoPE pairing and frequency schedule are a reading, not
 * something the pages fix ("parity unpinned" against the pages for that part;
 * pinned to the standard RoPE of a library for the frequencies and sign).
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static int threads_of(int nthreads) {
#ifdef _OPENMP
    return nthreads > 0 ? nthreads : omp_get_max_threads();
#else
    (void)nthreads;
    return 1;
#endif
}

/* a0: token n of a call covering frames [t0, t0+T) of a (T, Hg, Wg) latent grid.
 * Row-major order over (t, y, x).  pos[n] = (t0 + t, y, x); blk[n] = absolute
 * block index (t0 + t) / F.  (Block ordering: talk transcript, block-causal
 * walk-through; frame grouping into blocks of F latent frames.) */
void blin_oracle_grid(long T, long Hg, long Wg, long F, long t0, long *pos, long *blk) {
    long n = 0;
    for (long t = 0; t < T; ++t)
        for (long y = 0; y < Hg; ++y)
            for (long x = 0; x < Wg; ++x) {
                pos[3 * n + 0] = t0 + t;
                pos[3 * n + 1] = y;
                pos[3 * n + 2] = x;
                blk[n] = (t0 + t) / F;
                ++n;
            }
}

/* R_p u: 3D rotary embedding of a d-vector at position p = (t, y, x).
 * Axis a owns split[a] consecutive features (t first, then y, then x); inside
 * an axis, feature pair (2j, 2j+1) turns by angle p_a * theta^(-2j/split[a]).
 * (Talk transcript: 3D RoPE for linear attention.) */
void blin_oracle_rope(const double *u, double *out, int d, const int *split, double theta,
                      const long *p) {
    int off = 0;
    for (int a = 0; a < 3; ++a) {
        const int da = split[a];
        for (int j = 0; j < da / 2; ++j) {
            const double freq = pow(theta, -2.0 * (double)j / (double)da);
            const double ang = (double)p[a] * freq;
            const double c = cos(ang), s = sin(ang);
            const double x0 = u[off + 2 * j], x1 = u[off + 2 * j + 1];
            out[off + 2 * j] = x0 * c - x1 * s;
            out[off + 2 * j + 1] = x0 * s + x1 * c;
        }
        off += da;
    }
    (void)d;
}

static double relu(double x) { return x > 0.0 ? x : 0.0; }

/* phi(u) and R_p phi(u) for every row of a [BH][n][d] float32 array. */
static void features(const float *x, const long *pos, long BH, long n, int d, const int *split,
                     double theta, double *phi, double *rot, int nth) {
#pragma omp parallel for schedule(static) num_threads(nth)
    for (long r = 0; r < BH * n; ++r) {
        const long tok = r % n;
        double *ph = phi + (size_t)r * d;
        for (int i = 0; i < d; ++i) ph[i] = relu((double)x[(size_t)r * d + i]);
        blin_oracle_rope(ph, rot + (size_t)r * d, d, split, theta, pos + 3 * tok);
    }
}

/* Explicit masked double sum over query/key pairs (the O(N^2) definition).
 * For each head and query n, over keys m with blk_k[m] <= blk_q[n]:
 *   num_n += ((R_n phi(q_n)) . (R_m phi(k_m))) v_m      (RoPE in the numerator)
 *   den_n += phi(q_n) . phi(k_m)                         (no RoPE in the denominator)
 * Accumulates into num [BH][nq][d] and den [BH][nq], so callers may stream
 * keys block by block in ascending order.  (Talk transcript: block b attends
 * to its own and all earlier blocks; news article: RoPE only in the numerator.)
 * q: [BH][nq][d], k, v: [BH][nk][d]. */
int blin_oracle_pairsum(const float *q, const long *qpos, const long *qblk, long nq,
                        const float *k, const float *v, const long *kpos, const long *kblk, long nk,
                        long BH, int d, const int *split, double theta,
                        double *num, double *den, int nthreads) {
    const int nth = threads_of(nthreads);
    double *qphi = malloc(sizeof(double) * (size_t)BH * nq * d);
    double *qrot = malloc(sizeof(double) * (size_t)BH * nq * d);
    double *kphi = malloc(sizeof(double) * (size_t)BH * nk * d);
    double *krot = malloc(sizeof(double) * (size_t)BH * nk * d);
    if (!qphi || !qrot || !kphi || !krot) {
        free(qphi); free(qrot); free(kphi); free(krot);
        return -1;
    }
    features(q, qpos, BH, nq, d, split, theta, qphi, qrot, nth);
    features(k, kpos, BH, nk, d, split, theta, kphi, krot, nth);
#pragma omp parallel for schedule(dynamic, 1) num_threads(nth)
    for (long r = 0; r < BH * nq; ++r) {
        const long h = r / nq, n = r % nq;
        const double *qr = qrot + (size_t)r * d, *qp = qphi + (size_t)r * d;
        double *acc = num + (size_t)r * d;
        double dsum = den[r];
        for (long m = 0; m < nk; ++m) {
            if (kblk[m] > qblk[n]) continue;
            const double *kr = krot + ((size_t)h * nk + m) * d;
            const double *kp = kphi + ((size_t)h * nk + m) * d;
            const float *vm = v + ((size_t)h * nk + m) * d;
            double w = 0.0, s = 0.0;
            for (int i = 0; i < d; ++i) {
                w += qr[i] * kr[i];
                s += qp[i] * kp[i];
            }
            for (int j = 0; j < d; ++j) acc[j] += w * (double)vm[j];
            dsum += s;
        }
        den[r] = dsum;
    }
    free(qphi); free(qrot); free(kphi); free(krot);
    return 0;
}

/* o_n = num_n / (den_n + eps). */
void blin_oracle_finish(const double *num, const double *den, long rows, int d, double eps,
                        double *out) {
    for (long r = 0; r < rows; ++r)
        for (int j = 0; j < d; ++j) out[(size_t)r * d + j] = num[(size_t)r * d + j] / (den[r] + eps);
}

/* State (recurrent) form, all rows.  Blocks must be contiguous and ascending
 * in token order (true for the row-major grid).  Per head, starting from the
 * cached (S, z) (zero when S_in is NULL), for each block b in order:
 *   S += sum_{m in b} (R_m phi(k_m)) v_m^T      z += sum_{m in b} phi(k_m)
 * then every query of block b reads the updated state:
 *   o_n = (R_n phi(q_n))^T S / (phi(q_n) . z + eps).
 * The final (S, z) is returned for the next call.  (Talk transcript: the state
 * S_i is the cached S_{i-1} plus block i's contribution; the cache is fixed in
 * size.)  S: [BH][d][d] row = rotated key feature, column = value feature. */
int blin_oracle_recurrence(const float *q, const float *k, const float *v, const long *pos,
                           const long *blk, long BH, long N, int d, const int *split, double theta,
                           double eps, const double *S_in, const double *z_in, double *out,
                           double *S_out, double *z_out, int nthreads) {
    const int nth = threads_of(nthreads);
    int rc = 0;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nth) reduction(| : rc)
    for (long h = 0; h < BH; ++h) {
        double *S = calloc((size_t)d * d, sizeof(double));
        double *z = calloc((size_t)d, sizeof(double));
        double *ph = malloc(sizeof(double) * d), *rt = malloc(sizeof(double) * d);
        if (!S || !z || !ph || !rt) {
            rc |= 1;
            free(S); free(z); free(ph); free(rt);
            continue;
        }
        if (S_in) memcpy(S, S_in + (size_t)h * d * d, sizeof(double) * d * d);
        if (z_in) memcpy(z, z_in + (size_t)h * d, sizeof(double) * d);
        long b0 = 0;
        while (b0 < N) {
            long b1 = b0;
            while (b1 < N && blk[b1] == blk[b0]) ++b1;
            /* add this block's contribution */
            for (long m = b0; m < b1; ++m) {
                const float *km = k + ((size_t)h * N + m) * d;
                const float *vm = v + ((size_t)h * N + m) * d;
                for (int i = 0; i < d; ++i) ph[i] = relu((double)km[i]);
                blin_oracle_rope(ph, rt, d, split, theta, pos + 3 * m);
                for (int i = 0; i < d; ++i) {
                    z[i] += ph[i];
                    for (int j = 0; j < d; ++j) S[(size_t)i * d + j] += rt[i] * (double)vm[j];
                }
            }
            /* read it for every query of the block */
            for (long n = b0; n < b1; ++n) {
                const float *qn = q + ((size_t)h * N + n) * d;
                for (int i = 0; i < d; ++i) ph[i] = relu((double)qn[i]);
                blin_oracle_rope(ph, rt, d, split, theta, pos + 3 * n);
                double den = 0.0;
                for (int i = 0; i < d; ++i) den += ph[i] * z[i];
                den += eps;
                double *o = out + ((size_t)h * N + n) * d;
                for (int j = 0; j < d; ++j) {
                    double s = 0.0;
                    for (int i = 0; i < d; ++i) s += rt[i] * S[(size_t)i * d + j];
                    o[j] = s / den;
                }
            }
            b0 = b1;
        }
        if (S_out) memcpy(S_out + (size_t)h * d * d, S, sizeof(double) * d * d);
        if (z_out) memcpy(z_out + (size_t)h * d, z, sizeof(double) * d);
        free(S); free(z); free(ph); free(rt);
    }
    return rc ? -1 : 0;
}

/* Causal block temporal convolution of the Mix-FFN, with its one-frame cache.
 * (Talk transcript, causal-FFN passage: in causal training a zero token is put
 * between two blocks, so that block i cannot see block i+1; block i+1 must
 * see block i, so block i's last token is cached and put in front of block
 * i+1.)  Per batch entry, spatial position s and channel c, with taps
 * w[c] = (previous, current, next):
 *   y[t] = w[c][0] * x[t-1] + w[c][1] * x[t] + w[c][2] * x[t+1] + bias[c]
 * where x[t-1] is the previous frame (from this call, or `prev` -- the cache,
 * the last frame of the previous call -- for the call's first frame; zero
 * before the video's first frame), and x[t+1] is the next frame only when it
 * lies in the same block of F frames (t_abs / F) and in this call; otherwise
 * zero (the pad between blocks).
 *   x: [B][T][HW][C] float32 values of absolute frames t0 .. t0+T-1
 *   prev: [B][HW][C] (frame t0-1) or NULL for zero
 *   w: [C][3], bias: [C] or NULL;  y: [B][T][HW][C] */
void blin_oracle_tconv(const float *x, const double *prev, const double *w, const double *bias, long B,
                       long T, long HW, long C, long t0, long F, double *y) {
    for (long b = 0; b < B; ++b)
        for (long t = 0; t < T; ++t)
            for (long s = 0; s < HW; ++s)
                for (long c = 0; c < C; ++c) {
                    const long ta = t0 + t;
                    double xp = 0.0, xn = 0.0;
                    if (t > 0)
                        xp = (double)x[((b * T + t - 1) * HW + s) * C + c];
                    else if (ta > 0 && prev != NULL)
                        xp = prev[(b * HW + s) * C + c];
                    if (t + 1 < T && (ta + 1) / F == ta / F) xn = (double)x[((b * T + t + 1) * HW + s) * C + c];
                    const double xc = (double)x[((b * T + t) * HW + s) * C + c];
                    y[((b * T + t) * HW + s) * C + c] =
                        w[3 * c] * xp + w[3 * c + 1] * xc + w[3 * c + 2] * xn + (bias ? bias[c] : 0.0);
                }
}

/* NVFP4 block-scaled 4-bit inputs (news article, NVFP4 / SVDQuant paragraph:
 * the QKV projections run in NVFP4).  Element i of a d-vector is an E2M1 code
 * (bit 3 sign, bits 2..1 exponent with bias 1, bit 0 mantissa) in nibble i of
 * the row's d/2 bytes (even elements in the low nibble); each run of 16
 * consecutive elements shares one E4M3 scale byte (bit 7 sign, bits 6..3
 * exponent with bias 7, bits 2..0 mantissa; no infinities, 0x7f/0xff NaN);
 * the tensor has one global scale.  value = e2m1 * e4m3 * global. */
double blin_oracle_e2m1(int code) {
    const int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    const double mag = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

double blin_oracle_e4m3(int code) {
    const int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    const double mag = e == 0 ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Dequantise rows x rows of d elements: data [rows][d/2], scale [rows][d/16] -> out [rows][d]. */
void blin_oracle_nvfp4_decode(const unsigned char *data, const unsigned char *scale, long rows, int d,
                              double global, double *out) {
    for (long r = 0; r < rows; ++r)
        for (int i = 0; i < d; ++i) {
            const int byte = data[r * (d / 2) + i / 2];
            const int code = (i & 1) ? (byte >> 4) & 15 : byte & 15;
            out[r * d + i] = blin_oracle_e2m1(code) * blin_oracle_e4m3(scale[r * (d / 16) + i / 16]) * global;
        }
}
