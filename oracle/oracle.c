/*
 * oracle.c -- plain CPU reference; see oracle.h for the sources and contract.
 *
 * TEST INFRASTRUCTURE ONLY: the product library never links or calls this.
 * Written for reading, not for speed: one loop nest per definition, no
 * blocking, no reordering beyond what each definition states.  The loops over
 * independent output rows may run on several OpenMP threads; that changes no
 * result because every output element is computed by one thread in a fixed
 * order.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* number formats                                                            */
/* ------------------------------------------------------------------------ */

float oracle_bf16_to_f32(uint16_t b) {
    /* bf16 is the upper half of an IEEE binary32: widening is exact. */
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

uint16_t oracle_f32_to_f16(float x) {
    /* The C conversion to _Float16 rounds to nearest even (IEEE 754). */
    _Float16 h = (_Float16)x;
    uint16_t b;
    memcpy(&b, &h, 2);
    return b;
}

float oracle_f16_to_f32(uint16_t b) {
    _Float16 h;
    memcpy(&h, &b, 2);
    return (float)h;
}

static int f16_is_finite(uint16_t b) { return (b & 0x7C00u) != 0x7C00u; }

void oracle_set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

int oracle_get_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* MinMax group quantizer                                                    */
/* [GB] 模型量化 (1): classic group-wise MinMax quantizer, INT4 with group    */
/* size 128 and INT2 with group size 64.  Per group, with Q = 2^bits - 1:    */
/*   mn, mx   = min, max of the group (bf16 widened to fp32, exact)           */
/*   r        = fp32(mx - mn)                                               */
/*   scale    = fp16_rne(fp32(r / Q)); if r == 0 or it rounds to 0: 1.0      */
/*   zero     = fp16(rint(fp32(-mn / scale)))   (round half to even)        */
/*   q        = clamp(rint(fp32(w / scale)) + zero, 0, Q)                   */
/* where scale and zero are the stored fp16 values.                         */
/* ------------------------------------------------------------------------ */

int oracle_minmax_quantize(const uint16_t* W, int64_t n, int64_t k, int bits,
                           int group, uint8_t* codes, uint16_t* scale,
                           uint16_t* zero) {
    if (!(bits == 2 || bits == 4) || group <= 0 || k % group != 0 || n < 0)
        return -1;
    const int64_t ngroups = k / group;
    const float Q = (float)((1 << bits) - 1);
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int64_t row = 0; row < n; ++row) {
        for (int64_t g = 0; g < ngroups; ++g) {
            const uint16_t* w = W + row * k + g * group;
            float mn = INFINITY, mx = -INFINITY;
            for (int i = 0; i < group; ++i) {
                float v = oracle_bf16_to_f32(w[i]);
                if (!isfinite(v)) bad = 1;
                if (v < mn) mn = v;
                if (v > mx) mx = v;
            }
            /* -0 and +0 compare equal; adding +0 makes the extremes +0 so the
             * result does not depend on which of the two was seen first. */
            mn = mn + 0.0f;
            mx = mx + 0.0f;
            float r = mx - mn;
            float s32 = r / Q;
            uint16_t s16 = oracle_f32_to_f16(s32);
            if (r == 0.0f || (s16 & 0x7FFFu) == 0) s16 = oracle_f32_to_f16(1.0f);
            if (!f16_is_finite(s16)) bad = 1;
            float sf = oracle_f16_to_f32(s16);
            float z32 = rintf(-mn / sf);
            uint16_t z16 = oracle_f32_to_f16(z32);
            if (!f16_is_finite(z16)) bad = 1;
            float zf = oracle_f16_to_f32(z16);
            scale[row * ngroups + g] = s16;
            zero[row * ngroups + g] = z16;
            if (codes) {
                for (int i = 0; i < group; ++i) {
                    float v = oracle_bf16_to_f32(w[i]);
                    float t = v / sf;
                    float qf = rintf(t) + zf;
                    if (qf < 0.0f) qf = 0.0f;
                    if (qf > Q) qf = Q;
                    codes[row * k + g * group + i] = (uint8_t)qf;
                }
            }
        }
    }
    return bad ? -2 : 0;
}

/* [BNB] 量化数据的存储: two 4-bit codes per byte, the first code in the high
 * nibble: byte j = (q[2j] << 4) | q[2j+1].  2-bit codes extend the same order
 * to four codes per byte, the first in the top two bits. */
int oracle_pack(const uint8_t* codes, int64_t n, int64_t k, int bits,
                uint8_t* packed) {
    if (!(bits == 2 || bits == 4)) return -1;
    const int per = 8 / bits;
    if (k % per != 0) return -1;
    const int64_t bytes_per_row = k / per;
    for (int64_t row = 0; row < n; ++row)
        for (int64_t j = 0; j < bytes_per_row; ++j) {
            unsigned byte = 0;
            for (int t = 0; t < per; ++t) {
                unsigned q = codes[row * k + j * per + t];
                byte |= (q & ((1u << bits) - 1)) << (8 - bits * (t + 1));
            }
            packed[row * bytes_per_row + j] = (uint8_t)byte;
        }
    return 0;
}

int oracle_unpack(const uint8_t* packed, int64_t n, int64_t k, int bits,
                  uint8_t* codes) {
    if (!(bits == 2 || bits == 4)) return -1;
    const int per = 8 / bits;
    if (k % per != 0) return -1;
    const int64_t bytes_per_row = k / per;
    for (int64_t row = 0; row < n; ++row)
        for (int64_t j = 0; j < bytes_per_row; ++j) {
            unsigned byte = packed[row * bytes_per_row + j];
            for (int t = 0; t < per; ++t)
                codes[row * k + j * per + t] =
                    (uint8_t)((byte >> (8 - bits * (t + 1))) & ((1u << bits) - 1));
        }
    return 0;
}

/* Dequantize one element of the MinMax format: (q - zero) * scale in fp32.
 * The difference of two integers is exact; the product is exact whenever
 * |q - zero| < 2^13 (an integer of at most 13 bits times an 11-bit fp16
 * significand), and otherwise one correctly rounded fp32 multiply. */
static float minmax_element(const uint8_t* packed, const uint16_t* scale,
                            const uint16_t* zero, int64_t k, int bits,
                            int group, int64_t row, int64_t col) {
    const int per = 8 / bits;
    const int64_t bytes_per_row = k / per;
    unsigned byte = packed[row * bytes_per_row + col / per];
    int t = (int)(col % per);
    unsigned q = (byte >> (8 - bits * (t + 1))) & ((1u << bits) - 1);
    int64_t g = col / group;
    float sf = oracle_f16_to_f32(scale[row * (k / group) + g]);
    float zf = oracle_f16_to_f32(zero[row * (k / group) + g]);
    float d = (float)q - zf;
    return d * sf;
}

int oracle_minmax_dequantize(const uint8_t* packed, const uint16_t* scale,
                             const uint16_t* zero, int64_t n, int64_t k,
                             int bits, int group, float* W_hat) {
    if (!(bits == 2 || bits == 4) || group <= 0 || k % group != 0) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t row = 0; row < n; ++row)
        for (int64_t col = 0; col < k; ++col)
            W_hat[row * k + col] =
                minmax_element(packed, scale, zero, k, bits, group, row, col);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* 4-bit codebook quantizer ([QL] 关键技术细节 1; [BNB] nf4/fp4)             */
/* Blocks of 64 consecutive elements of the row-major flattened W:          */
/*   a    = max |w| over the block (fp32)                                   */
/*   x    = fp32(w / a)            (x = 0 when a == 0)                      */
/*   code = argmin_j |x - c_j| in fp32, the lower index on ties             */
/* ------------------------------------------------------------------------ */

int oracle_codebook_quantize(const uint16_t* W, int64_t n, int64_t k,
                             const float* codebook, uint8_t* codes,
                             float* absmax) {
    if ((n * k) % 64 != 0) return -1;
    /* any 16 entries in [-1, 1] that include a zero (+0 or -0), in any
     * order: a table in code order, such as the FP4 (E2M1) one with its two
     * zeros, is used as given */
    int has_zero = 0;
    for (int j = 0; j < 16; ++j) {
        if (codebook[j] == 0.0f) has_zero = 1;
        if (!(codebook[j] >= -1.0f && codebook[j] <= 1.0f)) return -1;
    }
    if (!has_zero) return -1;
    const int64_t nb = n * k / 64;
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int64_t b = 0; b < nb; ++b) {
        const uint16_t* w = W + b * 64;
        float a = 0.0f;
        for (int i = 0; i < 64; ++i) {
            float v = fabsf(oracle_bf16_to_f32(w[i]));
            if (!isfinite(v)) bad = 1;
            if (v > a) a = v;
        }
        absmax[b] = a;
        if (codes) {
            for (int i = 0; i < 64; ++i) {
                float x = (a == 0.0f) ? 0.0f : oracle_bf16_to_f32(w[i]) / a;
                int best = 0;
                float bestd = fabsf(x - codebook[0]);
                for (int j = 1; j < 16; ++j) {
                    float d = fabsf(x - codebook[j]);
                    if (d < bestd) { bestd = d; best = j; }
                }
                codes[b * 64 + i] = (uint8_t)best;
            }
        }
    }
    return bad ? -2 : 0;
}

/* Double quantization ([QL] 结论: the scale factors and their offset are
 * quantized again; [BNB] nested absmax).  Reading adopted:
 *   offset = fp32( fp64(sum of all absmax) / nb )
 *   c_i    = fp32(a_i - offset)
 *   per block of 256 (the last one may be shorter):
 *     s2   = max |c_i|
 *     q8_i = clamp(rint(fp32(fp32(c_i / s2) * 127)), -127, 127)  (0 if s2 == 0)
 * The fp64 sum is required to be exact (it is whenever the absmax values span
 * less than 2^(45 - log2 nb) in magnitude; they are bf16 values), so that the
 * result does not depend on the order of summation; -2 otherwise. */
int oracle_double_quant(const float* absmax, int64_t nb, int8_t* q8,
                        float* s2, float* offset) {
    if (nb <= 0) return -1;
    double sum = 0.0;
    int exact = 1;
    for (int64_t i = 0; i < nb; ++i) {
        /* Knuth's two-sum gives the rounding error of each addition exactly;
         * the sum is exact when every error is zero. */
        double a = sum, b = (double)absmax[i];
        double s_ = a + b;
        double bb = s_ - a;
        double err = (a - (s_ - bb)) + (b - bb);
        if (err != 0.0) exact = 0;
        sum = s_;
    }
    float off = (float)(sum / (double)nb);
    *offset = off;
    const int64_t nblk = (nb + 255) / 256;
    for (int64_t b = 0; b < nblk; ++b) {
        int64_t lo = b * 256, hi = lo + 256 < nb ? lo + 256 : nb;
        float m = 0.0f;
        for (int64_t i = lo; i < hi; ++i) {
            float c = absmax[i] - off;
            if (fabsf(c) > m) m = fabsf(c);
        }
        s2[b] = m;
        for (int64_t i = lo; i < hi; ++i) {
            float c = absmax[i] - off;
            float qf = 0.0f;
            if (m != 0.0f) {
                float t = c / m;
                float u = t * 127.0f;
                qf = rintf(u);
                if (qf > 127.0f) qf = 127.0f;
                if (qf < -127.0f) qf = -127.0f;
            }
            q8[i] = (int8_t)qf;
        }
    }
    return exact ? 0 : -2;
}

int oracle_double_dequant(const int8_t* q8, const float* s2, float offset,
                          int64_t nb, float* absmax_hat) {
    for (int64_t i = 0; i < nb; ++i) {
        float t = (float)q8[i] / 127.0f;
        float u = t * s2[i / 256];
        absmax_hat[i] = u + offset;
    }
    return 0;
}

int oracle_codebook_dequantize(const uint8_t* packed, const float* absmax,
                               const float* codebook, int64_t n, int64_t k,
                               float* W_hat) {
    if ((n * k) % 64 != 0 || k % 2 != 0) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t row = 0; row < n; ++row)
        for (int64_t col = 0; col < k; ++col) {
            int64_t idx = row * k + col;
            unsigned byte = packed[idx / 2];
            unsigned q = (idx % 2 == 0) ? (byte >> 4) : (byte & 15u);
            W_hat[idx] = codebook[q] * absmax[idx / 64];
        }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Quantized linear layer with a low-rank adapter                            */
/* [QL] QLoRA技术原理: the frozen 4-bit weight is dequantized and gradients    */
/* flow only into the adapters.  Forward Y = X W^T + s (X A^T) B^T; the      */
/* backward products follow from differentiating that expression.           */
/* ------------------------------------------------------------------------ */

int oracle_linear_fwd(const uint16_t* X, int64_t m, const float* W_hat,
                      int64_t n, int64_t k, const uint16_t* A,
                      const uint16_t* B, int r, double s, double* Y,
                      double* T, double* Ybound) {
    if (r < 0 || r > 256 || (r > 0 && (!A || !B))) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < m; ++i) {
        double t[256];
        double ta[256]; /* sum_k |x_ik| |A_tk| */
        for (int u = 0; u < r; ++u) {
            double acc = 0.0, acca = 0.0;
            for (int64_t c = 0; c < k; ++c) {
                double x = oracle_bf16_to_f32(X[i * k + c]);
                double a = oracle_bf16_to_f32(A[u * k + c]);
                acc += x * a;
                acca += fabs(x) * fabs(a);
            }
            t[u] = acc;
            ta[u] = acca;
            if (T) T[i * r + u] = acc;
        }
        for (int64_t j = 0; j < n; ++j) {
            double acc = 0.0, bnd = 0.0;
            for (int64_t c = 0; c < k; ++c) {
                double x = oracle_bf16_to_f32(X[i * k + c]);
                double w = W_hat[j * k + c];
                acc += x * w;
                bnd += fabs(x) * fabs(w);
            }
            double lora = 0.0, lbnd = 0.0;
            for (int u = 0; u < r; ++u) {
                double b = oracle_bf16_to_f32(B[j * r + u]);
                lora += t[u] * b;
                lbnd += ta[u] * fabs(b);
            }
            if (Y) Y[i * n + j] = acc + s * lora;
            if (Ybound) Ybound[i * n + j] = bnd + fabs(s) * lbnd;
        }
    }
    return 0;
}

int oracle_linear_bwd(const uint16_t* dY, int64_t m, const float* W_hat,
                      int64_t n, int64_t k, const uint16_t* A,
                      const uint16_t* B, int r, double s, double* dX,
                      double* U, double* dXbound) {
    if (r < 0 || r > 256 || (r > 0 && (!A || !B))) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < m; ++i) {
        double u_[256];
        double ub[256]; /* sum_j |dy_ij| |B_jt| */
        for (int t = 0; t < r; ++t) {
            double acc = 0.0, accb = 0.0;
            for (int64_t j = 0; j < n; ++j) {
                double g = oracle_bf16_to_f32(dY[i * n + j]);
                double b = oracle_bf16_to_f32(B[j * r + t]);
                acc += g * b;
                accb += fabs(g) * fabs(b);
            }
            u_[t] = acc;
            ub[t] = accb;
            if (U) U[i * r + t] = acc;
        }
        for (int64_t c = 0; c < k; ++c) {
            double acc = 0.0, bnd = 0.0;
            for (int64_t j = 0; j < n; ++j) {
                double g = oracle_bf16_to_f32(dY[i * n + j]);
                double w = W_hat[j * k + c];
                acc += g * w;
                bnd += fabs(g) * fabs(w);
            }
            double lora = 0.0, lbnd = 0.0;
            for (int t = 0; t < r; ++t) {
                double a = oracle_bf16_to_f32(A[t * k + c]);
                lora += u_[t] * a;
                lbnd += ub[t] * fabs(a);
            }
            if (dX) dX[i * k + c] = acc + s * lora;
            if (dXbound) dXbound[i * k + c] = bnd + fabs(s) * lbnd;
        }
    }
    return 0;
}

int oracle_lora_grads(const uint16_t* X, const uint16_t* dY, int64_t m,
                      int64_t n, int64_t k, const uint16_t* A,
                      const uint16_t* B, int r, double s, double* dA,
                      double* dB, double* dAbound, double* dBbound) {
    if (r <= 0) return -1;
    /* T = X A^T and U = dY B, with their magnitude sums */
    double* T = (double*)calloc((size_t)(m * r), sizeof(double));
    double* Ta = (double*)calloc((size_t)(m * r), sizeof(double));
    double* U = (double*)calloc((size_t)(m * r), sizeof(double));
    double* Ua = (double*)calloc((size_t)(m * r), sizeof(double));
    if (!T || !Ta || !U || !Ua) { free(T); free(Ta); free(U); free(Ua); return -3; }
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < m; ++i)
        for (int t = 0; t < r; ++t) {
            double acc = 0.0, acca = 0.0;
            for (int64_t c = 0; c < k; ++c) {
                double x = oracle_bf16_to_f32(X[i * k + c]);
                double a = oracle_bf16_to_f32(A[t * k + c]);
                acc += x * a;
                acca += fabs(x) * fabs(a);
            }
            T[i * r + t] = acc;
            Ta[i * r + t] = acca;
            acc = 0.0; acca = 0.0;
            for (int64_t j = 0; j < n; ++j) {
                double g = oracle_bf16_to_f32(dY[i * n + j]);
                double b = oracle_bf16_to_f32(B[j * r + t]);
                acc += g * b;
                acca += fabs(g) * fabs(b);
            }
            U[i * r + t] = acc;
            Ua[i * r + t] = acca;
        }
    /* dA[t, c] = s sum_i U[i, t] X[i, c] */
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < k; ++c)
        for (int t = 0; t < r; ++t) {
            double acc = 0.0, bnd = 0.0;
            for (int64_t i = 0; i < m; ++i) {
                double x = oracle_bf16_to_f32(X[i * k + c]);
                acc += U[i * r + t] * x;
                bnd += Ua[i * r + t] * fabs(x);
            }
            if (dA) dA[t * k + c] = s * acc;
            if (dAbound) dAbound[t * k + c] = fabs(s) * bnd;
        }
    /* dB[j, t] = s sum_i dY[i, j] T[i, t] */
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j)
        for (int t = 0; t < r; ++t) {
            double acc = 0.0, bnd = 0.0;
            for (int64_t i = 0; i < m; ++i) {
                double g = oracle_bf16_to_f32(dY[i * n + j]);
                acc += g * T[i * r + t];
                bnd += fabs(g) * Ta[i * r + t];
            }
            if (dB) dB[j * r + t] = s * acc;
            if (dBbound) dBbound[j * r + t] = fabs(s) * bnd;
        }
    free(T); free(Ta); free(U); free(Ua);
    return 0;
}

int oracle_linear_fwd_sampled_minmax(const uint16_t* X, int64_t m,
                                     const uint8_t* packed,
                                     const uint16_t* scale,
                                     const uint16_t* zero, int64_t n,
                                     int64_t k, int bits, int group,
                                     const uint16_t* A, const uint16_t* B,
                                     int r, double s, int64_t npairs,
                                     const int64_t* rows, const int64_t* cols,
                                     double* Y, double* Ybound) {
    if (!(bits == 2 || bits == 4) || k % group != 0 || r < 0) return -1;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t p = 0; p < npairs; ++p) {
        int64_t i = rows[p], j = cols[p];
        if (i < 0 || i >= m || j < 0 || j >= n) continue;
        double acc = 0.0, bnd = 0.0;
        for (int64_t c = 0; c < k; ++c) {
            double x = oracle_bf16_to_f32(X[i * k + c]);
            double w = minmax_element(packed, scale, zero, k, bits, group, j, c);
            acc += x * w;
            bnd += fabs(x) * fabs(w);
        }
        double lora = 0.0, lbnd = 0.0;
        for (int u = 0; u < r; ++u) {
            double t = 0.0, ta = 0.0;
            for (int64_t c = 0; c < k; ++c) {
                double x = oracle_bf16_to_f32(X[i * k + c]);
                double a = oracle_bf16_to_f32(A[u * k + c]);
                t += x * a;
                ta += fabs(x) * fabs(a);
            }
            double b = oracle_bf16_to_f32(B[j * r + u]);
            lora += t * b;
            lbnd += ta * fabs(b);
        }
        Y[p] = acc + s * lora;
        Ybound[p] = bnd + fabs(s) * lbnd;
    }
    return 0;
}

/* dX (and its bound) at a list of (token, feature) pairs, for sampled parity
 * at full size ([QL] QLoRA技术原理: dX = dY W_hat + s (dY B) A).  Each pair
 * is computed on its own from the packed MinMax weight, one column of W_hat
 * at a time, with U = dY B recomputed for its token. */
int oracle_linear_bwd_sampled_minmax(const uint16_t* dY, int64_t m,
                                     const uint8_t* packed,
                                     const uint16_t* scale,
                                     const uint16_t* zero, int64_t n,
                                     int64_t k, int bits, int group,
                                     const uint16_t* A, const uint16_t* B,
                                     int r, double s, int64_t npairs,
                                     const int64_t* rows, const int64_t* cols,
                                     double* dX, double* dXbound) {
    if (!(bits == 2 || bits == 4) || k % group != 0 || r < 0) return -1;
#pragma omp parallel for schedule(dynamic, 8)
    for (int64_t p = 0; p < npairs; ++p) {
        int64_t t = rows[p], col = cols[p];
        if (t < 0 || t >= m || col < 0 || col >= k) continue;
        double acc = 0.0, bnd = 0.0;
        for (int64_t c = 0; c < n; ++c) {
            double g = oracle_bf16_to_f32(dY[t * n + c]);
            double w = minmax_element(packed, scale, zero, k, bits, group, c, col);
            acc += g * w;
            bnd += fabs(g) * fabs(w);
        }
        double lora = 0.0, lbnd = 0.0;
        for (int u = 0; u < r; ++u) {
            double uu = 0.0, ub = 0.0;
            for (int64_t c = 0; c < n; ++c) {
                double g = oracle_bf16_to_f32(dY[t * n + c]);
                double b = oracle_bf16_to_f32(B[c * r + u]);
                uu += g * b;
                ub += fabs(g) * fabs(b);
            }
            double a = oracle_bf16_to_f32(A[u * k + col]);
            lora += uu * a;
            lbnd += ub * fabs(a);
        }
        dX[p] = acc + s * lora;
        dXbound[p] = bnd + fabs(s) * lbnd;
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Merging the adapter into the weight                                       */
/* [GB] introduction: after QLoRA fine-tuning the LoRA module is merged into */
/* the full-precision model.  The merged weight is W_hat + s B A; removing   */
/* the adapter again subtracts the same product.                             */
/* ------------------------------------------------------------------------ */

/* binary32 -> bf16, round to nearest, ties to even: keep the upper 16 bits
 * and round up when the dropped half is above one half ulp, or exactly one
 * half with an odd kept part (a carry into the exponent is the correct
 * result).  NaN stays a quiet NaN. */
static uint16_t f32_to_bf16_rne(float x) {
    uint32_t u;
    memcpy(&u, &x, 4);
    if (isnan(x)) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t hi = u >> 16, lo = u & 0xFFFFu;
    if (lo > 0x8000u || (lo == 0x8000u && (hi & 1u))) hi += 1u;
    return (uint16_t)hi;
}

int oracle_lora_merge(const float* W_in, int64_t n, int64_t k,
                      const uint16_t* A, const uint16_t* B, int r, float s,
                      int sign, uint16_t* W_out) {
    if (r < 0 || (r > 0 && (!A || !B)) || !(sign == 1 || sign == -1)) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t row = 0; row < n; ++row)
        for (int64_t col = 0; col < k; ++col) {
            float d = 0.0f;
            for (int u = 0; u < r; ++u)
                d = fmaf(oracle_bf16_to_f32(B[row * r + u]), oracle_bf16_to_f32(A[(int64_t)u * k + col]), d);
            float t = s * d;
            float v = (sign > 0) ? W_in[row * k + col] + t : W_in[row * k + col] - t;
            W_out[row * k + col] = f32_to_bf16_rne(v);
        }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* channel-mix selection by sensitivity ([GB] 模型量化 (1): the bit width of  */
/* each output channel follows how sensitive it is to quantization)          */
/*   m2[k]    = (1/T) sum_t x[t,k]^2               (second moment, fp64)      */
/*   e4, e2   = W_hat - w for the MinMax INT4 g128 / INT2 g64 quantization    */
/*   score[c] = sum_k m2[k] * (e2[c,k]^2 - e4[c,k]^2)                         */
/*   bound[c] = sum_k m2[k] * (e2[c,k]^2 + e4[c,k]^2)                         */
/* score is the rise of the expected squared output error of channel c when  */
/* it goes from INT4 to INT2, with the calibration activations' second        */
/* moments on the diagonal.  Selection: the n4 channels with the highest      */
/* score (the lower channel index first among equal scores) are INT4.        */
/* ------------------------------------------------------------------------ */
int oracle_channel_score(const uint16_t* W, int64_t n, int64_t k, const uint16_t* X, int64_t t, double* score,
                         double* bound) {
    if (n < 1 || k < 128 || k % 128 != 0 || t < 1) return -1;
    double* m2 = (double*)malloc(sizeof(double) * k);
    uint8_t* c4 = (uint8_t*)malloc(n * k);
    uint8_t* c2 = (uint8_t*)malloc(n * k);
    uint16_t* s4 = (uint16_t*)malloc(sizeof(uint16_t) * n * (k / 128));
    uint16_t* z4 = (uint16_t*)malloc(sizeof(uint16_t) * n * (k / 128));
    uint16_t* s2 = (uint16_t*)malloc(sizeof(uint16_t) * n * (k / 64));
    uint16_t* z2 = (uint16_t*)malloc(sizeof(uint16_t) * n * (k / 64));
    int rc = (m2 && c4 && c2 && s4 && z4 && s2 && z2) ? 0 : -1;
    if (rc == 0) {
        for (int64_t j = 0; j < k; ++j) {
            double acc = 0.0;
            for (int64_t i = 0; i < t; ++i) {
                double x = oracle_bf16_to_f32(X[i * k + j]);
                acc += x * x;
            }
            m2[j] = acc / (double)t;
        }
        rc = oracle_minmax_quantize(W, n, k, 4, 128, c4, s4, z4);
        if (rc == 0) rc = oracle_minmax_quantize(W, n, k, 2, 64, c2, s2, z2);
    }
    if (rc == 0) {
#pragma omp parallel for schedule(static)
        for (int64_t row = 0; row < n; ++row) {
            double sc = 0.0, bd = 0.0;
            for (int64_t j = 0; j < k; ++j) {
                const double w = oracle_bf16_to_f32(W[row * k + j]);
                /* the dequantized values, each one exact fp32 product */
                const float w4 = ((float)c4[row * k + j] - oracle_f16_to_f32(z4[row * (k / 128) + j / 128])) *
                                 oracle_f16_to_f32(s4[row * (k / 128) + j / 128]);
                const float w2 = ((float)c2[row * k + j] - oracle_f16_to_f32(z2[row * (k / 64) + j / 64])) *
                                 oracle_f16_to_f32(s2[row * (k / 64) + j / 64]);
                const double e4 = (double)w4 - w, e2 = (double)w2 - w;
                sc += m2[j] * (e2 * e2 - e4 * e4);
                bd += m2[j] * (e2 * e2 + e4 * e4);
            }
            score[row] = sc;
            if (bound) bound[row] = bd;
        }
    }
    free(m2); free(c4); free(c2); free(s4); free(z4); free(s2); free(z2);
    return rc;
}

int oracle_channel_mix_select(const double* score, int64_t n, int64_t n4, int32_t* perm) {
    if (n < 1 || n4 < 0 || n4 > n) return -1;
    /* rank of channel c: channels with a higher score, or an equal score and
     * a lower index, come before it */
    int64_t hi = 0, lo = n4;
    for (int64_t c = 0; c < n; ++c) {
        int64_t rank = 0;
        for (int64_t d = 0; d < n; ++d)
            if (score[d] > score[c] || (score[d] == score[c] && d < c)) ++rank;
        if (rank < n4) perm[hi++] = (int32_t)c;
        else perm[lo++] = (int32_t)c;
    }
    return (hi == n4 && lo == n) ? 0 : -1;
}
