/*
 * fp8_oracle.c -- plain, slow CPU oracle for the FP8 training-GEMM path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no code, header or table with the CUDA path under fp8_gemms_b200/.
 *
 * What it computes (sources):
 *  - "FP8 with dynamic tensorwise scaling on all three GEMMs (one forward,
 *    two backward)": decomputer.nl, "Het trainen van een 3.8B LLM tot 0.384
 *    CORE voor $998", section "Vroege experimenten", item 4, and section
 *    "Doorvoer (Throughput) verhogen", FP8 bullet; simpleprog.com,
 *    "Training a 3.8B LLM to 0.384 CORE for $998", section "Five Changes That
 *    Mattered" (fourth change).  manulx.blog (Japanese summary), section
 *    "実際に効いたもの", names the call as torch._scaled_mm: FP8 operands with
 *    one fp32 scale per tensor, bf16 result.
 *  - The non-gated relu^2 MLP at 4x: decomputer.nl, section "Doorvoer
 *    verhogen", bullet "Niet-gated MLPs", and "Appendix: De configuratie"
 *    (hidden_act: relu2, gated_mlp: false, intermediate_size 12288).
 *  - The pages never name the FP8 encodings.  The encodings used are the
 *    public OCP 8-bit floating point formats E4M3 ("fn": no infinities, one
 *    NaN mantissa pattern, max 448) and E5M2 (IEEE-like, max 57344), e4m3 for
 *    activations and weights, e5m2 for gradients.
 *
 * Readings taken where the pages are silent (each is a choice, written out):
 *  - encode: saturating (|x| > max -> +-max, infinities too), round to
 *    nearest, ties to even, on the exact fp32 value, subnormals included;
 *    NaN -> the canonical NaN code (0x7F e4m3, 0x7E e5m2).
 *  - amax = max |x| over the bf16 tensor, NaN if any element is NaN.
 *  - scale = fp32(fmax / max(amax, 1e-12)) by one IEEE fp32 division;
 *    inv_scale = fp32(1 / scale).  No power-of-two rounding of the scale.
 *  - cast: code = encode(fp32(float(x) * scale)), one fp32 multiply.
 *  - GEMM: C = sum_k dec(A[m,k]) * dec(B[n,k]) in fp64 (stands in for the
 *    exact sum of the FP8 products), times inv_sa then inv_sb in fp64, then
 *    rounded once to bf16, ties to even.
 *  - relu^2 forward: H = bf16(C); h = bf16(relu(H)^2).
 *    relu^2 backward: g = bf16(C); dH = bf16(g * 2 * relu(H)).
 *  - every amax reported next to a GEMM output is the amax of the tensor the
 *    next cast consumes: max|D|, max h, or max|dH|.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fopenmp -shared -fPIC.
 * No fast-math: every fp32 operation above must be a single IEEE operation.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_E4M3 = 0, ORC_E5M2 = 1 };
enum { ORC_EPI_NONE = 0, ORC_EPI_RELU2_FWD = 1, ORC_EPI_RELU2_BWD = 2 };

/* Format parameters from the OCP 8-bit floating point definition. */
typedef struct {
    int ebits, mbits, bias;
    double maxv;       /* largest finite magnitude */
    uint8_t max_code;  /* code of +maxv */
    uint8_t nan_code;  /* canonical +NaN */
} orc_fmt;

static const orc_fmt FMTS[2] = {
    /* E4M3fn: 1.75 * 2^8 = 448 is S.1111.110; S.1111.111 is NaN. */
    {4, 3, 7, 448.0, 0x7E, 0x7F},
    /* E5M2: 1.75 * 2^15 = 57344 is S.11110.11; exponent 11111 is inf/NaN. */
    {5, 2, 15, 57344.0, 0x7B, 0x7E},
};

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---------------------------------------------------------------- codecs */

/* Value of an FP8 code, by the format's definition (sign, biased exponent,
 * mantissa; exponent field 0 is subnormal). */
double orc_fp8_decode(uint8_t code, int fmt) {
    const orc_fmt* F = &FMTS[fmt];
    int sign = code >> 7;
    int e = (code >> F->mbits) & ((1 << F->ebits) - 1);
    int m = code & ((1 << F->mbits) - 1);
    int efield_max = (1 << F->ebits) - 1;
    double v;
    if (fmt == ORC_E4M3 && e == efield_max && m == (1 << F->mbits) - 1) return NAN;
    if (fmt == ORC_E5M2 && e == efield_max) {
        if (m != 0) return NAN;
        return sign ? -INFINITY : INFINITY;
    }
    if (e == 0)
        v = ldexp((double)m, 1 - F->bias - F->mbits);
    else
        v = ldexp((double)((1 << F->mbits) + m), e - F->bias - F->mbits);
    return sign ? -v : v;
}

/* Round a non-negative finite double to the grid of a binary format with
 * `mbits` explicit mantissa bits and minimum normal exponent `emin`,
 * ties to even.  Exact: the division by a power of two is exact and
 * nearbyint() rounds half to even in the default rounding mode. */
static double round_to_grid(double a, int mbits, int emin) {
    int e2;
    if (a == 0.0) return 0.0;
    frexp(a, &e2);            /* a = f * 2^e2, f in [0.5, 1) */
    int ex = e2 - 1;          /* floor(log2(a)) */
    if (ex < emin) ex = emin; /* subnormal range shares the emin quantum */
    double quantum = ldexp(1.0, ex - mbits);
    return nearbyint(a / quantum) * quantum;
}

/* Saturating round-to-nearest-even encode of an fp32 value. */
uint8_t orc_fp8_encode(float x, int fmt) {
    const orc_fmt* F = &FMTS[fmt];
    if (isnan(x)) return F->nan_code;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    int emin = 1 - F->bias;
    if (a > F->maxv) return sign | F->max_code; /* saturate, inf included */
    double r = round_to_grid(a, F->mbits, emin);
    if (r > F->maxv) return sign | F->max_code; /* rounded past max */
    if (r == 0.0) return sign;
    int e2;
    frexp(r, &e2);
    int ex = e2 - 1;
    if (ex < emin) { /* subnormal: exponent field 0 */
        int m = (int)(r / ldexp(1.0, emin - F->mbits));
        return sign | (uint8_t)m;
    }
    int m = (int)(r / ldexp(1.0, ex - F->mbits)) - (1 << F->mbits);
    return sign | (uint8_t)(((ex + F->bias) << F->mbits) | m);
}

/* bf16 value (sign, 8-bit exponent, 7-bit mantissa) as double: the bits are
 * the top half of an IEEE binary32. */
double orc_bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round a double to bf16 once, ties to even (IEEE overflow to infinity).
 * The rounded value is exactly representable in binary32, whose top 16 bits
 * are then the bf16 code. */
uint16_t orc_bf16_from_double(double v) {
    if (isnan(v)) return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0x0000;
    double a = fabs(v);
    double r = round_to_grid(a, 7, -126);
    if (r >= ldexp(1.0, 128)) return sign | 0x7F80; /* infinity */
    float f = (float)r;                              /* exact */
    uint32_t u;
    memcpy(&u, &f, 4);
    return sign | (uint16_t)(u >> 16);
}

/* ------------------------------------------------------- amax / scale / cast */

/* h = bf16(relu(x)^2) for a bf16 x, computed in fp64 then rounded once. */
static uint16_t relu2_bf16(uint16_t xb) {
    double x = orc_bf16_to_double(xb);
    double r = x > 0.0 ? x : 0.0;
    if (isnan(x)) r = x;
    return orc_bf16_from_double(r * r);
}

/* amax over a rows x cols bf16 tensor with leading dimension ld (elements).
 * relu2_input != 0 takes the amax of h = bf16(relu(x)^2) instead of x. */
float orc_amax(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, int relu2_input) {
    double amax = 0.0;
    int any_nan = 0;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            uint16_t b = x[r * ld + c];
            if (relu2_input) b = relu2_bf16(b);
            double v = fabs(orc_bf16_to_double(b));
            if (isnan(v)) any_nan = 1;
            else if (v > amax) amax = v;
        }
    return any_nan ? NAN : (float)amax; /* bf16 -> fp32 is exact */
}

/* scale = fmax / max(amax, 1e-12) in one fp32 division; inv = 1 / scale. */
void orc_scale(float amax, int fmt, float* scale, float* inv_scale) {
    const float fmax = (float)FMTS[fmt].maxv;
    const float floor_amax = 1e-12f;
    float a = (amax < floor_amax) ? floor_amax : amax; /* NaN stays NaN */
    float s = fmax / a;
    *scale = s;
    *inv_scale = 1.0f / s;
}

/* q[r, c] = encode(fp32(float(x[r, c]) * scale)); qT[c, r] = q[r, c].
 * Either output may be NULL.  relu2_input != 0 casts h = bf16(relu(x)^2). */
void orc_cast(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, int fmt,
              int relu2_input, float scale, uint8_t* q, uint8_t* qT) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            uint16_t b = x[r * ld + c];
            if (relu2_input) b = relu2_bf16(b);
            float v = (float)orc_bf16_to_double(b);
            float p = v * scale; /* one fp32 multiply, round to nearest */
            uint8_t code = orc_fp8_encode(p, fmt);
            if (q) q[r * cols + c] = code;
            if (qT) qT[c * rows + r] = code;
        }
}

/* ------------------------------------------------------------------- GEMM */

/* C[i, n] = sum_k dec(A[row_i, k]) * dec(B[n, k]) in fp64, k ascending.
 * A is M x K and B is N x K, both row-major codes ("K-major").  rows == NULL
 * means every row of A in order; otherwise nrows listed row indices. */
void orc_gemm_acc(const uint8_t* A, int fa, const uint8_t* B, int fb, int64_t M, int64_t N,
                  int64_t K, const int64_t* rows, int64_t nrows, double* C) {
    double da[256], db[256];
    for (int c = 0; c < 256; ++c) {
        da[c] = orc_fp8_decode((uint8_t)c, fa);
        db[c] = orc_fp8_decode((uint8_t)c, fb);
    }
    int64_t nr = rows ? nrows : M;
#pragma omp parallel
    {
        double* arow = (double*)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < nr; ++i) {
            int64_t m = rows ? rows[i] : i;
            for (int64_t k = 0; k < K; ++k) arow[k] = da[A[m * K + k]];
            for (int64_t n = 0; n < N; ++n) {
                const uint8_t* b = B + n * K;
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k) acc += arow[k] * db[b[k]];
                C[i * N + n] = acc;
            }
        }
        free(arow);
    }
}

/* D = epi(C * inv_sa * inv_sb) as bf16, for the listed rows (or all rows).
 *  NONE:      D = bf16(C s)                               amax = max |D|
 *  RELU2_FWD: D = H = bf16(C s)                           amax = max bf16(relu(H)^2)
 *  RELU2_BWD: g = bf16(C s); D = bf16(g * 2 * relu(aux))  amax = max |D|
 * aux (RELU2_BWD only) is the saved bf16 H, M x N row-major; for a row subset
 * it is indexed by the original row.  D has nrows (or M) rows of N. */
void orc_gemm(const uint8_t* A, int fa, const uint8_t* B, int fb, int64_t M, int64_t N,
              int64_t K, float inv_sa, float inv_sb, int epi, const uint16_t* aux,
              const int64_t* rows, int64_t nrows, uint16_t* D, float* amax_out) {
    int64_t nr = rows ? nrows : M;
    double* C = (double*)malloc(sizeof(double) * (size_t)(nr * N > 0 ? nr * N : 1));
    orc_gemm_acc(A, fa, B, fb, M, N, K, rows, nrows, C);
    const double s_a = (double)inv_sa, s_b = (double)inv_sb;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nr; ++i) {
        int64_t m = rows ? rows[i] : i;
        for (int64_t n = 0; n < N; ++n) {
            uint16_t y = orc_bf16_from_double(C[i * N + n] * s_a * s_b);
            if (epi == ORC_EPI_RELU2_BWD) {
                double g = orc_bf16_to_double(y);
                double h = orc_bf16_to_double(aux[m * N + n]);
                double rh = h > 0.0 ? h : 0.0;
                y = orc_bf16_from_double(g * 2.0 * rh);
            }
            D[i * N + n] = y;
        }
    }
    free(C);
    if (amax_out) *amax_out = orc_amax(D, nr, N, N, epi == ORC_EPI_RELU2_FWD);
}

/* Gradient accumulation into an fp32 buffer: for the listed rows (or all),
 * D[i, n] = fp32(D[i, n] + fp32(C * inv_sa * inv_sb)): the scaled fp64 sum is
 * rounded once to fp32, then added to the accumulator with one fp32 addition.
 * (Micro-batches, grad_accum 7: decomputer.nl, "Appendix: De configuratie",
 * total_batch_size; section "Vroege experimenten" item 2.) */
void orc_gemm_accum_f32(const uint8_t* A, int fa, const uint8_t* B, int fb, int64_t M,
                        int64_t N, int64_t K, float inv_sa, float inv_sb, const int64_t* rows,
                        int64_t nrows, float* D) {
    int64_t nr = rows ? nrows : M;
    double* C = (double*)malloc(sizeof(double) * (size_t)(nr * N > 0 ? nr * N : 1));
    orc_gemm_acc(A, fa, B, fb, M, N, K, rows, nrows, C);
    const double s_a = (double)inv_sa, s_b = (double)inv_sb;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nr; ++i)
        for (int64_t n = 0; n < N; ++n) {
            float part = (float)(C[i * N + n] * s_a * s_b);
            D[i * N + n] = D[i * N + n] + part; /* one fp32 add */
        }
    free(C);
}

/* RMSNorm producer of the FP8 GEMM input: for each row,
 *   X[r, c] = bf16( R[r, c] / sqrt(mean_c R[r, c]^2 + eps) * w[c] )
 * in fp64, rounded once to bf16 (w == NULL means w = 1).  The model's norm is
 * RMSNorm with rms_norm_eps 1e-6 computed by PyTorch's F.rms_norm
 * (decomputer.nl, "Appendix: De configuratie"; section "Wat niet werkte",
 * Liger RMSNorm bullet). */
void orc_rmsnorm(const uint16_t* R, const uint16_t* w, int64_t rows, int64_t cols, double eps,
                 uint16_t* X) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double ss = 0.0;
        for (int64_t c = 0; c < cols; ++c) {
            double v = orc_bf16_to_double(R[r * cols + c]);
            ss += v * v;
        }
        double inv = 1.0 / sqrt(ss / (double)cols + eps);
        for (int64_t c = 0; c < cols; ++c) {
            double v = orc_bf16_to_double(R[r * cols + c]) * inv;
            if (w) v *= orc_bf16_to_double(w[c]);
            X[r * cols + c] = orc_bf16_from_double(v);
        }
    }
}

/* ------------------------------------------ gated (SwiGLU) MLP variant */
/* The comparison workload of the "Niet-gated MLPs" bullet (decomputer.nl,
 * section "Doorvoer (Throughput) verhogen"): h = silu(G) * U with
 * G = X W_gate^T, U = X W_up^T, silu(x) = x / (1 + exp(-x)).  G, U, h, dG and
 * dU are separate row-major [M x f] tensors here.  Readings: h and dG, dU are
 * each rounded once to bf16 from the exact (fp64) value of the product. */
static double silu(double x) { return x / (1.0 + exp(-x)); }
static double dsilu(double x) {
    double sg = 1.0 / (1.0 + exp(-x));
    return sg * (1.0 + x * (1.0 - sg));
}

/* h [M x f] from G and U [M x f] (bf16 bits); returns the amax of h. */
float orc_swiglu_h(const uint16_t* G, const uint16_t* U, int64_t M, int64_t f, uint16_t* h) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t j = 0; j < f; ++j) {
            double g = orc_bf16_to_double(G[m * f + j]);
            double u = orc_bf16_to_double(U[m * f + j]);
            h[m * f + j] = orc_bf16_from_double(silu(g) * u);
        }
    return orc_amax(h, M, f, f, 0);
}

/* dG = g U silu'(G) and dU = g silu(G) [M x f] from g = dh and G, U [M x f];
 * returns the amax over both (they form one tensor for the next cast). */
float orc_swiglu_bwd(const uint16_t* g_, const uint16_t* G, const uint16_t* U, int64_t M,
                     int64_t f, uint16_t* dG, uint16_t* dU) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t j = 0; j < f; ++j) {
            int64_t i = m * f + j;
            double g = orc_bf16_to_double(g_[i]);
            double gv = orc_bf16_to_double(G[i]), uv = orc_bf16_to_double(U[i]);
            dG[i] = orc_bf16_from_double(g * uv * dsilu(gv));
            dU[i] = orc_bf16_from_double(g * silu(gv));
        }
    float a = orc_amax(dG, M, f, f, 0), b = orc_amax(dU, M, f, f, 0);
    if (a != a || b != b) return a != a ? a : b; /* a NaN amax propagates */
    return a > b ? a : b;
}

/* ----------------------------- softcapped cross-entropy of the LM head */
/* Loss of the run: Liger's fused linear cross-entropy with softcap 15
 * (decomputer.nl, "Het trainen van een 3.8B LLM tot 0.384 CORE voor $998",
 * "Appendix: De configuratie", loss; section "Doorvoer verhogen", fused CE
 * bullet).  For each row r of bf16 logits l (V entries):
 *   z = c tanh(l / c),  lse = log sum_v exp(z_v),  loss_r = lse - z[label_r]
 *   dlogits_v = bf16( (exp(z_v - lse) - [v == label_r]) (1 - (z_v / c)^2) * inv_count )
 * in fp64; inv_count is 1 / (number of tokens) for the mean reduction.  All V
 * columns take part in the softmax (the padded vocabulary rows are ordinary
 * rows of the weight).  Returns the row losses in loss_rows. */
void orc_softcap_ce(const uint16_t* logits, const int32_t* labels, int64_t rows, int64_t V,
                    double c, double inv_count, uint16_t* dlogits, double* loss_rows) {
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t* l = logits + r * V;
        double m = -INFINITY;
        for (int64_t v = 0; v < V; ++v) {
            double z = c * tanh(orc_bf16_to_double(l[v]) / c);
            if (z > m) m = z;
        }
        double sum = 0.0;
        for (int64_t v = 0; v < V; ++v) sum += exp(c * tanh(orc_bf16_to_double(l[v]) / c) - m);
        double lse = m + log(sum);
        double zl = c * tanh(orc_bf16_to_double(l[labels[r]]) / c);
        loss_rows[r] = lse - zl;
        if (dlogits)
            for (int64_t v = 0; v < V; ++v) {
                double z = c * tanh(orc_bf16_to_double(l[v]) / c);
                double p = exp(z - lse) - (v == labels[r] ? 1.0 : 0.0);
                dlogits[r * V + v] = orc_bf16_from_double(p * (1.0 - (z / c) * (z / c)) * inv_count);
            }
    }
}

/* Plain fp64 LM head with the softcapped cross-entropy, no quantisation and
 * no chunking: the sanity reference for the FP8 chunked head, and the
 * function whose gradient is pinned by finite differences of its loss.
 *   l = X W^T [M x V],  z = c tanh(l / c),  loss = mean_r (lse_r - z[r, label_r])
 *   dl = (softmax(z) - onehot) (1 - (z / c)^2) / M
 *   dX = dl W [M x d],  dW = dl^T X [V x d]
 * X: M x d, W: V x d (row-major doubles).  dX and dW may be NULL. */
void orc_lmhead_ce_f64(const double* X, const double* W, const int32_t* labels, int64_t M,
                       int64_t d, int64_t V, double c, double* loss_out, double* dX,
                       double* dW) {
    double* dl = (double*)calloc((size_t)(M * V > 0 ? M * V : 1), sizeof(double));
    double total = 0.0;
    for (int64_t r = 0; r < M; ++r) {
        double* z = dl + r * V; /* holds z first, then dl */
        double m = -INFINITY;
        for (int64_t v = 0; v < V; ++v) {
            double l = 0.0;
            for (int64_t k = 0; k < d; ++k) l += X[r * d + k] * W[v * d + k];
            z[v] = c * tanh(l / c);
            if (z[v] > m) m = z[v];
        }
        double sum = 0.0;
        for (int64_t v = 0; v < V; ++v) sum += exp(z[v] - m);
        double lse = m + log(sum);
        total += lse - z[labels[r]];
        for (int64_t v = 0; v < V; ++v) {
            double p = exp(z[v] - lse) - (v == labels[r] ? 1.0 : 0.0);
            z[v] = p * (1.0 - (z[v] / c) * (z[v] / c)) / (double)M;
        }
    }
    *loss_out = total / (double)M;
    if (dX)
        for (int64_t r = 0; r < M; ++r)
            for (int64_t k = 0; k < d; ++k) {
                double acc = 0.0;
                for (int64_t v = 0; v < V; ++v) acc += dl[r * V + v] * W[v * d + k];
                dX[r * d + k] = acc;
            }
    if (dW)
        for (int64_t v = 0; v < V; ++v)
            for (int64_t k = 0; k < d; ++k) {
                double acc = 0.0;
                for (int64_t r = 0; r < M; ++r) acc += dl[r * V + v] * X[r * d + k];
                dW[v * d + k] = acc;
            }
    free(dl);
}

/* ---------------------------------------------- unquantised fp64 MLP chain */

/* Plain fp64 SwiGLU MLP, no quantisation (same role as orc_mlp_f64):
 *   G = X Wg^T, U = X Wu^T, h = silu(G) U, Y = h Wd^T
 *   dh = dY Wd, dG = dh U silu'(G), dU = dh silu(G)
 *   dX = dG Wg + dU Wu, dWg = dG^T X, dWu = dU^T X, dWd = dY^T h
 * Wg, Wu: f x d; Wd: d x f.  Output pointers may be NULL. */
void orc_swiglu_f64(const double* X, const double* Wg, const double* Wu, const double* Wd,
                    const double* dY, int64_t M, int64_t d, int64_t f, double* Y, double* dX,
                    double* dWg, double* dWu, double* dWd) {
    size_t Mf = (size_t)(M * f > 0 ? M * f : 1);
    double* G = (double*)calloc(Mf, sizeof(double));
    double* U = (double*)calloc(Mf, sizeof(double));
    double* h = (double*)calloc(Mf, sizeof(double));
    double* dG = (double*)calloc(Mf, sizeof(double));
    double* dU = (double*)calloc(Mf, sizeof(double));
    for (int64_t m = 0; m < M; ++m)
        for (int64_t j = 0; j < f; ++j) {
            double a = 0.0, b = 0.0;
            for (int64_t k = 0; k < d; ++k) {
                a += X[m * d + k] * Wg[j * d + k];
                b += X[m * d + k] * Wu[j * d + k];
            }
            G[m * f + j] = a;
            U[m * f + j] = b;
            h[m * f + j] = silu(a) * b;
        }
    if (Y)
        for (int64_t m = 0; m < M; ++m)
            for (int64_t i = 0; i < d; ++i) {
                double acc = 0.0;
                for (int64_t j = 0; j < f; ++j) acc += h[m * f + j] * Wd[i * f + j];
                Y[m * d + i] = acc;
            }
    if (dY) {
        for (int64_t m = 0; m < M; ++m)
            for (int64_t j = 0; j < f; ++j) {
                double acc = 0.0;
                for (int64_t i = 0; i < d; ++i) acc += dY[m * d + i] * Wd[i * f + j];
                dG[m * f + j] = acc * U[m * f + j] * dsilu(G[m * f + j]);
                dU[m * f + j] = acc * silu(G[m * f + j]);
            }
        if (dX)
            for (int64_t m = 0; m < M; ++m)
                for (int64_t k = 0; k < d; ++k) {
                    double acc = 0.0;
                    for (int64_t j = 0; j < f; ++j)
                        acc += dG[m * f + j] * Wg[j * d + k] + dU[m * f + j] * Wu[j * d + k];
                    dX[m * d + k] = acc;
                }
        if (dWg || dWu)
            for (int64_t j = 0; j < f; ++j)
                for (int64_t k = 0; k < d; ++k) {
                    double a = 0.0, b = 0.0;
                    for (int64_t m = 0; m < M; ++m) {
                        a += dG[m * f + j] * X[m * d + k];
                        b += dU[m * f + j] * X[m * d + k];
                    }
                    if (dWg) dWg[j * d + k] = a;
                    if (dWu) dWu[j * d + k] = b;
                }
        if (dWd)
            for (int64_t i = 0; i < d; ++i)
                for (int64_t j = 0; j < f; ++j) {
                    double acc = 0.0;
                    for (int64_t m = 0; m < M; ++m) acc += dY[m * d + i] * h[m * f + j];
                    dWd[i * f + j] = acc;
                }
    }
    free(G);
    free(U);
    free(h);
    free(dG);
    free(dU);
}

/* Plain fp64 relu^2 MLP, no quantisation: the sanity reference that the FP8
 * chain must approach within FP8 error, and whose backward is pinned by
 * finite differences of its forward.
 *   H = X W_up^T, h = relu(H)^2, Y = h W_down^T
 *   dh = dY W_down, dH = dh * 2 relu(H), dX = dH W_up,
 *   dW_down = dY^T h, dW_up = dH^T X
 * X: M x d, W_up: f x d, W_down: d x f, dY: M x d (row-major).  Any output
 * pointer may be NULL. */
void orc_mlp_f64(const double* X, const double* Wu, const double* Wd, const double* dY,
                 int64_t M, int64_t d, int64_t f, double* Y, double* dX, double* dWu,
                 double* dWd) {
    double* H = (double*)calloc((size_t)(M * f > 0 ? M * f : 1), sizeof(double));
    double* h = (double*)calloc((size_t)(M * f > 0 ? M * f : 1), sizeof(double));
    double* dH = (double*)calloc((size_t)(M * f > 0 ? M * f : 1), sizeof(double));
    for (int64_t m = 0; m < M; ++m)
        for (int64_t j = 0; j < f; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < d; ++k) acc += X[m * d + k] * Wu[j * d + k];
            H[m * f + j] = acc;
            double r = acc > 0.0 ? acc : 0.0;
            h[m * f + j] = r * r;
        }
    if (Y)
        for (int64_t m = 0; m < M; ++m)
            for (int64_t i = 0; i < d; ++i) {
                double acc = 0.0;
                for (int64_t j = 0; j < f; ++j) acc += h[m * f + j] * Wd[i * f + j];
                Y[m * d + i] = acc;
            }
    if (dY) {
        for (int64_t m = 0; m < M; ++m)
            for (int64_t j = 0; j < f; ++j) {
                double acc = 0.0;
                for (int64_t i = 0; i < d; ++i) acc += dY[m * d + i] * Wd[i * f + j];
                double r = H[m * f + j] > 0.0 ? H[m * f + j] : 0.0;
                dH[m * f + j] = acc * 2.0 * r;
            }
        if (dX)
            for (int64_t m = 0; m < M; ++m)
                for (int64_t k = 0; k < d; ++k) {
                    double acc = 0.0;
                    for (int64_t j = 0; j < f; ++j) acc += dH[m * f + j] * Wu[j * d + k];
                    dX[m * d + k] = acc;
                }
        if (dWd)
            for (int64_t i = 0; i < d; ++i)
                for (int64_t j = 0; j < f; ++j) {
                    double acc = 0.0;
                    for (int64_t m = 0; m < M; ++m) acc += dY[m * d + i] * h[m * f + j];
                    dWd[i * f + j] = acc;
                }
        if (dWu)
            for (int64_t j = 0; j < f; ++j)
                for (int64_t k = 0; k < d; ++k) {
                    double acc = 0.0;
                    for (int64_t m = 0; m < M; ++m) acc += dH[m * f + j] * X[m * d + k];
                    dWu[j * d + k] = acc;
                }
    }
    free(H);
    free(h);
    free(dH);
}
