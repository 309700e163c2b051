/*
 * mxq_oracle.c -- plain, slow, scalar CPU oracle for the microscaling W4A4 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call this file;
 * only the test suite, the smoke check and the benchmark's CPU-baseline leg use it.  It shares
 * no code, header, table or constant generator with the CUDA library.
 *
 * What it follows (page titles of the reference model cards):
 *   - "Qwen3.5-27B-MXFP4-QAD-W4A4-LR1e-5-s1000", "How this checkpoint was produced", Training row:
 *     MXFP4 = E2M1 elements, block 32, E8M0 shared scale chosen by the EVEN rule (weights), plus
 *     dynamic MXFP4 activation quantization.
 *   - "Qwen3.5-9B-MXFP4-QAD-W4A4-LR1e-5-s3000", "Training mode" paragraph: activations quantized
 *     per token in blocks of 32 E2M1 elements with CEIL-rule UE8M0 scales.
 *   - "Qwen3.5-27B-NVFP4-RTN-weight-only" / "Qwen3.5-27B-NVFP4-GPTQ": NVFP4 = E2M1 elements with
 *     block scales and a per-tensor fp32 global scale (input_global_scale).
 *   - "intel-ai/Qwen3.8-27B-MXFP4-AutoRound", section 1 and section 7: MXFP8 = E4M3 elements with an
 *     E8M0 scale per 32-element group, per the OCP Microscaling Formats (MX) specification.
 * The pages name the EVEN and CEIL rules without formulas; this oracle uses
 *   EVEN:  e = floor(log2 amax) - emax_elem           (OCP MX v1.0 shared-exponent rule)
 *   CEIL:  e = the least integer with amax <= elem_max * 2^e, i.e. ceil(log2(amax / elem_max))
 * with emax_elem = 2, elem_max = 6 for E2M1 and emax_elem = 8, elem_max = 448 for E4M3, e clamped
 * to [-127, 127], an all-zero block taking e = -127.  Elements are rounded to nearest, ties to the
 * even code, and saturate at the largest finite magnitude.
 *
 * NVFP4 (block 16, E4M3 block scale s, fp32 global scale g in the decode direction, x ~ q*s*g)
 * is computed in IEEE fp32 in this order:
 *   t = fl(amax_b / 6);  u = fl(t / g);  s = RNE_E4M3_satfinite(u)   (s = 0 when amax_b = 0)
 *   d = fl(dec(s) * g);  r = fl(1 / d);  v_i = fl(x_i * r);  q_i = RNE_E2M1_sat(v_i)
 * and a block whose d is 0 gets zero-magnitude codes that keep the sign of x.
 *
 * The weight-only (W4A16) GEMM multiplies bf16 activations by dequantized MXFP4 / NVFP4 weights
 * ("Qwen3.5-27B-NVFP4-RTN-weight-only": activations run bf16).
 *
 * Parity status: every function here is pinned by the CPU test suite against library decoders
 * (ml_dtypes, torch), exact rational arithmetic or brute force, except the NVFP4 operation order
 * and the CEIL rule applied to MXFP8, which are readings (the pages do not fix them; MXFP8 under
 * EVEN is the OCP MX rule that the AutoRound card's section 7 cites).
 *
 * Threads: orc_quantize_mt and orc_gemm_mt split the rows (quantizer) or the output columns (GEMM)
 * into contiguous ranges, one per POSIX thread, each running exactly the single-threaded code on its
 * range; every output value is computed by the same operations in the same order as with one
 * thread, so the results do not depend on the thread count.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -pthread -ffp-contract=off -o liboracle.so mxq_oracle.c -lm
 * (no -ffast-math: fp32 steps must be plain IEEE operations).
 */
#define _GNU_SOURCE
#include <math.h>
#include <pthread.h>
#include <sched.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORC_MXFP4 0
#define ORC_NVFP4 1
#define ORC_MXFP8 2
#define ORC_EVEN 0
#define ORC_CEIL 1

/* ---------------------------------------------------------------- element formats */

/* bf16 bit pattern -> exact double (bf16 is the top half of an IEEE binary32). */
double orc_bf16_value(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* A sign + ebits + mbits minifloat with exponent bias `bias`; exponent field 0 is subnormal. */
static double minifloat_value(unsigned code, int ebits, int mbits, int bias) {
    unsigned sign = (code >> (ebits + mbits)) & 1u;
    unsigned ef = (code >> mbits) & ((1u << ebits) - 1u);
    unsigned mf = code & ((1u << mbits) - 1u);
    double mag;
    if (ef == 0)
        mag = ldexp((double)mf, 1 - bias - mbits);
    else
        mag = ldexp(1.0 + ldexp((double)mf, -mbits), (int)ef - bias);
    return sign ? -mag : mag;
}

/* Round |v| to nearest on the minifloat grid (ties to even mantissa), saturating to maxfin. */
static unsigned minifloat_encode(double v, int ebits, int mbits, int bias, double maxfin) {
    unsigned sign = signbit(v) ? 1u : 0u;
    double a = fabs(v);
    int emin = 1 - bias; /* exponent of the smallest normal */
    unsigned mag;
    if (a >= maxfin) {
        a = maxfin;
    }
    int E;
    if (a < ldexp(1.0, emin)) {
        E = emin; /* subnormal range shares the quantum of the first normal binade */
    } else {
        int p;
        (void)frexp(a, &p);
        E = p - 1;
    }
    double quantum = ldexp(1.0, E - mbits);
    double n = rint(a / quantum); /* a / quantum is exact; rint rounds ties to even */
    double r = n * quantum;
    if (r > maxfin) r = maxfin;
    if (r < ldexp(1.0, emin)) {
        mag = (unsigned)(r / ldexp(1.0, emin - mbits)); /* exponent field 0 */
    } else {
        int p;
        (void)frexp(r, &p);
        int Er = p - 1;
        unsigned mf = (unsigned)((r / ldexp(1.0, Er) - 1.0) * (double)(1u << mbits));
        mag = ((unsigned)(Er + bias) << mbits) | mf;
    }
    return (sign << (ebits + mbits)) | mag;
}

/* E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; magnitudes 0,0.5,1,1.5,2,3,4,6. */
double orc_e2m1_value(uint8_t code) { return minifloat_value(code & 0xFu, 2, 1, 1); }

uint8_t orc_e2m1_encode(double v) { return (uint8_t)minifloat_encode(v, 2, 1, 1, 6.0); }

/* E4M3 (the "fn" variant: no infinities, S.1111.111 is NaN, largest finite 448). */
double orc_e4m3_value(uint8_t code) {
    if ((code & 0x7Fu) == 0x7Fu) return NAN;
    return minifloat_value(code, 4, 3, 7);
}

uint8_t orc_e4m3_encode(double v) { return (uint8_t)minifloat_encode(v, 4, 3, 7, 448.0); }

/* E8M0: unsigned power of two 2^(code-127); 0xFF is NaN. */
double orc_e8m0_value(uint8_t code) {
    if (code == 0xFFu) return NAN;
    return ldexp(1.0, (int)code - 127);
}

/* ---------------------------------------------------------------- scale rules */

static int fmt_block(int fmt) { return fmt == ORC_NVFP4 ? 16 : 32; }

/* Shared exponent of one MX block.  elem_emax = exponent of the element format's largest
 * binade (2 for E2M1, 8 for E4M3); elem_max = its largest finite magnitude (6 or 448). */
int orc_mx_exponent(double amax, int elem_emax, double elem_max, int rule) {
    int e;
    if (amax == 0.0) return -127;
    int p;
    (void)frexp(amax, &p);
    int floor_log2 = p - 1; /* amax = f * 2^p with f in [0.5, 1) */
    if (rule == ORC_EVEN) {
        e = floor_log2 - elem_emax;
    } else {
        /* least e with amax <= elem_max * 2^e */
        e = floor_log2 - elem_emax - 1;
        while (amax > ldexp(elem_max, e)) e++;
    }
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

static double block_amax(const uint16_t* x, int64_t n) {
    double amax = 0.0;
    for (int64_t i = 0; i < n; i++) {
        double a = fabs(orc_bf16_value(x[i]));
        if (a > amax) amax = a;
    }
    return amax;
}

/* One NVFP4 block in IEEE fp32, in the order stated in the file header. */
static void nvfp4_block(const uint16_t* x, float g, uint8_t* codes, uint8_t* scale) {
    float amax = (float)block_amax(x, 16);
    uint8_t s = 0;
    if (amax != 0.0f) {
        volatile float t = amax / 6.0f;
        volatile float u = t / g;
        s = orc_e4m3_encode((double)u);
    }
    volatile float d = (float)orc_e4m3_value(s) * g;
    for (int i = 0; i < 16; i++) {
        double xv = orc_bf16_value(x[i]);
        if (d == 0.0f) {
            codes[i] = signbit(xv) ? 0x8u : 0x0u;
        } else {
            volatile float r = 1.0f / d;
            /* r overflows to +inf when d < 2^-128 (a subnormal g): x * r is then +-inf for x != 0
             * (saturating to +-6) and NaN for x = 0, which has no E2M1 code; a zero element
             * encodes as a zero with its sign, whatever the scale. */
            volatile float v = xv == 0.0 ? (float)xv : (float)xv * r;
            codes[i] = orc_e2m1_encode((double)v);
        }
    }
    *scale = s;
}

/* Quantize a row-major bf16 matrix x[rows][K] along K.
 *   q:  MXFP4/NVFP4 -> rows*K/2 bytes, element 2i in the low nibble of byte i;
 *       MXFP8       -> rows*K bytes of E4M3 codes.
 *   sf: rows*(K/bs) scale bytes, row-major (E8M0 codes for MX, E4M3 codes for NVFP4).
 *   g:  NVFP4 global scale (decode direction); ignored otherwise.
 * Returns 0, or -1 if K is not a multiple of the block size. */
int orc_quantize(const uint16_t* x, int64_t rows, int64_t K, int fmt, int rule, float g,
                 uint8_t* q, uint8_t* sf) {
    int bs = fmt_block(fmt);
    if (K % bs != 0) return -1;
    int64_t kb = K / bs;
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t b = 0; b < kb; b++) {
            const uint16_t* xb = x + r * K + b * bs;
            uint8_t codes[32];
            if (fmt == ORC_NVFP4) {
                nvfp4_block(xb, g, codes, &sf[r * kb + b]);
            } else {
                int elem_emax = fmt == ORC_MXFP8 ? 8 : 2;
                double elem_max = fmt == ORC_MXFP8 ? 448.0 : 6.0;
                int e = orc_mx_exponent(block_amax(xb, bs), elem_emax, elem_max, rule);
                sf[r * kb + b] = (uint8_t)(e + 127);
                for (int i = 0; i < bs; i++) {
                    double v = ldexp(orc_bf16_value(xb[i]), -e); /* exact */
                    codes[i] = fmt == ORC_MXFP8 ? orc_e4m3_encode(v) : orc_e2m1_encode(v);
                }
            }
            for (int i = 0; i < bs; i++) {
                int64_t k = b * bs + i;
                if (fmt == ORC_MXFP8) {
                    q[r * K + k] = codes[i];
                } else {
                    uint8_t* byte = &q[(r * K + k) / 2];
                    if (k % 2 == 0)
                        *byte = (uint8_t)((*byte & 0xF0u) | codes[i]);
                    else
                        *byte = (uint8_t)((*byte & 0x0Fu) | (codes[i] << 4));
                }
            }
        }
    }
    return 0;
}

/* ---------------------------------------------------------------- threads */

/* Logical CPUs this process may run on (its affinity mask), and the host's online CPU count. */
int orc_cpus_usable(void) {
    cpu_set_t set;
    CPU_ZERO(&set);
    if (sched_getaffinity(0, sizeof set, &set) == 0) {
        int n = CPU_COUNT(&set);
        if (n > 0) return n;
    }
    return 1;
}

int orc_cpus_online(void) {
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

typedef struct {
    const uint16_t* x;
    int64_t rows, K;
    int fmt, rule;
    float g;
    uint8_t *q, *sf;
    int rc;
} quant_job;

static void* quant_worker(void* arg) {
    quant_job* j = (quant_job*)arg;
    j->rc = orc_quantize(j->x, j->rows, j->K, j->fmt, j->rule, j->g, j->q, j->sf);
    return NULL;
}

/* orc_quantize over `nthreads` POSIX threads, each quantizing a contiguous range of rows (rows are
 * independent).  Same bytes as orc_quantize.  Returns 0, or -1 as orc_quantize, or -2 when a
 * thread cannot be created. */
int orc_quantize_mt(const uint16_t* x, int64_t rows, int64_t K, int fmt, int rule, float g, uint8_t* q,
                    uint8_t* sf, int nthreads) {
    int bs = fmt_block(fmt);
    if (K % bs != 0) return -1;
    if (nthreads > rows) nthreads = (int)rows;
    if (nthreads <= 1) return orc_quantize(x, rows, K, fmt, rule, g, q, sf);
    int64_t qrow = fmt == ORC_MXFP8 ? K : K / 2, kb = K / bs;
    quant_job* jobs = (quant_job*)calloc((size_t)nthreads, sizeof(quant_job));
    pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !th) {
        free(jobs);
        free(th);
        return -2;
    }
    int started = 0, rc = 0;
    for (int t = 0; t < nthreads; t++) {
        int64_t r0 = rows * t / nthreads, r1 = rows * (t + 1) / nthreads;
        quant_job j = {x + r0 * K, r1 - r0, K, fmt, rule, g, q + r0 * qrow, sf + r0 * kb, 0};
        jobs[t] = j;
        if (pthread_create(&th[t], NULL, quant_worker, &jobs[t]) != 0) {
            rc = -2;
            break;
        }
        started++;
    }
    for (int t = 0; t < started; t++) {
        pthread_join(th[t], NULL);
        if (jobs[t].rc != 0 && rc == 0) rc = jobs[t].rc;
    }
    free(jobs);
    free(th);
    return rc;
}

/* Decoded value of element (r, k) of a quantized matrix, without the NVFP4 global scale. */
static double dq_elem(const uint8_t* q, const uint8_t* sf, int64_t r, int64_t k, int64_t K, int fmt) {
    int bs = fmt_block(fmt);
    int64_t kb = K / bs;
    uint8_t s = sf[r * kb + k / bs];
    double scale = fmt == ORC_NVFP4 ? orc_e4m3_value(s) : orc_e8m0_value(s);
    double elem;
    if (fmt == ORC_MXFP8) {
        elem = orc_e4m3_value(q[r * K + k]);
    } else {
        uint8_t byte = q[(r * K + k) / 2];
        elem = orc_e2m1_value(k % 2 == 0 ? (byte & 0xFu) : (byte >> 4));
    }
    return elem * scale;
}

/* Dequantize to double: out[r][k] = elem * block_scale (* g for NVFP4). */
void orc_dequantize(const uint8_t* q, const uint8_t* sf, int64_t rows, int64_t K, int fmt, double g,
                    double* out) {
    for (int64_t r = 0; r < rows; r++)
        for (int64_t k = 0; k < K; k++) {
            double v = dq_elem(q, sf, r, k, K, fmt);
            out[r * K + k] = fmt == ORC_NVFP4 ? v * g : v;
        }
}

/* ---------------------------------------------------------------- scale layout */

/* Byte offset of scale (r, c) in the tensor-core scale layout: 128-row x 4-column tiles of 512 B,
 * tiles ordered row-tile major, inside a tile row r at (r%32)*16 + ((r%128)/32)*4 + c%4. */
int64_t orc_swizzle_offset(int64_t r, int64_t c, int64_t kblocks) {
    int64_t col_tiles = (kblocks + 3) / 4;
    return ((r / 128) * col_tiles + c / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);
}

int64_t orc_swizzled_bytes(int64_t rows, int64_t kblocks) {
    return ((rows + 127) / 128) * 128 * ((kblocks + 3) / 4) * 4;
}

void orc_swizzle(const uint8_t* sf, int64_t rows, int64_t kblocks, uint8_t* out) {
    memset(out, 0, (size_t)orc_swizzled_bytes(rows, kblocks));
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < kblocks; c++) out[orc_swizzle_offset(r, c, kblocks)] = sf[r * kblocks + c];
}

void orc_unswizzle(const uint8_t* sw, int64_t rows, int64_t kblocks, uint8_t* sf) {
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < kblocks; c++) sf[r * kblocks + c] = sw[orc_swizzle_offset(r, c, kblocks)];
}

/* ---------------------------------------------------------------- global scale */

/* NVFP4 per-tensor global scale in the decode direction: fl(amax / (6 * 448)) in fp32. */
float orc_global_scale(const uint16_t* x, int64_t n, float* amax_out) {
    float amax = (float)block_amax(x, n);
    volatile float g = amax / 2688.0f;
    if (amax_out) *amax_out = amax;
    return g;
}

/* ---------------------------------------------------------------- GEMM */

/* Out[i][j] = alpha * sum_k dq(A)[rows[i]][k] * dq(B)[cols[j]][k] in fp64, alpha = gA*gB for
 * NVFP4 and 1 otherwise; abs_out[i][j] = |alpha| * sum_k |dq(A) dq(B)|.  A is [M][K], B is [N][K]
 * (nn.Linear layout), both quantized along K with row-major scales.  rows / cols select which
 * outputs to compute (pass NULL for all).  Each sum runs over k in increasing order. */
typedef struct {
    const uint8_t *Bq, *Bsf;
    const double* arow; /* dequantized selected A rows, [nrows][K] */
    const int64_t* cols;
    int64_t K, nrows, ncols, j0, j1;
    int fmt;
    double alpha;
    double *out, *abs_out;
    int rc;
} gemm_job;

static void* gemm_cols(void* arg) {
    gemm_job* g = (gemm_job*)arg;
    int64_t K = g->K;
    double* brow = (double*)malloc(sizeof(double) * (size_t)K);
    if (!brow) {
        g->rc = -1;
        return NULL;
    }
    for (int64_t j = g->j0; j < g->j1; j++) {
        int64_t n = g->cols ? g->cols[j] : j;
        for (int64_t k = 0; k < K; k++) brow[k] = dq_elem(g->Bq, g->Bsf, n, k, K, g->fmt);
        for (int64_t i = 0; i < g->nrows; i++) {
            double acc = 0.0, aacc = 0.0;
            const double* a = g->arow + i * K;
            for (int64_t k = 0; k < K; k++) {
                double p = a[k] * brow[k];
                acc += p;
                aacc += fabs(p);
            }
            g->out[i * g->ncols + j] = g->alpha * acc;
            if (g->abs_out) g->abs_out[i * g->ncols + j] = fabs(g->alpha) * aacc;
        }
    }
    free(brow);
    g->rc = 0;
    return NULL;
}

/* The GEMM over `nthreads` POSIX threads, each taking a contiguous range of the selected output
 * columns.  Returns 0, or -1 when memory runs out or a thread cannot be created. */
int orc_gemm_mt(const uint8_t* Aq, const uint8_t* Asf, const uint8_t* Bq, const uint8_t* Bsf, double gA,
                double gB, int64_t M, int64_t N, int64_t K, int fmt, const int64_t* rows, int64_t nrows,
                const int64_t* cols, int64_t ncols, double* out, double* abs_out, int nthreads) {
    double alpha = fmt == ORC_NVFP4 ? gA * gB : 1.0;
    if (!rows) nrows = M;
    if (!cols) ncols = N;
    if (nthreads > ncols) nthreads = (int)ncols;
    if (nthreads < 1) nthreads = 1;
    double* arow = (double*)malloc(sizeof(double) * (size_t)(nrows * K));
    gemm_job* jobs = (gemm_job*)calloc((size_t)nthreads, sizeof(gemm_job));
    pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!arow || !jobs || !th) {
        free(arow);
        free(jobs);
        free(th);
        return -1;
    }
    for (int64_t i = 0; i < nrows; i++) {
        int64_t m = rows ? rows[i] : i;
        for (int64_t k = 0; k < K; k++) arow[i * K + k] = dq_elem(Aq, Asf, m, k, K, fmt);
    }
    int rc = 0, started = 0;
    for (int t = 0; t < nthreads; t++) {
        gemm_job j = {Bq, Bsf, arow, cols, K, nrows, ncols, ncols * t / nthreads, ncols * (t + 1) / nthreads,
                      fmt, alpha, out, abs_out, 0};
        jobs[t] = j;
    }
    if (nthreads == 1) {
        gemm_cols(&jobs[0]);
        rc = jobs[0].rc;
    } else {
        for (int t = 0; t < nthreads; t++) {
            if (pthread_create(&th[t], NULL, gemm_cols, &jobs[t]) != 0) {
                rc = -1;
                break;
            }
            started++;
        }
        for (int t = 0; t < started; t++) {
            pthread_join(th[t], NULL);
            if (jobs[t].rc != 0) rc = -1;
        }
    }
    free(arow);
    free(jobs);
    free(th);
    return rc;
}

/* The GEMM on one thread.  Returns 0, or -1 when memory runs out. */
int orc_gemm(const uint8_t* Aq, const uint8_t* Asf, const uint8_t* Bq, const uint8_t* Bsf, double gA,
             double gB, int64_t M, int64_t N, int64_t K, int fmt, const int64_t* rows, int64_t nrows,
             const int64_t* cols, int64_t ncols, double* out, double* abs_out) {
    return orc_gemm_mt(Aq, Asf, Bq, Bsf, gA, gB, M, N, K, fmt, rows, nrows, cols, ncols, out, abs_out, 1);
}

/* Weight-only (W4A16) GEMM, the serving mode of "Qwen3.5-27B-NVFP4-RTN-weight-only" (first paragraph:
 * the checkpoint's weights are NVFP4, activations run bf16) and the Marlin mode of
 * "Qwen3.5-27B-MXFP4-QAD-W4A4-LR1e-5-s1000" ("Evaluation results": one artifact serves W4A4 and
 * W4A16).  Out[i][j] = alpha * sum_k bf16(A[rows[i]][k]) * dq(B)[cols[j]][k] in fp64, alpha = gB for
 * NVFP4 and 1 otherwise; abs_out likewise with |.|.  A is [M][K] bf16 bit patterns, B [N][K]
 * quantized along K with row-major scales (MXFP4 or NVFP4).  Returns 0, or -1 when memory runs out. */
int orc_gemm_w4a16(const uint16_t* A, const uint8_t* Bq, const uint8_t* Bsf, double gB, int64_t M, int64_t N,
                   int64_t K, int fmt, const int64_t* rows, int64_t nrows, const int64_t* cols, int64_t ncols,
                   double* out, double* abs_out) {
    double alpha = fmt == ORC_NVFP4 ? gB : 1.0;
    if (!rows) nrows = M;
    if (!cols) ncols = N;
    double* arow = (double*)malloc(sizeof(double) * (size_t)(nrows * K));
    double* brow = (double*)malloc(sizeof(double) * (size_t)K);
    if (!arow || !brow) {
        free(arow);
        free(brow);
        return -1;
    }
    for (int64_t i = 0; i < nrows; i++) {
        int64_t m = rows ? rows[i] : i;
        for (int64_t k = 0; k < K; k++) arow[i * K + k] = orc_bf16_value(A[m * K + k]);
    }
    for (int64_t j = 0; j < ncols; j++) {
        int64_t n = cols ? cols[j] : j;
        for (int64_t k = 0; k < K; k++) brow[k] = dq_elem(Bq, Bsf, n, k, K, fmt);
        for (int64_t i = 0; i < nrows; i++) {
            double acc = 0.0, aacc = 0.0;
            const double* a = arow + i * K;
            for (int64_t k = 0; k < K; k++) {
                double p = a[k] * brow[k];
                acc += p;
                aacc += fabs(p);
            }
            out[i * ncols + j] = alpha * acc;
            if (abs_out) abs_out[i * ncols + j] = fabs(alpha) * aacc;
        }
    }
    free(arow);
    free(brow);
    return 0;
}

/* ---------------------------------------------------------------- fake quantization */

/* fp32 -> bf16 bit pattern with round to nearest, ties to even (finite inputs; overflow -> inf). */
uint16_t orc_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint32_t r = u + 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(r >> 16);
}

/* Quantize-then-dequantize x[rows][K] (bf16) into bf16 out[rows][K] -- the fake-quantized forward
 * of quantization-aware training ("Qwen3.5-9B-MXFP4-QAD-W4A4-LR1e-5-s3000", "Training mode": the
 * training fake-quant is bit-identical to the serving quantizer).  Each element is decoded in its
 * format's own precision and rounded once to bf16:
 *   MX:    v = elem * 2^e, exact in fp64, then fp32 (exact unless it overflows) and bf16 RNE;
 *   NVFP4: v = fl32(elem * d) with d = fl32(dec(s) * g), the same d the encoder used, then bf16 RNE.
 * Returns 0, or -1 if K is not a multiple of the block size or memory runs out. */
int orc_fake_quantize(const uint16_t* x, int64_t rows, int64_t K, int fmt, int rule, float g, uint16_t* out) {
    int bs = fmt_block(fmt);
    if (K % bs != 0) return -1;
    int64_t qrow = fmt == ORC_MXFP8 ? K : K / 2;
    uint8_t* q = (uint8_t*)malloc((size_t)(rows * qrow));
    uint8_t* sf = (uint8_t*)malloc((size_t)(rows * (K / bs)));
    if (!q || !sf) {
        free(q);
        free(sf);
        return -1;
    }
    memset(q, 0, (size_t)(rows * qrow));
    orc_quantize(x, rows, K, fmt, rule, g, q, sf);
    for (int64_t r = 0; r < rows; r++)
        for (int64_t k = 0; k < K; k++) {
            uint8_t s = sf[r * (K / bs) + k / bs];
            double elem;
            if (fmt == ORC_MXFP8) {
                elem = orc_e4m3_value(q[r * K + k]);
            } else {
                uint8_t byte = q[(r * K + k) / 2];
                elem = orc_e2m1_value(k % 2 == 0 ? (byte & 0xFu) : (byte >> 4));
            }
            float v;
            if (fmt == ORC_NVFP4) {
                volatile float d = (float)orc_e4m3_value(s) * g;
                volatile float prod = (float)elem * d;
                v = prod;
            } else {
                v = (float)(elem * orc_e8m0_value(s));
            }
            out[r * K + k] = orc_f32_to_bf16(v);
        }
    free(q);
    free(sf);
    return 0;
}

/* ---------------------------------------------------------------- running-max observer */

/* NVFP4 quantization with a running-max global scale ("Qwen3.5-27B-NVFP4-GPTQ", Serving-KL table:
 * running-max input scales): g = fl(amax_in / 2688), codes and scales as orc_quantize with that g,
 * and *amax_out = max(amax_in, max |x|).  Returns orc_quantize's status. */
int orc_quantize_running(const uint16_t* x, int64_t rows, int64_t K, float amax_in, float* amax_out, uint8_t* q,
                         uint8_t* sf) {
    volatile float g = amax_in / 2688.0f;
    float a = (float)block_amax(x, rows * K);
    *amax_out = a > amax_in ? a : amax_in;
    return orc_quantize(x, rows, K, ORC_NVFP4, 0, g, q, sf);
}
