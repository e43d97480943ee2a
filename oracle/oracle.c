/*
 * CPU oracle for the block-scaled GEMM D = A * B^T and the UE8M0 scale-factor
 * packing.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the bench's
 * CPU-baseline leg call it; the CUDA library never does, and this file shares no
 * code, header or table with it.
 *
 * Everything here is the plain definition, in fp64, one output element at a time:
 *
 *   FP8  (DeepGEMM-Ascend coverage list: "Cobertura de operações" on the
 *        crazystack.com.br page; scale factors: "Fatores de escala FP8 e o
 *        formato UE8M0" on the same page):
 *        D[m,n] = sum_kb 2^(ea[m,kb]-127) * 2^(eb[n/gn,kb]-127)
 *                        * sum_{k in block kb} e4m3(A[m,k]) * e4m3(B[n,k])
 *        with 128-wide K blocks, A scales per (row, block), B scales per
 *        (gn rows, block) (gn = 128 for 128x128 weight blocks, 1 for per-row).
 *   FP4  the same with E2M1 values (two per byte, even K index in the low nibble)
 *        and 32-wide K blocks, scales per (row, block) for A and B.
 *   BF16 D[m,n] = sum_k bf16(A[m,k]) * bf16(B[n,k]).
 *   Grouped (MoE, "Execução de MoE" on the aireiter.com page): row m uses expert
 *        g = m_indices[m] (B := B[g], SFB := SFB[g]); rows with g = -1 are 0.
 *   Masked grouped (the decode-time MoE layout the crazystack page lists as not
 *        implemented, "Cobertura de operações e a lacuna declarada no repositório"):
 *        expert g owns rows [0, max_m) of its own slab of A and D; only rows
 *        m < masked_m[g] are products, D[g][m] = FP8 formula with B := B[g],
 *        SFB := SFB[g]; the other rows are not part of the result.
 *   SF packing ("Qué incluye" on the bigchange.ai/es page; "Fatores de escala"
 *        on the crazystack page): each pair of UE8M0 bytes along K goes into one
 *        16-bit word, stored MN-major: out[j*ld + mn] = e[mn][2j] | e[mn][2j+1] << 8.
 *        Reading (the pages give no byte order): the lower K block sits in the
 *        low byte; mn >= MN and the missing high byte of an odd count are 0.
 *   Quantiser ("Fatores de escala FP8 e o formato UE8M0" on the crazystack page:
 *        one power-of-two scale per block, so that the block fits the FP8 range):
 *        per block of block_rows x 128 values, e = the smallest integer with
 *        448 * 2^e >= max |x| (0 for an all-zero block), clamped to [-126, 127],
 *        stored as the UE8M0 byte e + 127; each value becomes x / 2^e rounded to
 *        the nearest E4M3 value, ties to the even code, sign kept (also for a
 *        zero result), magnitudes above 448 saturated.
 *
 * Decode tables are built from each format's bit fields (sign, exponent,
 * mantissa), not typed in.  For FP8 every product has at most 8 significant
 * bits and a 128-term block sum fits in 53 bits, so the fp64 block sums are exact.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double T_E4M3[256];
static double T_E2M1[16];
static double T_UE8M0[256];
static int tables_ready = 0;

/* E4M3 "FN" (finite) format: 1 sign, 4 exponent (bias 7), 3 mantissa bits;
 * exponent field 0 is subnormal (2^-6 * m/8); S.1111.111 is NaN; no infinity. */
static double decode_e4m3(unsigned code) {
    unsigned s = (code >> 7) & 1u, e = (code >> 3) & 0xFu, m = code & 7u;
    double v;
    if (e == 15u && m == 7u) return NAN;
    if (e == 0u) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, (int)e - 7);
    return s ? -v : v;
}

/* E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; exponent 0 is subnormal
 * (m * 0.5); no NaN or infinity. */
static double decode_e2m1(unsigned code) {
    unsigned s = (code >> 3) & 1u, e = (code >> 1) & 3u, m = code & 1u;
    double v;
    if (e == 0u) v = 0.5 * (double)m;
    else v = ldexp(1.0 + (double)m / 2.0, (int)e - 1);
    return s ? -v : v;
}

/* UE8M0: 8-bit unsigned exponent, bias 127, no mantissa; 0xFF is NaN. */
static double decode_ue8m0(unsigned code) {
    if (code == 255u) return NAN;
    return ldexp(1.0, (int)code - 127);
}

static double decode_bf16(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static void build_tables(void) {
    if (tables_ready) return;
    for (unsigned c = 0; c < 256; ++c) {
        T_E4M3[c] = decode_e4m3(c);
        T_UE8M0[c] = decode_ue8m0(c);
    }
    for (unsigned c = 0; c < 16; ++c) T_E2M1[c] = decode_e2m1(c);
    tables_ready = 1;
}

void oracle_tables(double* e4m3, double* e2m1, double* ue8m0) {
    build_tables();
    memcpy(e4m3, T_E4M3, sizeof T_E4M3);
    memcpy(e2m1, T_E2M1, sizeof T_E2M1);
    memcpy(ue8m0, T_UE8M0, sizeof T_UE8M0);
}

/* ---------------------------------------------------------------- SF packing */

int oracle_sf_pack(const uint8_t* e, int mn, int kb, int64_t ld_in, uint16_t* out, int64_t ld_out) {
    if (mn < 0 || kb < 0 || ld_in < kb || ld_out < mn) return -1;
    int pairs = (kb + 1) / 2;
    for (int j = 0; j < pairs; ++j) {
        for (int64_t r = 0; r < ld_out; ++r) {
            uint16_t v = 0;
            if (r < mn) {
                unsigned lo = e[r * ld_in + 2 * j];
                unsigned hi = (2 * j + 1 < kb) ? e[r * ld_in + 2 * j + 1] : 0u;
                v = (uint16_t)(lo | (hi << 8));
            }
            out[(int64_t)j * ld_out + r] = v;
        }
    }
    return 0;
}

int oracle_sf_unpack(const uint16_t* in, int mn, int kb, int64_t ld_in, uint8_t* e, int64_t ld_out) {
    if (mn < 0 || kb < 0 || ld_in < mn || ld_out < kb) return -1;
    for (int r = 0; r < mn; ++r) {
        for (int k = 0; k < kb; ++k) {
            uint16_t w = in[(int64_t)(k / 2) * ld_in + r];
            e[(int64_t)r * ld_out + k] = (uint8_t)((k % 2) ? (w >> 8) : (w & 0xFF));
        }
    }
    return 0;
}

/* fp32 power-of-two scales -> biased UE8M0 exponent bytes.  Only exact positive
 * normal powers of two are accepted (anything else returns -1). */
int oracle_fp32_scales_to_ue8m0(const float* s, int64_t count, uint8_t* e) {
    for (int64_t i = 0; i < count; ++i) {
        int ex;
        double f = frexp((double)s[i], &ex); /* s = f * 2^ex, f in [0.5, 1) */
        if (!(s[i] > 0.0f) || !isfinite(s[i]) || f != 0.5) return -1;
        int biased = ex - 1 + 127;
        if (biased < 1 || biased > 254) return -1;
        e[i] = (uint8_t)biased;
    }
    return 0;
}

/* fp64 -> bf16 bit pattern with a single round-to-nearest-even step. */
static uint16_t round_bf16(double x) {
    if (isnan(x)) return 0x7FC0;
    double q;
    if (x == 0.0) {
        q = x;
    } else {
        int ex;
        frexp(x, &ex); /* |x| in [2^(ex-1), 2^ex) */
        int lsb = (ex - 1 < -126) ? -133 : ex - 8; /* 8 significant bits, subnormal floor 2^-133 */
        q = ldexp(rint(ldexp(x, -lsb)), lsb);
    }
    if (fabs(q) >= ldexp(1.0, 128)) return (uint16_t)(q < 0 ? 0xFF80 : 0x7F80);
    float f = (float)q; /* exact: q has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

void oracle_bf16_round(const double* x, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = round_bf16(x[i]);
}

/* ------------------------------------------------------------------- GEMMs
 * rows/cols select the output elements (NULL = all); out is [nrows][ncols]. */

static double dot_fp8(const uint8_t* a, const uint8_t* sa, const uint8_t* b, const uint8_t* sb, int K) {
    double acc = 0.0;
    for (int kb = 0; kb < K / 128; ++kb) {
        double s = 0.0;
        for (int k = kb * 128; k < kb * 128 + 128; ++k) s += T_E4M3[a[k]] * T_E4M3[b[k]];
        acc += T_UE8M0[sa[kb]] * T_UE8M0[sb[kb]] * s;
    }
    return acc;
}

int oracle_gemm_fp8(const uint8_t* A, const uint8_t* sfa, const uint8_t* B, const uint8_t* sfb,
                    int gran_n, int M, int N, int K, const int32_t* rows, int nrows,
                    const int32_t* cols, int ncols, double* out) {
    if (K % 128 || gran_n < 1 || M < 0 || N < 0) return -1;
    build_tables();
    int R = rows ? nrows : M, C = cols ? ncols : N, KB = K / 128;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < R; ++i) {
        int m = rows ? rows[i] : i;
        for (int j = 0; j < C; ++j) {
            int n = cols ? cols[j] : j;
            out[(int64_t)i * C + j] = dot_fp8(A + (int64_t)m * K, sfa + (int64_t)m * KB,
                                              B + (int64_t)n * K, sfb + (int64_t)(n / gran_n) * KB, K);
        }
    }
    return 0;
}

int oracle_gemm_fp4(const uint8_t* A, const uint8_t* sfa, const uint8_t* B, const uint8_t* sfb,
                    int M, int N, int K, const int32_t* rows, int nrows,
                    const int32_t* cols, int ncols, double* out) {
    if (K % 32 || M < 0 || N < 0) return -1;
    build_tables();
    int R = rows ? nrows : M, C = cols ? ncols : N, KB = K / 32;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < R; ++i) {
        int m = rows ? rows[i] : i;
        const uint8_t* a = A + (int64_t)m * (K / 2);
        for (int j = 0; j < C; ++j) {
            int n = cols ? cols[j] : j;
            const uint8_t* b = B + (int64_t)n * (K / 2);
            double acc = 0.0;
            for (int kb = 0; kb < KB; ++kb) {
                double s = 0.0;
                for (int k = kb * 32; k < kb * 32 + 32; ++k) {
                    unsigned ca = (a[k / 2] >> ((k % 2) * 4)) & 0xFu;
                    unsigned cb = (b[k / 2] >> ((k % 2) * 4)) & 0xFu;
                    s += T_E2M1[ca] * T_E2M1[cb];
                }
                acc += T_UE8M0[sfa[(int64_t)m * KB + kb]] * T_UE8M0[sfb[(int64_t)n * KB + kb]] * s;
            }
            out[(int64_t)i * C + j] = acc;
        }
    }
    return 0;
}

int oracle_gemm_bf16(const uint16_t* A, const uint16_t* B, int M, int N, int K,
                     const int32_t* rows, int nrows, const int32_t* cols, int ncols, double* out) {
    if (M < 0 || N < 0 || K < 0) return -1;
    int R = rows ? nrows : M, C = cols ? ncols : N;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < R; ++i) {
        int m = rows ? rows[i] : i;
        for (int j = 0; j < C; ++j) {
            int n = cols ? cols[j] : j;
            double acc = 0.0;
            for (int k = 0; k < K; ++k)
                acc += decode_bf16(A[(int64_t)m * K + k]) * decode_bf16(B[(int64_t)n * K + k]);
            out[(int64_t)i * C + j] = acc;
        }
    }
    return 0;
}

int oracle_gemm_grouped_fp8(const uint8_t* A, const uint8_t* sfa, const uint8_t* B, const uint8_t* sfb,
                            const int32_t* m_indices, int gran_n, int G, int M, int N, int K,
                            const int32_t* rows, int nrows, const int32_t* cols, int ncols, double* out) {
    if (K % 128 || gran_n < 1 || G < 1 || M < 0 || N < 0) return -1;
    build_tables();
    int R = rows ? nrows : M, C = cols ? ncols : N, KB = K / 128, NB = (N + gran_n - 1) / gran_n;
    for (int i = 0; i < R; ++i) {
        int g = m_indices[rows ? rows[i] : i];
        if (g < -1 || g >= G) return -1;
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < R; ++i) {
        int m = rows ? rows[i] : i;
        int g = m_indices[m];
        for (int j = 0; j < C; ++j) {
            int n = cols ? cols[j] : j;
            double v = 0.0;
            if (g >= 0) {
                const uint8_t* Bg = B + (int64_t)g * N * K;
                const uint8_t* sbg = sfb + (int64_t)g * NB * KB;
                v = dot_fp8(A + (int64_t)m * K, sfa + (int64_t)m * KB, Bg + (int64_t)n * K,
                            sbg + (int64_t)(n / gran_n) * KB, K);
            }
            out[(int64_t)i * C + j] = v;
        }
    }
    return 0;
}

/* Masked grouped FP8: A [G][max_m][K], sfa [G*max_m][K/128], B [G][N][K],
 * sfb [G][ceil(N/gran_n)][K/128], masked_m [G] with 0 <= masked_m[g] <= max_m.
 * out [G][max_m][N]: the products for m < masked_m[g]; rows past masked_m[g] are
 * set to NAN (not part of the result).  rows (NULL = all) selects rows of the
 * flattened [G*max_m] row index; cols selects columns. */
int oracle_gemm_masked_fp8(const uint8_t* A, const uint8_t* sfa, const uint8_t* B, const uint8_t* sfb,
                           const int32_t* masked_m, int gran_n, int G, int max_m, int N, int K,
                           const int32_t* rows, int nrows, const int32_t* cols, int ncols, double* out) {
    if (K % 128 || gran_n < 1 || G < 1 || max_m < 0 || N < 0) return -1;
    for (int g = 0; g < G; ++g)
        if (masked_m[g] < 0 || masked_m[g] > max_m) return -1;
    build_tables();
    int R = rows ? nrows : G * max_m, C = cols ? ncols : N, KB = K / 128, NB = (N + gran_n - 1) / gran_n;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < R; ++i) {
        int r = rows ? rows[i] : i;
        int g = r / max_m, m = r % max_m;
        for (int j = 0; j < C; ++j) {
            int n = cols ? cols[j] : j;
            double v = NAN;
            if (m < masked_m[g])
                v = dot_fp8(A + (int64_t)r * K, sfa + (int64_t)r * KB, B + ((int64_t)g * N + n) * K,
                            sfb + ((int64_t)g * NB + n / gran_n) * KB, K);
            out[(int64_t)i * C + j] = v;
        }
    }
    return 0;
}

/* --------------------------------------------------------------- quantiser */

/* Smallest integer e with qmax * 2^e >= amax (0 for amax == 0): an exact search
 * upward from a start at least one binade too low. */
static int exponent_for_amax(double amax, double qmax) {
    if (amax == 0.0) return 0;
    int ex, eq;
    frexp(amax, &ex); /* amax in [2^(ex-1), 2^ex) */
    frexp(qmax, &eq); /* qmax in [2^(eq-1), 2^eq) */
    int e = ex - eq - 1;
    while (ldexp(qmax, e) < amax) ++e;
    return e;
}

/* Finite v -> E4M3 (FN) code, round to nearest with ties to the even code.  The value
 * grid of a binade [2^E, 2^(E+1)) has spacing 2^(E-3) for E >= -6 and 2^-9 below
 * (subnormals), so rint(|v| / spacing) picks the nearest grid point and rint's ties go
 * to the even integer, which is the even mantissa. */
static uint8_t encode_e4m3_rne(double v) {
    unsigned s = signbit(v) ? 0x80u : 0u;
    double a = fabs(v);
    int ex;
    frexp(a, &ex);
    int E = ex - 1;
    double step = (a == 0.0 || E < -6) ? ldexp(1.0, -9) : ldexp(1.0, E - 3);
    double r = rint(a / step) * step;
    if (r > 448.0) r = 448.0;
    if (r == 0.0) return (uint8_t)s;
    frexp(r, &ex);
    E = ex - 1;
    unsigned code;
    if (E < -6)
        code = (unsigned)(r / ldexp(1.0, -9)); /* exponent field 0, mantissa 1..7 */
    else
        code = ((unsigned)(E + 7) << 3) | (unsigned)((r / ldexp(1.0, E) - 1.0) * 8.0);
    return (uint8_t)(s | code);
}

/* x [rows][ld_x] fp32 -> q [rows][cols] E4M3 codes and e [ceil(rows/block_rows)][cols/128]
 * biased UE8M0 bytes.  Returns -1 for bad sizes or a non-finite input. */
int oracle_quantize_fp8(const float* x, int rows, int cols, int64_t ld_x, int block_rows, uint8_t* q,
                        uint8_t* e) {
    if (rows < 0 || cols < 0 || cols % 128 || block_rows < 1 || ld_x < cols) return -1;
    for (int r = 0; r < rows; ++r)
        for (int c = 0; c < cols; ++c)
            if (!isfinite(x[(int64_t)r * ld_x + c])) return -1;
    int KB = cols / 128, RB = (rows + block_rows - 1) / block_rows;
    for (int rb = 0; rb < RB; ++rb) {
        int r0 = rb * block_rows, r1 = r0 + block_rows < rows ? r0 + block_rows : rows;
        for (int kb = 0; kb < KB; ++kb) {
            double amax = 0.0;
            for (int r = r0; r < r1; ++r)
                for (int c = kb * 128; c < kb * 128 + 128; ++c) {
                    double a = fabs((double)x[(int64_t)r * ld_x + c]);
                    if (a > amax) amax = a;
                }
            int ex = exponent_for_amax(amax, 448.0);
            if (ex < -126) ex = -126;
            if (ex > 127) ex = 127;
            e[(int64_t)rb * KB + kb] = (uint8_t)(ex + 127);
            for (int r = r0; r < r1; ++r)
                for (int c = kb * 128; c < kb * 128 + 128; ++c)
                    q[(int64_t)r * cols + c] = encode_e4m3_rne(ldexp((double)x[(int64_t)r * ld_x + c], -ex));
        }
    }
    return 0;
}
