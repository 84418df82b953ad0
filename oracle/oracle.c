/*
 * CPU oracle for the FP8 NT GEMM with fine-grained scaling -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the smoke check and the bench's CPU-baseline leg use this file.  It shares no code,
 * header, table or constant with the CUDA library, and the library never calls it.
 *
 * What it computes (the plain definition; "FP8 GEMM kernels with fine-grained scaling", DeepGEMM-for-PPU
 * README, "Interfaces": gemm_fp8_fp8_bf16_nt, NT only -- LHS [M,K] and RHS [N,K] both K-major; scaling
 * recipe (1, 128, 128) from the MATE deep_gemm wrapper API list):
 *
 *   ref[m][n] = sum_{kb} sfa(m,kb) * sfb(g, n/128, kb) * sum_{k in block kb} dec(a[m][k]) * dec(b_g[n][k])
 *
 * evaluated in double.  dec() is the OCP E4M3 ("e4m3fn") decode written out from its bit fields.  Each
 * 128-term inner sum is exact in double (products of two e4m3 values carry <= 8 significant bits and lie in
 * [2^-18, 2^18)), so the only rounding is in the sum over K blocks.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC oracle.c -o liboracle.so   (oracle/build.py does this)
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>

/* OCP 8-bit floating point, E4M3 variant: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits.
 * Exponent field 0 is subnormal: (m/8) * 2^(1-7).  S.1111.111 is NaN; there is no infinity. */
double oracle_e4m3_decode(uint8_t code) {
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, 1 - 7);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

void oracle_e4m3_decode_array(const uint8_t *codes, int64_t n, double *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_decode(codes[i]);
}

/*
 * Rows of the product, one listed row at a time.
 *
 *   a            e4m3 codes; listed row i reads a[rows[i] * K + k]
 *   sfa          fp32 scales; row i, K block kb reads sfa[sfa_row_off[i] + kb * sfa_kb_stride]
 *   b            e4m3 codes, groups of [N][K] at b + g * b_group_stride
 *   sfb          fp32 scales, [G][ceil(N/128)][K/128] with group stride sfb_group_stride
 *   groups[i]    the group whose B row i multiplies
 *   out          double [n_rows][N]
 */
void oracle_gemm_rows(const uint8_t *a, const float *sfa, const int64_t *sfa_row_off, int64_t sfa_kb_stride,
                      const uint8_t *b, int64_t b_group_stride, const float *sfb, int64_t sfb_group_stride,
                      const int64_t *rows, const int32_t *groups, int64_t n_rows, int64_t N, int64_t K,
                      double *out) {
    const int64_t nkb = K / 128;
    double table[256];
    for (int c = 0; c < 256; ++c) table[c] = oracle_e4m3_decode((uint8_t)c);

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < n_rows; ++i) {
        const uint8_t *arow = a + rows[i] * K;
        const uint8_t *bg = b + (int64_t)groups[i] * b_group_stride;
        const float *sfbg = sfb + (int64_t)groups[i] * sfb_group_stride;
        for (int64_t n = 0; n < N; ++n) {
            const uint8_t *brow = bg + n * K;
            double acc = 0.0;
            for (int64_t kb = 0; kb < nkb; ++kb) {
                double block = 0.0;
                for (int64_t k = kb * 128; k < kb * 128 + 128; ++k) block += table[arow[k]] * table[brow[k]];
                double sa = (double)sfa[sfa_row_off[i] + kb * sfa_kb_stride];
                double sb = (double)sfbg[(n / 128) * nkb + kb];
                acc += sa * sb * block;
            }
            out[i * N + n] = acc;
        }
    }
}

int oracle_num_threads(void) {
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        n = omp_get_num_threads();
    }
    return n;
}
