/*
 * Drives every entry point of the CPU oracle on small inputs, for a build of
 * the oracle with AddressSanitizer and UndefinedBehaviorSanitizer (test
 * infrastructure; run by tests/test_sanitizers_cpu.py).  Exits 0 when every
 * call returns and the results are finite; the sanitizers abort on the first
 * out-of-bounds access, use of freed memory or undefined operation.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

double oracle_e4m3_decode(uint8_t code);
uint8_t oracle_e4m3_encode(float y);
uint8_t oracle_e4m3_near_boundary(float y);
void oracle_rope3d(const float* x, float* y, int D, int n_t, int n_h, int n_w, long t, long h,
                   long w, double base);
void oracle_quantize_row(const float* x, int D, uint8_t* codes, float* scale, uint8_t* near);
void oracle_append_tensor(const uint16_t* x_bf16, int rows, int H, int D, int T, int grid_w, long t0,
                          int apply_rope, int n_t, int n_h, int n_w, double base, uint8_t* codes,
                          float* scales, uint8_t* near_boundary);
void oracle_attend(int H, int D, int M, const uint8_t* qc, const float* sq, int NK, const uint8_t* kc,
                   const float* sk, const uint8_t* vc, const float* sv, int n_rows, const int* rows,
                   double* out, double* psum);

static uint32_t rng = 12345u;
static uint32_t next(void) { rng = rng * 1664525u + 1013904223u; return rng >> 8; }
static float unit(void) { return (float)(next() & 0xffff) / 32768.0f - 1.0f; }

int main(void)
{
    int c, i;
    /* E4M3: every code, and a spread of values including 0, +-448 and beyond */
    for (c = 0; c < 256; ++c) {
        double v = oracle_e4m3_decode((uint8_t)c);
        if ((c & 0x7f) != 0x7f && !isfinite(v)) return 1;
    }
    for (i = 0; i < 100000; ++i) {
        float y = unit() * 600.0f;
        (void)oracle_e4m3_encode(y);
        (void)oracle_e4m3_near_boundary(y);
    }
    (void)oracle_e4m3_encode(0.0f);
    (void)oracle_e4m3_encode(-0.0f);
    (void)oracle_e4m3_encode(1e-30f);

    /* RoPE and quantisation of one row, both head_dims */
    {
        float x[128], y[128], sc;
        uint8_t codes[128], near[128];
        for (i = 0; i < 128; ++i) x[i] = unit() * 4.0f;
        oracle_rope3d(x, y, 128, 32, 48, 48, 7, 3, 5, 10000.0);
        oracle_quantize_row(y, 128, codes, &sc, near);
        oracle_rope3d(x, y, 64, 16, 24, 24, 0, 0, 0, 10000.0);
        oracle_quantize_row(y, 64, codes, &sc, NULL);
        memset(x, 0, sizeof x);
        oracle_quantize_row(x, 128, codes, &sc, near);   /* all-zero row: scale 0 */
        if (sc != 0.0f) return 2;
    }

    /* append of a 2-frame chunk (T = 12 tokens on a 3x4 grid), then attention */
    {
        const int H = 3, D = 64, T = 12, F = 2, rows = F * T, NK = 3 * T, M = rows;
        uint16_t* xb = malloc(sizeof(uint16_t) * rows * H * D);
        uint8_t *qc = malloc(H * rows * D), *kc = malloc(H * NK * D), *vc = malloc(H * NK * D);
        uint8_t* near = malloc(H * rows * D);
        float *sq = malloc(sizeof(float) * H * rows), *sk = malloc(sizeof(float) * H * NK),
              *sv = malloc(sizeof(float) * H * NK);
        double *out = malloc(sizeof(double) * M * H * D), *psum = malloc(sizeof(double) * M * H);
        int rws[3] = {0, 5, M - 1};
        for (i = 0; i < rows * H * D; ++i) {
            float f = unit() * 3.0f;
            uint32_t u;
            memcpy(&u, &f, 4);
            xb[i] = (uint16_t)(u >> 16);
        }
        oracle_append_tensor(xb, rows, H, D, T, 4, 5, 1, 16, 24, 24, 10000.0, qc, sq, near);
        oracle_append_tensor(xb, rows, H, D, T, 4, 5, 0, 16, 24, 24, 10000.0, qc, sq, NULL);
        for (i = 0; i < H * NK * D; ++i) {
            kc[i] = (uint8_t)(next() & 0x7e);
            vc[i] = (uint8_t)(next() & 0xfe);
            if ((vc[i] & 0x7f) == 0x7f) vc[i] = 0x38;
        }
        for (i = 0; i < H * NK; ++i) {
            sk[i] = 0.01f + 0.001f * (float)(i % 7);
            sv[i] = 0.02f;
        }
        oracle_attend(H, D, M, qc, sq, NK, kc, sk, vc, sv, M, NULL, out, psum);
        for (i = 0; i < M * H; ++i)
            if (fabs(psum[i] - 1.0) > 1e-12) return 3;
        oracle_attend(H, D, M, qc, sq, NK, kc, sk, vc, sv, 3, rws, out, NULL);
        for (i = 0; i < 3 * H * D; ++i)
            if (!isfinite(out[i])) return 4;
        free(xb); free(qc); free(kc); free(vc); free(near); free(sq); free(sk); free(sv);
        free(out); free(psum);
    }
    printf("oracle driver ok\n");
    return 0;
}
