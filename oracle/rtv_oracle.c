/*
 * rtv_oracle.c -- plain, slow CPU oracle for the per-chunk KV-cache upkeep and
 * attention path of batch-size-one autoregressive video diffusion serving.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check and the CPU-baseline
 * leg of the benchmark may load this library.  It shares no source, header,
 * table or helper with the CUDA path in kv_cache_serving_append_b200/csrc.
 *
 * What the method computes, and where it is stated:
 *   - rotary embedding and FP8 quantisation are done a single time, when a
 *     frame is written into the cache, and the cache is a ring buffer whose
 *     advance copies nothing (aidose.in, "Runway explains how it serves a 57B
 *     video model in real time", third paragraph; pttl.gr, section
 *     "Από οκτώ H100 σε τέσσερις", second paragraph).
 *   - the new chunk then attends over the cached frames (same paragraphs:
 *     cache-upkeep time is set against attention time, 240 attention calls
 *     per step).
 * The pages fix neither the RoPE layout, nor the FP8 format, nor the scale
 * granularity, nor the attention mask; the readings used here (3D axial
 * rotate-half RoPE t|h|w with base 10000 and fp64 angles, OCP E4M3 with one
 * fp32 scale per token and head, amax/448 scaling by reciprocal multiply,
 * softmax scale 1/sqrt(D), bidirectional within the chunk and full over the
 * cached frames) are listed with their reasons in the design notes.
 *
 * Build: gcc -O2 -ffp-contract=off -fopenmp -shared -fPIC (no -ffast-math).
 * fp32 steps are written one rounding at a time; -ffp-contract=off forbids the
 * compiler from fusing a multiply and an add into one FMA.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ bf16 -- */

/* bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32 bits. */
static float bf16_bits_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* ------------------------------------------------------------------ E4M3 -- */
/*
 * OCP 8-bit floating point, E4M3 variant ("OCP 8-bit Floating Point
 * Specification", E4M3 encoding table): 1 sign bit, 4 exponent bits with bias
 * 7, 3 mantissa bits; exponent field 0 encodes subnormals m * 2^-9; there is
 * no infinity; S.1111.111 is NaN, so the largest finite magnitude is
 * S.1111.110 = 1.75 * 2^8 = 448.
 */

double oracle_e4m3_decode(uint8_t code)
{
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);             /* subnormal: m/8 * 2^-6 */
    else
        v = ldexp((double)(8 + m), e - 10);   /* (1 + m/8) * 2^(e-7)   */
    return s ? -v : v;
}

/* Exponent of the E4M3 binade that holds magnitude a (a < 448), clamped to the
 * subnormal binade: every value in binade E is a multiple of 2^(E-3). */
static int e4m3_binade(double a)
{
    int e;
    if (a == 0.0)
        return -6;
    frexp(a, &e);            /* a = f * 2^e, f in [0.5, 1) => floor(log2 a) = e - 1 */
    e -= 1;
    return e < -6 ? -6 : e;
}

/*
 * Round-to-nearest-even to E4M3, saturating: magnitudes at or above the
 * largest finite value map to +-448 (the reading: a product x * (448/amax)
 * may exceed 448 by rounding, and it must clamp, not become NaN).
 * The sign of zero is kept (-0 -> 0x80).
 */
uint8_t oracle_e4m3_encode(float y)
{
    uint8_t s;
    double a, q, n, r;
    int E;
    if (isnan(y))
        return 0x7F;
    s = signbit(y) ? 0x80 : 0x00;
    a = fabs((double)y);
    if (a >= 448.0)
        return (uint8_t)(s | 0x7E);
    E = e4m3_binade(a);
    q = ldexp(1.0, E - 3);   /* spacing of representable values in this binade */
    n = a / q;               /* exact: q is a power of two                      */
    r = rint(n);             /* default rounding mode: nearest, ties to even    */
    if (E == -6 && r < 8.0)  /* subnormal (or zero): code = m                   */
        return (uint8_t)(s | (uint8_t)r);
    if (r >= 16.0) {         /* rounded up into the next binade                 */
        E += 1;
        r = 8.0;
    }
    return (uint8_t)(s | (uint8_t)(((E + 7) << 3) | ((int)r - 8)));
}

/*
 * 1 when y lies within 1e-6 relative of a rounding boundary of E4M3, i.e. of
 * the midpoint between two adjacent finite E4M3 values of the same sign.
 * There a one-step difference between two correct fp32 pipelines is allowed.
 */
uint8_t oracle_e4m3_near_boundary(float y)
{
    double a = fabs((double)y), q, mid;
    long k, kk;
    int E;
    if (isnan(y) || a >= 464.0)
        return 0;
    E = e4m3_binade(a);
    q = ldexp(1.0, E - 3);
    k = (long)floor(a / q);
    for (kk = k - 1; kk <= k; ++kk) {
        if (kk < 0)
            continue;
        if (E == 8 && kk + 1 > 14)   /* no finite value above 448 */
            continue;
        mid = ((double)kk + 0.5) * q;
        if (fabs(a / mid - 1.0) <= 1e-6)
            return 1;
    }
    return 0;
}

/* ------------------------------------------------------------------ RoPE -- */
/*
 * 3D axial rotary position embedding, rotate-half inside each axis segment.
 * head_dim D = n_t + n_h + n_w, segments in the order t | h | w.  For a
 * segment of size n starting at offset o, at integer position p, and pair
 * index j in [0, n/2):
 *     theta = p * base^(-2j/n)                    (fp64)
 *     c = (float)cos(theta), s = (float)sin(theta)
 *     x'[o+j]       = fl(fl(x[o+j] * c)       - fl(x[o+j+n/2] * s))
 *     x'[o+j+n/2]   = fl(fl(x[o+j+n/2] * c)   + fl(x[o+j] * s))
 * This fixed order, one fp32 rounding per operation and no FMA, is the
 * definition the GPU path is held to.
 */
static void rope_segment(const float* x, float* y, int o, int n, long p, double base)
{
    int j, half = n / 2;
    for (j = 0; j < half; ++j) {
        double inv_freq = pow(base, -2.0 * (double)j / (double)n);
        double theta = (double)p * inv_freq;
        float c = (float)cos(theta);
        float s = (float)sin(theta);
        float a = x[o + j], b = x[o + j + half];
        float ac = a * c, bs = b * s, bc = b * c, as = a * s;
        y[o + j] = ac - bs;
        y[o + j + half] = bc + as;
    }
}

/* Rotate one head vector x[D] at grid position (t, h, w). */
void oracle_rope3d(const float* x, float* y, int D, int n_t, int n_h, int n_w,
                   long t, long h, long w, double base)
{
    (void)D;
    rope_segment(x, y, 0, n_t, t, base);
    rope_segment(x, y, n_t, n_h, h, base);
    rope_segment(x, y, n_t + n_h, n_w, w, base);
}

/* ------------------------------------------------------------ quantise -- */
/*
 * Per (token, head) row of D values:
 *     amax  = max_d |x_d|                         (exact in fp32)
 *     inv   = fl(448 / amax)      (inv = 0 when amax < 2^-119)
 *     code  = E4M3_RNE_sat(fl(x_d * inv))
 *     scale = fl(amax / 448)      (scale = 0 when amax < 2^-119)
 * so that decode(code) * scale approximates x_d.  Below 2^-119 the fp32
 * reciprocal would overflow (448 / 2^-120 > FLT_MAX) and the product x_d * inv
 * would turn zeros into NaN: such an item is stored as zero, as an all-zero
 * item is (the reading: values under 2e-36 carry nothing the format can keep).
 */
void oracle_quantize_row(const float* x, int D, uint8_t* codes, float* scale,
                         uint8_t* near_boundary)
{
    int d;
    float amax = 0.0f, inv;
    for (d = 0; d < D; ++d) {
        float a = fabsf(x[d]);
        if (a > amax)
            amax = a;
    }
    inv = amax >= 0x1p-119f ? 448.0f / amax : 0.0f;
    for (d = 0; d < D; ++d) {
        float yv = x[d] * inv;
        codes[d] = oracle_e4m3_encode(yv);
        if (near_boundary)
            near_boundary[d] = oracle_e4m3_near_boundary(yv);
    }
    *scale = amax >= 0x1p-119f ? amax / 448.0f : 0.0f;
}

/* -------------------------------------------------------------- append -- */
/*
 * One tensor (Q, K or V) of one chunk: bf16 input laid out [rows][H][D] as a
 * QKV projection produces it, rows = n_frames * T, row r = frame r / T, token
 * r % T.  Frame f of the chunk has absolute frame index t0 + f; token k sits
 * at grid row k / grid_w and column k % grid_w.  RoPE is applied when
 * apply_rope is set (Q and K; V is not rotated).  Outputs are head-major:
 * codes[H][rows][D], scales[H][rows], near_boundary[H][rows][D] (nullable).
 */
void oracle_append_tensor(const uint16_t* x_bf16, int rows, int H, int D,
                          int T, int grid_w, long t0, int apply_rope,
                          int n_t, int n_h, int n_w, double base,
                          uint8_t* codes, float* scales, uint8_t* near_boundary)
{
    long idx;
    long total = (long)rows * H;
#pragma omp parallel for schedule(static)
    for (idx = 0; idx < total; ++idx) {
        int r = (int)(idx / H), h = (int)(idx % H), d;
        float xin[512], xr[512];
        const uint16_t* src = x_bf16 + ((long)r * H + h) * D;
        long frame = t0 + r / T;
        int tok = r % T;
        size_t o = ((size_t)h * rows + r);
        for (d = 0; d < D; ++d)
            xin[d] = bf16_bits_to_float(src[d]);
        if (apply_rope)
            oracle_rope3d(xin, xr, D, n_t, n_h, n_w, frame, tok / grid_w, tok % grid_w, base);
        else
            memcpy(xr, xin, sizeof(float) * (size_t)D);
        oracle_quantize_row(xr, D, codes + o * D, scales + o,
                            near_boundary ? near_boundary + o * D : NULL);
    }
}

/* ----------------------------------------------------------- attention -- */
/*
 * fp64 softmax attention on dequantised tensors, for one chunk:
 *     q^_id = decode(qc_id) * sq_i,  k^_jd = decode(kc_jd) * sk_j,  v^ alike
 *     s_ij  = (sum_d q^_id k^_jd) / sqrt(D)
 *     p_ij  = exp(s_ij - max_j s_ij)
 *     o_i   = sum_j p_ij v^_j / sum_j p_ij
 * over every key j of the key set (pinned frame, the window frames and the
 * chunk's own frames, gathered by the caller into kc/vc [H][NK][D]).  The mask
 * is full over the key set: no key of the set is hidden from any query.
 * Query rows: rows[0..n_rows) (or all M rows when rows is NULL).
 * out: [n_rows][H][D] fp64.  psum (nullable): [n_rows][H] = sum_j p_ij / l_i,
 * which must be 1 (the softmax-row-sum invariant).
 */
void oracle_attend(int H, int D, int M, const uint8_t* qc, const float* sq,
                   int NK, const uint8_t* kc, const float* sk,
                   const uint8_t* vc, const float* sv,
                   int n_rows, const int* rows, double* out, double* psum)
{
    int h;
    int nr = rows ? n_rows : M;
    double inv_sqrt_d = 1.0 / sqrt((double)D);
    double* kd = (double*)malloc(sizeof(double) * (size_t)NK * D);
    double* vd = (double*)malloc(sizeof(double) * (size_t)NK * D);
    double lut[256];
    int c;
    for (c = 0; c < 256; ++c)
        lut[c] = oracle_e4m3_decode((uint8_t)c);
    for (h = 0; h < H; ++h) {
        long j;
        int ii;
        const uint8_t* kch = kc + (size_t)h * NK * D;
        const uint8_t* vch = vc + (size_t)h * NK * D;
#pragma omp parallel for schedule(static)
        for (j = 0; j < NK; ++j) {
            int d;
            double ks = (double)sk[(size_t)h * NK + j], vs = (double)sv[(size_t)h * NK + j];
            for (d = 0; d < D; ++d) {
                kd[(size_t)j * D + d] = lut[kch[(size_t)j * D + d]] * ks;
                vd[(size_t)j * D + d] = lut[vch[(size_t)j * D + d]] * vs;
            }
        }
#pragma omp parallel for schedule(dynamic, 1)
        for (ii = 0; ii < nr; ++ii) {
            int i = rows ? rows[ii] : ii, d;
            long jj;
            double q[512], acc[512], mx = -INFINITY, l = 0.0, chk = 0.0;
            double* s = (double*)malloc(sizeof(double) * (size_t)NK);
            double qs = (double)sq[(size_t)h * M + i];
            for (d = 0; d < D; ++d) {
                q[d] = lut[qc[((size_t)h * M + i) * D + d]] * qs;
                acc[d] = 0.0;
            }
            for (jj = 0; jj < NK; ++jj) {
                double dot = 0.0;
                const double* kr = kd + (size_t)jj * D;
                for (d = 0; d < D; ++d)
                    dot += q[d] * kr[d];
                s[jj] = dot * inv_sqrt_d;
                if (s[jj] > mx)
                    mx = s[jj];
            }
            for (jj = 0; jj < NK; ++jj) {
                double p = exp(s[jj] - mx);
                const double* vr = vd + (size_t)jj * D;
                s[jj] = p;
                l += p;
                for (d = 0; d < D; ++d)
                    acc[d] += p * vr[d];
            }
            for (d = 0; d < D; ++d)
                out[((size_t)ii * H + h) * D + d] = acc[d] / l;
            if (psum) {
                for (jj = 0; jj < NK; ++jj)
                    chk += s[jj] / l;
                psum[(size_t)ii * H + h] = chk;
            }
            free(s);
        }
    }
    free(kd);
    free(vd);
}

/* Number of OpenMP threads the oracle runs with (reported beside timings). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------ array forms for tests -- */

void oracle_e4m3_encode_array(const float* y, long n, uint8_t* codes)
{
    long i;
    for (i = 0; i < n; ++i)
        codes[i] = oracle_e4m3_encode(y[i]);
}

void oracle_e4m3_near_boundary_array(const float* y, long n, uint8_t* mask)
{
    long i;
    for (i = 0; i < n; ++i)
        mask[i] = oracle_e4m3_near_boundary(y[i]);
}

void oracle_e4m3_decode_array(const uint8_t* codes, long n, double* v)
{
    long i;
    for (i = 0; i < n; ++i)
        v[i] = oracle_e4m3_decode(codes[i]);
}

/* x, y: [n][D]; positions pos: [n][3] = (t, h, w). */
void oracle_rope3d_array(const float* x, float* y, long n, int D, int n_t, int n_h,
                         int n_w, const long* pos, double base)
{
    long i;
    for (i = 0; i < n; ++i)
        oracle_rope3d(x + i * D, y + i * D, D, n_t, n_h, n_w, pos[3 * i], pos[3 * i + 1],
                      pos[3 * i + 2], base);
}

/* x: [n][D] fp32 rows -> codes [n][D], scales [n]. */
void oracle_quantize_rows(const float* x, long n, int D, uint8_t* codes, float* scales,
                          uint8_t* near_boundary)
{
    long i;
    for (i = 0; i < n; ++i)
        oracle_quantize_row(x + i * D, D, codes + i * D, scales + i,
                            near_boundary ? near_boundary + i * D : NULL);
}
