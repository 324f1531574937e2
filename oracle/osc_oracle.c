/*
 * OSC W4A4 oracle: plain, slow, single-threaded C in fp64.
 *
 * TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference leg of bench.py may load this library. The product
 * path (libosc.so and its Python binding) never calls it, shares no code,
 * header, table or constant with it, and fails loudly if its own CUDA library
 * is missing.
 *
 * Source: the OSC page, "W4A4量化技术：OSC框架如何实现高效LLM部署"
 * (coreui.cn/article/2607942.html), cited below by its own section numbers.
 * Where the page is silent the plain reading is taken and marked READING;
 * the design notes list every one of them.
 *
 * Layout conventions (logical, not the GPU's):
 *   X, W      bf16 bit patterns, row-major, rows x K (tokens x channels /
 *             out-features x in-features).
 *   L         int8, K/G entries: local channel index 0..G-1 of the group's
 *             outlier, or -1.
 *   codes     one unpacked 4-bit (E2M1) or 8-bit (E4M3) code per element,
 *             row-major rows x K.
 *   exps      one signed shared exponent e per scale slot, row-major
 *             rows x (K / V), V = 16 for G = 16, else 32 (G = 64 writes the
 *             same e into both 32-slots of a 64-group). The E8M0 byte is e+127.
 *
 * Inputs must be finite; the functions return -1 on a non-finite input or a
 * bad argument and 0 on success.
 *
 * Every function here is pinned by tests/test_oracle_pins.py to something other
 * than itself (format definitions, brute force, closed forms, invariants, library
 * matmul), and tests/test_oracle_mutants.py checks that planted mistakes fail those
 * pins. Parity unpinned: the output of the table build (Algorithm 1) on inputs
 * without planted structure. It follows from the READING of the outlier event
 * below and is pinned only where that reading fixes it (planted channels,
 * closed-form thresholds, tie rules).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_FMT_E2M1 0
#define ORC_FMT_E4M3 1

/* ---- bf16 <-> double ------------------------------------------------------ */

double orc_bf16_to_double(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16, ties to even (used only to state the
 * expected BF16 output of a given fp64 value). Finite inputs; overflow goes
 * to infinity as IEEE round-to-nearest does. */
uint16_t orc_double_to_bf16(double x)
{
    if (x == 0.0) return signbit(x) ? 0x8000u : 0x0000u;
    uint16_t sign = signbit(x) ? 0x8000u : 0x0000u;
    double a = fabs(x);
    int ex;
    frexp(a, &ex);                       /* a = f * 2^ex, f in [0.5, 1) */
    int E = ex - 1;                      /* floor(log2 a) */
    if (E < -126) E = -126;              /* subnormal quantum 2^-133 */
    double quantum = ldexp(1.0, E - 7);  /* 7 stored mantissa bits */
    double q = nearbyint(a / quantum) * quantum;   /* default mode: ties to even */
    if (q >= ldexp(1.0, 128)) return sign | 0x7F80u;
    float f = (float)q;                  /* exact: q has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return sign | (uint16_t)((u >> 16) & 0x7FFFu);
}

static int all_finite_bf16(const uint16_t* x, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        if ((x[i] & 0x7F80u) == 0x7F80u) return 0;
    return 1;
}

/* ---- Algorithm 1 and the clustering density ---------------------------------
 *
 * The page (§3.1, Algorithm 1) loops over the channel groups of one (position,
 * layer) and stores, per group, the channel returned by
 * find_consistent_outlier(group, alpha), else -1. The page does not define
 * that function; READING: for each calibration token t the group's outlier
 * event is the channel j_t holding the largest |x| (lowest j on ties), and it
 * counts only when that maximum is at least alpha times the group's mean
 * magnitude:  G * |x_max| >= alpha * sum_j |x_j|, with |x_max| > 0.
 * The sum is accumulated in fp32 in ascending j and the comparison is done in
 * fp64, so both sides of any parity test take the same decision.
 * The channel with the most events wins (lowest j on ties) if it has at least
 * min_hits events; otherwise the group has no consistent outlier (-1).
 * j* = 0 is a valid channel: the printed algorithm keeps the found channel only
 * when its index is nonzero, which reads as a shorthand for "a channel was
 * found", not as a rule.
 */
static int group_event(const uint16_t* xg, int G, float alpha, int* j_out)
{
    double best = -1.0;
    int jb = 0;
    float s = 0.0f;
    for (int j = 0; j < G; ++j) {
        double a = fabs(orc_bf16_to_double(xg[j]));
        s += (float)a;                     /* fp32, ascending j */
        if (a > best) { best = a; jb = j; }
    }
    *j_out = jb;
    if (!(best > 0.0)) return 0;
    return (double)G * best >= (double)alpha * (double)s;
}

int orc_build_table(const uint16_t* X, int S, int K, int G, float alpha,
                    int min_hits, int8_t* L)
{
    if (!X || !L || S < 0 || K <= 0 || G <= 0 || K % G != 0 || G > 127) return -1;
    if (!all_finite_bf16(X, (int64_t)S * K)) return -1;
    int Kg = K / G;
    int64_t* hits = (int64_t*)calloc((size_t)G, sizeof(int64_t));
    if (!hits) return -1;
    for (int k = 0; k < Kg; ++k) {
        memset(hits, 0, (size_t)G * sizeof(int64_t));
        for (int t = 0; t < S; ++t) {
            int j;
            if (group_event(X + (int64_t)t * K + (int64_t)k * G, G, alpha, &j))
                hits[j] += 1;
        }
        int js = 0;
        for (int j = 1; j < G; ++j)
            if (hits[j] > hits[js]) js = j;
        L[k] = (hits[js] >= (int64_t)min_hits && hits[js] > 0) ? (int8_t)js : (int8_t)-1;
    }
    free(hits);
    return 0;
}

/* Clustering density, §2.2: C_k = N_k^hit / N_k^total, where N_k^total counts
 * the outlier events of group k over the given tokens and N_k^hit those whose
 * channel is the table's static index L[k] (0 hits when L[k] = -1). Events use
 * the same test as the table build. */
int orc_density(const uint16_t* X, int S, int K, int G, float alpha,
                const int8_t* L, int64_t* n_hit, int64_t* n_total)
{
    if (!X || !L || !n_hit || !n_total || S < 0 || K <= 0 || G <= 0 || K % G) return -1;
    if (!all_finite_bf16(X, (int64_t)S * K)) return -1;
    int Kg = K / G;
    for (int k = 0; k < Kg; ++k) { n_hit[k] = 0; n_total[k] = 0; }
    for (int t = 0; t < S; ++t)
        for (int k = 0; k < Kg; ++k) {
            int j;
            if (group_event(X + (int64_t)t * K + (int64_t)k * G, G, alpha, &j)) {
                n_total[k] += 1;
                if (L[k] >= 0 && j == L[k]) n_hit[k] += 1;
            }
        }
    return 0;
}

/* Protection of up to R channels per group (§6, "multi-outlier protection" for extreme
 * cases; the page gives no procedure). READING: R rounds of Algorithm 1; round r runs on the
 * calibration activations with the channels of rounds 0 .. r-1 set to zero, i.e. on what
 * extraction would leave, so a further channel is protected only when it is still a consistent
 * outlier once the stronger ones are out. L holds K/G x R entries, slot r of group k at
 * L[k*R + r]; a group whose round r finds nothing keeps -1 from there on (later rounds see the
 * same data). R = 1 is orc_build_table. */
int orc_build_table_multi(const uint16_t* X, int S, int K, int G, float alpha,
                          int min_hits, int R, int8_t* L)
{
    if (!X || !L || S < 0 || K <= 0 || G <= 0 || K % G != 0 || R < 1) return -1;
    int Kg = K / G;
    uint16_t* work = (uint16_t*)malloc((size_t)S * (size_t)K * sizeof(uint16_t) + 1);
    int8_t* Lr = (int8_t*)malloc((size_t)Kg + 1);
    if (!work || !Lr) { free(work); free(Lr); return -1; }
    memcpy(work, X, (size_t)S * (size_t)K * sizeof(uint16_t));
    int rc = 0;
    for (int r = 0; r < R && rc == 0; ++r) {
        rc = orc_build_table(work, S, K, G, alpha, min_hits, Lr);
        for (int k = 0; k < Kg && rc == 0; ++k) {
            L[k * R + r] = Lr[k];
            if (Lr[k] >= 0)
                for (int t = 0; t < S; ++t) work[(int64_t)t * K + k * G + Lr[k]] = 0x0000u;
        }
    }
    free(work);
    free(Lr);
    return rc;
}

/* ---- Outlier extraction (§3.2, Figure 2 caption) ----------------------------
 *
 * For every group k whose table entry is j = L[k] >= 0, the value
 * x[t, k*G + j] is moved into the high-precision buffer B and the slot in X is
 * set to zero, before the microscaling step. READING: B is stored compactly,
 * one column per table entry in ascending k (the page's B in R^{S x K} holds
 * exactly these values; the product B * W_L is the same either way), padded
 * with zero columns up to K_L; the zeroed slot becomes +0.
 */
int orc_table_count(const int8_t* L, int Kg)
{
    int c = 0;
    for (int k = 0; k < Kg; ++k) c += (L[k] >= 0);
    return c;
}

int orc_extract(const uint16_t* X, int M, int K, int G, const int8_t* L, int R,
                int K_L, uint16_t* Xz, uint16_t* B)
{
    if (!X || !L || !Xz || M < 0 || K <= 0 || G <= 0 || K % G || R < 1) return -1;
    int Kg = K / G;
    int cnt = orc_table_count(L, Kg * R);
    if (K_L < cnt || (K_L > 0 && !B)) return -1;
    for (int i = 0; i < Kg * R; ++i)
        if (L[i] >= G) return -1;
    memcpy(Xz, X, (size_t)M * (size_t)K * sizeof(uint16_t));
    for (int64_t i = 0; i < (int64_t)M * K_L; ++i) B[i] = 0;
    /* entries in (group, slot) order; each copies what the earlier ones left in the slot, so
     * a channel named twice gives its value once and 0 the second time */
    int pos = 0;
    for (int k = 0; k < Kg; ++k)
        for (int m = 0; m < R; ++m) {
            int j = L[k * R + m];
            if (j < 0) continue;
            int c = k * G + j;
            for (int t = 0; t < M; ++t) {
                B[(int64_t)t * K_L + pos] = Xz[(int64_t)t * K + c];
                Xz[(int64_t)t * K + c] = 0x0000u;
            }
            ++pos;
        }
    return 0;
}

/* W_L (§3.2, §3.3): the high-precision weight rows of the table's channels,
 * stored as one contiguous block. With W as out x in (rows n, columns = input
 * channels), the i-th table channel c_i = k_i*G + L[k_i] gives
 * W_L[n][i] = W[n][c_i]; pad columns are zero. Then B * W_L^T supplies the
 * outlier channels' contribution to Y. */
int orc_gather_wl(const uint16_t* W, int N, int K, int G, const int8_t* L, int R,
                  int K_L, uint16_t* WL)
{
    if (!W || !L || N < 0 || K <= 0 || G <= 0 || K % G || R < 1) return -1;
    int Kg = K / G;
    int cnt = orc_table_count(L, Kg * R);
    if (K_L < cnt || (K_L > 0 && !WL)) return -1;
    for (int64_t i = 0; i < (int64_t)N * K_L; ++i) WL[i] = 0;
    int pos = 0;
    for (int k = 0; k < Kg; ++k)
        for (int m = 0; m < R; ++m) {
            int jw = L[(int64_t)k * R + m];
            if (jw < 0) continue;
            int c = k * G + jw;
            for (int n = 0; n < N; ++n) WL[(int64_t)n * K_L + pos] = W[(int64_t)n * K + c];
            ++pos;
        }
    return 0;
}

/* ---- The producer step before the quantize: RMSNorm --------------------------
 *
 * Figure 2 (§3.2) places extraction and microscaling directly before the GEMM; in
 * the Qwen3 layers the page measures (§1, §5.2) the activations that reach the QKV
 * and FFN up/gate projections come straight out of an RMSNorm. The page does not
 * describe that step; READING (the usual RMSNorm, with its order of operations fixed
 * so that both sides reach the same bits), for one row x of K bf16 values, weight
 * gamma (K bf16 values) and eps, all in fp32 with every operation rounded to
 * nearest even:
 *   s_b    = x_{32b}^2 + x_{32b+1}^2 + ... + x_{32b+31}^2, added in ascending
 *            order, one sum per 32-channel block b = 0 .. K/32 - 1;
 *   total  the block sums padded with zeros to a power of two P and combined
 *            pairwise: for h = P/2, P/4, ..., 1: s_b <- s_b + s_{b+h} (b < h);
 *            total = s_0;
 *   inv    = 1 / sqrt(total / K + eps);
 *   y_j    = bf16( (x_j * inv) * gamma_j ).
 * The normalized row y then goes through extraction and microscaling unchanged.
 */
static float f32_of_bf16(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Sum of squares of one row in the stated order. */
float orc_row_sumsq(const uint16_t* x, int K)
{
    int nb = K / 32, P = 1;
    while (P < nb) P *= 2;
    float* s = (float*)calloc((size_t)P, sizeof(float));
    if (!s) return NAN;
    for (int b = 0; b < nb; ++b) {
        float acc = 0.0f;
        for (int j = 0; j < 32; ++j) {
            float v = f32_of_bf16(x[b * 32 + j]);
            float sq = v * v;
            acc = acc + sq;
        }
        s[b] = acc;
    }
    for (int h = P / 2; h >= 1; h /= 2)
        for (int b = 0; b < h; ++b) s[b] = s[b] + s[b + h];
    float total = s[0];
    free(s);
    return total;
}

int orc_rmsnorm(const uint16_t* X, int M, int K, const uint16_t* gamma, float eps,
                uint16_t* Y, float* inv_out)
{
    if (!X || !gamma || !Y || M < 0 || K <= 0 || K % 32 != 0 || !(eps >= 0.0f)) return -1;
    if (!all_finite_bf16(X, (int64_t)M * K) || !all_finite_bf16(gamma, K)) return -1;
    for (int t = 0; t < M; ++t) {
        const uint16_t* x = X + (int64_t)t * K;
        float total = orc_row_sumsq(x, K);
        float mean = total / (float)K;
        float root = sqrtf(mean + eps);
        float inv = 1.0f / root;
        if (inv_out) inv_out[t] = inv;
        for (int j = 0; j < K; ++j) {
            float a = f32_of_bf16(x[j]) * inv;
            float b = a * f32_of_bf16(gamma[j]);
            Y[(int64_t)t * K + j] = orc_double_to_bf16((double)b);
        }
    }
    return 0;
}

/* ---- Microscaling (§3.2, the dynamic-range step) ------------------------------
 *
 * After the table channels are zeroed the page rescales each group with its
 * now smaller range and quantizes it to 4 bits; the element and scale formats
 * are the OCP MX ones: E2M1 elements
 * with one shared E8M0 power-of-two scale per block (E4M3 elements for the
 * FP8 fallback of §4).
 *   shared exponent   e = floor(log2(amax)) - emax_elem, emax_elem = 2 (E2M1)
 *                     or 8 (E4M3); floor(log2) via frexp, so it takes no
 *                     route through the bits of the input; e clamped to
 *                     [-127, 127]; READING: amax = 0 gives e = -127 (0x00).
 *   element           v = x * 2^-e (exact in fp64), rounded to the element
 *                     format, ties to even, |v| beyond the largest finite
 *                     element saturates to it (6 for E2M1, 448 for E4M3).
 *   sign              READING: the code keeps the sign of x even when the
 *                     magnitude rounds to zero (IEEE rounding never flips a
 *                     sign), so -0.1 -> 0x8 (E2M1) / 0x80 (E4M3).
 * Rounding is written as the format's own definition: the quantum of the
 * binade holding |v| (one mantissa bit for E2M1, three for E4M3, a fixed
 * subnormal quantum below the smallest normal), and nearbyint() in the
 * default ties-to-even mode.
 */
static int shared_exponent(double amax, int emax_elem)
{
    if (!(amax > 0.0)) return -127;
    int ex;
    frexp(amax, &ex);          /* amax = f * 2^ex, f in [0.5, 1) */
    int e = (ex - 1) - emax_elem;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

static uint8_t encode_e2m1(double v)
{
    uint8_t sign = signbit(v) ? 0x8 : 0x0;
    double a = fabs(v);
    /* E2M1: 2 exponent bits (bias 1), 1 mantissa bit. Normal binades [1,2),
     * [2,4), [4,8) have quanta 0.5, 1, 2; the subnormal range [0,1) has 0.5. */
    double quantum = (a < 2.0) ? 0.5 : (a < 4.0 ? 1.0 : 2.0);
    double q = nearbyint(a / quantum) * quantum;
    if (q > 6.0) q = 6.0;
    uint8_t mag;
    if (q < 1.0) {
        mag = (uint8_t)(q / 0.5);               /* subnormal: 0 -> 0, 0.5 -> 1 */
    } else {
        int ex;
        double f = frexp(q, &ex);               /* q = f*2^ex, f in [0.5,1) */
        int E = ex;                             /* biased exponent: q in [2^(E-1), 2^E) */
        int m = (int)(f * 4.0) - 2;             /* 1 mantissa bit */
        mag = (uint8_t)(E * 2 + m);
    }
    return sign | mag;
}

static uint8_t encode_e4m3(double v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs(v);
    /* E4M3 (OCP): 4 exponent bits (bias 7), 3 mantissa bits, largest finite
     * 448 (0x7E), 0x7F is NaN, smallest normal 2^-6, subnormal quantum 2^-9. */
    double quantum;
    if (a < ldexp(1.0, -6)) {
        quantum = ldexp(1.0, -9);
    } else {
        int ex;
        frexp(a, &ex);
        quantum = ldexp(1.0, (ex - 1) - 3);
    }
    double q = nearbyint(a / quantum) * quantum;
    if (q > 448.0) q = 448.0;
    uint8_t code;
    if (q < ldexp(1.0, -6)) {
        code = (uint8_t)(q / ldexp(1.0, -9));              /* E = 0 */
    } else {
        int ex;
        double f = frexp(q, &ex);                          /* q = f * 2^ex */
        int E = (ex - 1) + 7;
        int m = (int)(f * 16.0) - 8;
        code = (uint8_t)((E << 3) | m);
    }
    return sign | code;
}

double orc_decode_e2m1(uint8_t code)
{
    int s = (code >> 3) & 1, E = (code >> 1) & 3, m = code & 1;
    double mag = (E == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, E - 1);
    return s ? -mag : mag;
}

double orc_decode_e4m3(uint8_t code)
{
    int s = (code >> 7) & 1, E = (code >> 3) & 15, m = code & 7;
    double mag = (E == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, E - 7);
    if (E == 15 && m == 7) mag = NAN;
    return s ? -mag : mag;
}

/* One scale block: amax over n elements, e, and the element codes. */
static void quantize_block(const uint16_t* x, int n, int fmt, uint8_t* codes, int* e_out)
{
    double amax = 0.0;
    for (int i = 0; i < n; ++i) {
        double a = fabs(orc_bf16_to_double(x[i]));
        if (a > amax) amax = a;
    }
    int e = shared_exponent(amax, fmt == ORC_FMT_E2M1 ? 2 : 8);
    for (int i = 0; i < n; ++i) {
        double v = ldexp(orc_bf16_to_double(x[i]), -e);
        codes[i] = (fmt == ORC_FMT_E2M1) ? encode_e2m1(v) : encode_e4m3(v);
    }
    *e_out = e;
}

/* Quantize rows x K. fmt = E2M1: block = G in {16, 32, 64}; fmt = E4M3:
 * block = 32 (G ignored). exps has rows x (K / V) entries with V = 16 when the
 * block is 16, else 32. */
int orc_mx_quantize(const uint16_t* X, int rows, int K, int G, int fmt,
                    uint8_t* codes, int16_t* exps)
{
    if (!X || !codes || !exps || rows < 0 || K <= 0) return -1;
    int blk = (fmt == ORC_FMT_E4M3) ? 32 : G;
    if (fmt != ORC_FMT_E2M1 && fmt != ORC_FMT_E4M3) return -1;
    if (blk != 16 && blk != 32 && blk != 64) return -1;
    if (K % blk) return -1;
    if (!all_finite_bf16(X, (int64_t)rows * K)) return -1;
    int V = (blk == 16) ? 16 : 32;
    int nslot = K / V;
    for (int t = 0; t < rows; ++t)
        for (int b = 0; b < K / blk; ++b) {
            int e;
            quantize_block(X + (int64_t)t * K + (int64_t)b * blk, blk, fmt,
                           codes + (int64_t)t * K + (int64_t)b * blk, &e);
            for (int s = 0; s < blk / V; ++s)
                exps[(int64_t)t * nslot + (int64_t)b * (blk / V) + s] = (int16_t)e;
        }
    return 0;
}

/* Dequantized value of one element: decode(code) * 2^e. */
int orc_mx_dequantize(const uint8_t* codes, const int16_t* exps, int rows, int K,
                      int V, int fmt, double* out)
{
    if (!codes || !exps || !out || rows < 0 || K <= 0 || (V != 16 && V != 32) || K % V) return -1;
    int nslot = K / V;
    for (int t = 0; t < rows; ++t)
        for (int k = 0; k < K; ++k) {
            uint8_t c = codes[(int64_t)t * K + k];
            double d = (fmt == ORC_FMT_E2M1) ? orc_decode_e2m1(c) : orc_decode_e4m3(c);
            out[(int64_t)t * K + k] = ldexp(d, exps[(int64_t)t * nslot + k / V]);
        }
    return 0;
}

/* ---- Dual-path product (§3.2, the equation for Y) ----------------------------
 *
 *   Y = (Q_X (x) Q_W) * S  +  B * W_L
 * Base path: sum over scale slots b of 2^(e_X[t,b] + e_W[n,b]) times the sum of
 * the slot's element products; compensation path: sum over the K_L table
 * columns of B[t,i] * W_L[n,i]. All in fp64. rows (nrows entries, or NULL for
 * all M rows) selects which rows of Y are computed; Y is nrows x N.
 */
int orc_linear(const uint8_t* cx, const int16_t* ex, const uint8_t* cw,
               const int16_t* ew, const uint16_t* B, const uint16_t* WL,
               int M, int N, int K, int V, int fmt, int K_L,
               const int32_t* rows, int nrows, double* Y)
{
    if (!cx || !ex || !cw || !ew || !Y || M < 0 || N < 0 || K <= 0) return -1;
    if ((V != 16 && V != 32) || K % V) return -1;
    if (K_L < 0 || (K_L > 0 && (!B || !WL))) return -1;
    int nslot = K / V;
    int nr = rows ? nrows : M;
    /* decode the selected rows of X once, then each row of W once; every (t, n) sum runs in
     * the same order as the formula: slots ascending, elements ascending within a slot, then
     * the K_L compensation terms ascending */
    double* qx = (double*)malloc((size_t)nr * (size_t)K * sizeof(double));
    double* qw = (double*)malloc((size_t)K * sizeof(double));
    if (!qx || !qw) { free(qx); free(qw); return -1; }
    for (int r = 0; r < nr; ++r) {
        int t = rows ? rows[r] : r;
        if (t < 0 || t >= M) { free(qx); free(qw); return -1; }
        for (int k = 0; k < K; ++k) {
            uint8_t c = cx[(int64_t)t * K + k];
            qx[(int64_t)r * K + k] = (fmt == ORC_FMT_E2M1) ? orc_decode_e2m1(c) : orc_decode_e4m3(c);
        }
    }
    for (int n = 0; n < N; ++n) {
        for (int k = 0; k < K; ++k) {
            uint8_t c = cw[(int64_t)n * K + k];
            qw[k] = (fmt == ORC_FMT_E2M1) ? orc_decode_e2m1(c) : orc_decode_e4m3(c);
        }
        for (int r = 0; r < nr; ++r) {
            int t = rows ? rows[r] : r;
            const double* xr = qx + (int64_t)r * K;
            double acc = 0.0;
            for (int b = 0; b < nslot; ++b) {
                double part = 0.0;
                for (int i = b * V; i < (b + 1) * V; ++i) part += xr[i] * qw[i];
                acc += ldexp(part, ex[(int64_t)t * nslot + b] + ew[(int64_t)n * nslot + b]);
            }
            for (int i = 0; i < K_L; ++i)
                acc += orc_bf16_to_double(B[(int64_t)t * K_L + i]) *
                       orc_bf16_to_double(WL[(int64_t)n * K_L + i]);
            Y[(int64_t)r * N + n] = acc;
        }
    }
    free(qx);
    free(qw);
    return 0;
}
