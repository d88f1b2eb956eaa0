/*
 * echo_oracle.c -- the oracle: a plain CPU restatement of the Echo 4-bit
 * error-compensated all-reduce, simulated over P virtual ranks.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the package smoke check and
 * the benchmark's CPU-baseline leg load this library. The CUDA product path
 * never calls it, and the two share no source, header, table or helper.
 *
 * Style: plain and slow on purpose. Nested loops over ranks, groups and
 * elements; one IEEE binary32 operation per statement (built with
 * -ffp-contract=off and without fast-math, so no fused multiply-add and no
 * reassociation); its own bf16 / fp16 converters written from the IEEE-754
 * definitions of rounding (round-to-nearest-even, toward -inf, toward +inf).
 *
 * Sources. The method is described in prose on two pages; neither prints
 * code or a worked example:
 *   [ABS] "Echo: Error-Compensated 4-Bit Tensor-Parallel Communication for
 *         LLM Training and Inference" (arXiv 2610.14277), abstract.
 *   [EXP] the Japanese explainer "テンソル並列の通信を4bitに圧縮する「Echo」",
 *         sections "Echoの仕組み①" (mechanism 1: add in high precision, move
 *         in low precision), "Echoの仕組み②" (mechanism 2: dual time-constant
 *         feedback), "理論保証" (theory), "よくある質問" (FAQ).
 *
 * What the pages fix:
 *   - the all-reduce is restructured as all-to-all + high-precision sum at
 *     the owner of each segment + all-gather; a rank quantizes only the
 *     segments it does not own, the owner requantizes the sum, so every
 *     value passes through the quantizer at most twice ([EXP] mechanism 1;
 *     [ABS]);
 *   - the quantizer is asymmetric and zero-point aware ([EXP] mechanism 1)
 *     and ships 4-bit integers plus half-precision parameters ([EXP] FAQ);
 *   - the residuals the ranks keep sum to minus the injected error, and are
 *     stored in a long and a short moving average that are added back into
 *     the next call's input, fused into the entry pass ([EXP] mechanism 2);
 *   - an 8-bit mode exists and is used for early layers ([EXP] results).
 *
 * Readings taken where the pages are silent (each also listed in the design
 * notes of the repository):
 *   R1 compensation c = eta * (w * e_short + (1 - w) * e_long), evaluated
 *      t1 = w*e_short; t2 = (1-w)*e_long; c = eta*(t1 + t2); x' = x + c.
 *      Each EMA: e <- (1 - alpha) * e + alpha * rho, evaluated
 *      u = (1-alpha)*e; v = alpha*rho; e = u + v. (1-w), (1-alpha) are
 *      computed once in binary32. State starts at zero and carries from call
 *      to call. Without state, x' = x exactly.
 *   R2 every rank compensates its whole input, owned segment included.
 *   R3 segment s owns groups [floor(s*G/P), floor((s+1)*G/P)); a group is a
 *      contiguous run of `group` elements of the flattened message; the last
 *      group may be partial.
 *   R4 quantizer: mn = min + 0, mx = max + 0 (the +0 turns -0 into +0);
 *      z = fp16_down(mn); s = fp16_up((mx - z) / Q); codes
 *      clamp(rint((v - z) * (1/s)), 0, Q) with rint half-to-even, all codes
 *      0 when s == 0; dequantization (code * s) + z. Directed rounding of
 *      the parameters keeps [z, z + Q*s] around [mn, mx].
 *   R5 packing (4-bit): element 2i in the low nibble and 2i+1 in the high
 *      nibble of byte i of the group's code block; padding codes are 0;
 *      parameters are a pair of fp16 bit patterns {s, z}. 8-bit: one byte
 *      per code.
 *   R6 the owner adds its own x' unquantized; the sum runs in binary32 in
 *      rank order 0, 1, ..., P-1.
 *   R7 with P >= 2 the owner requantizes the sum and every rank, the owner
 *      included, outputs bf16_rn(code * s + z); with P == 1 nothing is sent
 *      and the output is bf16_rn(x').
 *   R8 residuals: a non-owner keeps x' - x_hat; the owner keeps
 *      sum - float(y), y being the bf16 value every rank receives.
 *   R9 values outside [-65504, 65504] (or NaN) in a group that is quantized,
 *      or in a P == 1 output, raise the sticky RANGE flag.
 *
 * Quantizer variants for the ablations (the pages name the asymmetric
 * zero-point form but fix neither the rounding of the half-precision
 * parameters nor whether the zero is a float or an integer):
 *   R10 "nearest": z = fp16_nearest(mn); s = fp16_nearest((mx - mn) / Q);
 *      codes clamp(rint((v - z) * (1/s)), 0, Q) -- the clamp now matters,
 *      because [z, z + Q*s] need not cover [mn, mx]; dequantization as R4.
 *   R11 "integer zero point": the range is widened to include zero,
 *      lo = min(mn, 0), hi = max(mx, 0); s = fp16_up((hi - lo) / Q);
 *      inv = 1/s; zp = clamp(rint(-lo * inv), 0, Q) (0 when s == 0);
 *      codes clamp(rint(v * inv) + zp, 0, Q); dequantization (code - zp) * s,
 *      exact in binary32. The parameter pair carries {s, zp} with zp as an
 *      unsigned 16-bit integer in place of z.
 *
 * The 16-bit baseline the pages compare Echo against ([ABS]; [EXP] results
 * table: "16-bit NCCL all-reduce"), simulated the same way over P virtual
 * ranks: every rank receives bf16_rn(sum_r float(x_r)), the binary32 sum in
 * rank order 0, 1, ..., P-1 (R15: the pages fix neither the order nor the
 * accumulation precision of that all-reduce; this reading takes the same
 * order and precision as R6, so that the two differ only by quantization).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_FLAG_RANGE 1u

/* quantizer forms: R4 (default), R10, R11 */
enum { ORACLE_Q_DIRECTED = 0, ORACLE_Q_NEAREST = 1, ORACLE_Q_INT_ZERO = 2 };

enum { ORACLE_RN = 0, ORACLE_RD = 1, ORACLE_RU = 2 };

/* ------------------------------------------------------------------ */
/* IEEE-754 rounding onto a narrower binary format, from the definition */
/* ------------------------------------------------------------------ */

/*
 * Round the magnitude a > 0 (held exactly in a double) onto the grid of a
 * binary format with a p-bit significand (implicit bit included) and
 * smallest normal exponent emin. `negative` tells which way "down" and "up"
 * point for the directed modes. The result may exceed the format's largest
 * finite value; the caller decides overflow.
 */
static double round_magnitude(double a, int p, int emin, int mode, int negative)
{
    int e;
    frexp(a, &e);           /* a = f * 2^e with 0.5 <= f < 1 */
    int E = e - 1;          /* floor(log2(a)) */
    if (E < emin) {
        E = emin;           /* subnormal range: fixed spacing */
    }
    double ulp = ldexp(1.0, E - (p - 1));
    double q = a / ulp;     /* exact: division by a power of two */
    double lo = floor(q);
    double hi = ceil(q);
    double k;
    if (mode == ORACLE_RN) {
        double dlo = q - lo;
        double dhi = hi - q;
        if (dlo < dhi) {
            k = lo;
        } else if (dhi < dlo) {
            k = hi;
        } else {
            k = (fmod(lo, 2.0) == 0.0) ? lo : hi;   /* tie: even significand */
        }
    } else {
        /* toward +inf grows the magnitude of a positive value, toward -inf
         * grows the magnitude of a negative one */
        int grow = (mode == ORACLE_RU) ? !negative : negative;
        k = grow ? hi : lo;
    }
    return k * ulp;
}

/* overflow rule: round-to-nearest and "magnitude-growing" directed modes go
 * to infinity, the others stop at the largest finite value */
static int overflows_to_inf(int mode, int negative)
{
    if (mode == ORACLE_RN) {
        return 1;
    }
    return (mode == ORACLE_RU) ? !negative : negative;
}

/* binary16: 1 sign, 5 exponent, 10 fraction bits; largest finite 65504 */
static uint16_t encode_f16(double m, int negative)
{
    uint16_t sign = negative ? 0x8000u : 0u;
    if (m == 0.0) {
        return sign;
    }
    if (m < ldexp(1.0, -14)) {
        /* subnormal: m = k * 2^-24, 1 <= k <= 1023 */
        return (uint16_t)(sign | (uint16_t)(m / ldexp(1.0, -24)));
    }
    int e;
    double f = frexp(m, &e);     /* m = (2f) * 2^(e-1), 1 <= 2f < 2 */
    int E = e - 1;
    uint16_t frac = (uint16_t)((2.0 * f - 1.0) * 1024.0);
    return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | frac);
}

uint16_t oracle_f32_to_f16(float x, int mode)
{
    uint32_t u;
    memcpy(&u, &x, 4);
    int negative = (int)(u >> 31);
    if (x != x) {
        return (uint16_t)(negative ? 0xFE00u : 0x7E00u);
    }
    double a = fabs((double)x);
    if (isinf(a)) {
        return (uint16_t)(negative ? 0xFC00u : 0x7C00u);
    }
    if (a == 0.0) {
        return (uint16_t)(negative ? 0x8000u : 0u);
    }
    double m = round_magnitude(a, 11, -14, mode, negative);
    if (m > 65504.0) {
        if (overflows_to_inf(mode, negative)) {
            return (uint16_t)(negative ? 0xFC00u : 0x7C00u);
        }
        m = 65504.0;
    }
    return encode_f16(m, negative);
}

float oracle_f16_to_f32(uint16_t h)
{
    int negative = (h >> 15) & 1;
    int E = (h >> 10) & 0x1F;
    int F = h & 0x3FF;
    double v;
    if (E == 0) {
        v = ldexp((double)F, -24);
    } else if (E == 31) {
        v = (F != 0) ? NAN : INFINITY;
    } else {
        v = ldexp(1.0 + (double)F / 1024.0, E - 15);
    }
    return (float)(negative ? -v : v);
}

/* bfloat16: the top half of a binary32 word (8 exponent, 7 fraction bits) */
float oracle_bf16_to_f32(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

uint16_t oracle_f32_to_bf16(float x)
{
    uint32_t u;
    memcpy(&u, &x, 4);
    int negative = (int)(u >> 31);
    uint16_t sign = negative ? 0x8000u : 0u;
    if (x != x) {
        return (uint16_t)(sign | 0x7FC0u);
    }
    double a = fabs((double)x);
    if (isinf(a)) {
        return (uint16_t)(sign | 0x7F80u);
    }
    if (a == 0.0) {
        return sign;
    }
    const double bf16_max = ldexp(255.0, 127 - 7);   /* (2 - 2^-7) * 2^127 */
    double m = round_magnitude(a, 8, -126, ORACLE_RN, negative);
    if (m > bf16_max) {
        return (uint16_t)(sign | 0x7F80u);
    }
    float mf = (float)m;        /* exact: every bf16 value is a binary32 value */
    uint32_t mu;
    memcpy(&mu, &mf, 4);
    return (uint16_t)(sign | (uint16_t)(mu >> 16));
}

/* ------------------------------------------------------------------ */
/* Group quantizer (reading R4)                                         */
/* ------------------------------------------------------------------ */

static int outside_domain(float v)
{
    /* NaN fails both comparisons */
    return !(v >= -65504.0f && v <= 65504.0f);
}

/* clamp(rint(u) + add, 0, Q) with rint half to even (the default rounding mode) */
static int round_clamp(float u, int add, int Q)
{
    float r = rintf(u);
    int c;
    if (r != r) {
        c = -1024;      /* NaN: only in a group already flagged out of range */
    } else if (r < -1024.0f) {
        c = -1024;
    } else if (r > 1024.0f) {
        c = 1024;
    } else {
        c = (int)r;
    }
    c = c + add;
    if (c < 0) {
        c = 0;
    }
    if (c > Q) {
        c = Q;
    }
    return c;
}

/*
 * Quantize m values of one group to codes in [0, Q] with quantizer form
 * `qmode` (R4, R10 or R11). Writes one code per element (unpacked), the two
 * 16-bit parameter words (fp16 s, and fp16 z or the integer zero point), and
 * the dequantized values. Returns ORACLE_FLAG_RANGE when a value lies outside
 * the fp16 parameter domain, 0 otherwise.
 */
uint32_t oracle_quantize_group_q(const float* v, int m, int bits, int qmode, uint8_t* codes,
                                 uint16_t* s_bits, uint16_t* z_bits, float* vhat)
{
    int Q = (1 << bits) - 1;
    uint32_t flag = 0;
    float mn = v[0];
    float mx = v[0];
    for (int i = 0; i < m; i++) {
        if (outside_domain(v[i])) {
            flag = ORACLE_FLAG_RANGE;
        }
        if (v[i] < mn) {
            mn = v[i];
        }
        if (v[i] > mx) {
            mx = v[i];
        }
    }
    mn = mn + 0.0f;
    mx = mx + 0.0f;
    if (qmode == ORACLE_Q_INT_ZERO) {
        float lo = mn < 0.0f ? mn : 0.0f;
        float hi = mx > 0.0f ? mx : 0.0f;
        float d = hi - lo;
        float step = d / (float)Q;
        uint16_t sh = oracle_f32_to_f16(step, ORACLE_RU);
        float s = oracle_f16_to_f32(sh);
        int zp = 0;
        float inv = 0.0f;
        if (s != 0.0f) {
            inv = 1.0f / s;
            float nlo = -lo;
            float t = nlo * inv;
            zp = round_clamp(t, 0, Q);
        }
        for (int i = 0; i < m; i++) {
            int c = 0;
            if (s != 0.0f) {
                float u = v[i] * inv;
                c = round_clamp(u, zp, Q);
            }
            codes[i] = (uint8_t)c;
            int k = c - zp;
            vhat[i] = (float)k * s;       /* exact: |k| <= 255, s has 11 bits */
        }
        *s_bits = sh;
        *z_bits = (uint16_t)zp;
        return flag;
    }
    uint16_t zh;
    uint16_t sh;
    if (qmode == ORACLE_Q_NEAREST) {
        zh = oracle_f32_to_f16(mn, ORACLE_RN);
        float d = mx - mn;
        float step = d / (float)Q;
        sh = oracle_f32_to_f16(step, ORACLE_RN);
    } else {
        zh = oracle_f32_to_f16(mn, ORACLE_RD);
        float zd = oracle_f16_to_f32(zh);
        float d = mx - zd;
        float step = d / (float)Q;
        sh = oracle_f32_to_f16(step, ORACLE_RU);
    }
    float z = oracle_f16_to_f32(zh);
    float s = oracle_f16_to_f32(sh);
    float inv = 0.0f;
    if (s != 0.0f) {
        inv = 1.0f / s;
    }
    for (int i = 0; i < m; i++) {
        int c = 0;
        if (s != 0.0f) {
            float t = v[i] - z;
            float u = t * inv;
            c = round_clamp(u, 0, Q);
        }
        codes[i] = (uint8_t)c;
        float cs = (float)c * s;
        vhat[i] = cs + z;
    }
    *s_bits = sh;
    *z_bits = zh;
    return flag;
}

/* the default form (R4) */
uint32_t oracle_quantize_group(const float* v, int m, int bits, uint8_t* codes,
                               uint16_t* s_bits, uint16_t* z_bits, float* vhat)
{
    return oracle_quantize_group_q(v, m, bits, ORACLE_Q_DIRECTED, codes, s_bits, z_bits, vhat);
}

/* dequantize one code with the parameter words of its group */
static float dequant(int code, uint16_t s_bits, uint16_t z_bits, int qmode)
{
    float s = oracle_f16_to_f32(s_bits);
    if (qmode == ORACLE_Q_INT_ZERO) {
        int k = code - (int)z_bits;
        return (float)k * s;
    }
    float z = oracle_f16_to_f32(z_bits);
    float cs = (float)code * s;
    return cs + z;
}

/* ------------------------------------------------------------------ */
/* Packing (reading R5)                                                 */
/* ------------------------------------------------------------------ */

void oracle_pack_codes(const uint8_t* codes, int group, int bits, uint8_t* out)
{
    if (bits == 8) {
        for (int i = 0; i < group; i++) {
            out[i] = codes[i];
        }
        return;
    }
    for (int i = 0; i < group / 2; i++) {
        uint8_t lo = (uint8_t)(codes[2 * i] & 0xF);
        uint8_t hi = (uint8_t)(codes[2 * i + 1] & 0xF);
        out[i] = (uint8_t)(lo | (hi << 4));
    }
}

void oracle_unpack_codes(const uint8_t* packed, int group, int bits, uint8_t* codes)
{
    if (bits == 8) {
        for (int i = 0; i < group; i++) {
            codes[i] = packed[i];
        }
        return;
    }
    for (int i = 0; i < group / 2; i++) {
        codes[2 * i] = (uint8_t)(packed[i] & 0xF);
        codes[2 * i + 1] = (uint8_t)(packed[i] >> 4);
    }
}

/* ------------------------------------------------------------------ */
/* Segments and owners (reading R3)                                     */
/* ------------------------------------------------------------------ */

long long oracle_segment_begin(int s, long long G, int P)
{
    return ((long long)s * G) / P;
}

int oracle_owner(long long j, long long G, int P)
{
    for (int s = 0; s < P; s++) {
        if (j >= oracle_segment_begin(s, G, P) && j < oracle_segment_begin(s + 1, G, P)) {
            return s;
        }
    }
    return -1;
}

/* ------------------------------------------------------------------ */
/* Feedback pieces (reading R1)                                         */
/* ------------------------------------------------------------------ */

float oracle_compensation(float e_long, float e_short, float eta, float w)
{
    float one_minus_w = 1.0f - w;
    float t1 = w * e_short;
    float t2 = one_minus_w * e_long;
    float sum = t1 + t2;
    return eta * sum;
}

void oracle_ema_update(float* e, const float* rho, long long count, float alpha)
{
    float keep = 1.0f - alpha;
    for (long long i = 0; i < count; i++) {
        float u = keep * e[i];
        float v = alpha * rho[i];
        e[i] = u + v;
    }
}

/* ------------------------------------------------------------------ */
/* One all-reduce call over the group columns [j0, j0 + jc)             */
/* ------------------------------------------------------------------ */

/*
 * Arguments (all host memory, element (r, k) at index r * ld + k with
 * ld = jc * group; local element k is message element j0 * group + k and is
 * ignored when that index is >= n_total):
 *   x        [P][ld] bf16 bit patterns, the ranks' partial sums (input)
 *   y        [P][ld] bf16 bit patterns, the reduced result of each rank
 *   e_long, e_short  [P][ld] binary32 EMAs updated in place; both NULL
 *            means "no feedback state" (x' = x, no update)
 *   a2a_codes   [P][jc][group*bits/8] packed all-to-all payload; the slot
 *            of a group's owner is left untouched          (may be NULL)
 *   a2a_params  [P][jc][2] {s, z} (or {s, zp}, R11) of that payload (may be NULL)
 *   gather_codes [jc][group*bits/8], gather_params [jc][2]: the owner's
 *            requantized sum, sent to every rank            (may be NULL;
 *            untouched when P == 1)
 *   xprime, rho [P][ld] binary32 debug copies of x' and the residuals
 *   passes   [P][ld] number of quantizer passes each rank's contribution to
 *            an element went through in this call          (debug, may be NULL)
 *   flags    sticky flag word, ORACLE_FLAG_RANGE on a domain violation
 * Returns 0, or -1 on invalid arguments / allocation failure.
 */
int oracle_echo_allreduce_q(int P, long long n_total, int group, int bits, int qmode,
                            long long j0, long long jc,
                            const uint16_t* x, uint16_t* y,
                            float* e_long, float* e_short,
                            float eta, float alpha_long, float alpha_short, float w,
                            uint8_t* a2a_codes, uint16_t* a2a_params,
                            uint8_t* gather_codes, uint16_t* gather_params,
                            float* xprime, float* rho, uint8_t* passes,
                            uint32_t* flags)
{
    if (P < 1 || n_total < 1 || group < 2 || (bits != 4 && bits != 8) || jc < 0 || j0 < 0 ||
        qmode < ORACLE_Q_DIRECTED || qmode > ORACLE_Q_INT_ZERO) {
        return -1;
    }
    long long G = (n_total + group - 1) / group;
    if (j0 + jc > G) {
        return -1;
    }
    int feedback = (e_long != NULL && e_short != NULL);
    long long ld = jc * group;
    long long cb = (long long)group * bits / 8;    /* code bytes per group */
    size_t nel = (size_t)P * (size_t)ld;

    float* xp = (float*)malloc(nel * sizeof(float) + 1);
    float* res = (float*)malloc(nel * sizeof(float) + 1);
    uint8_t* a2a_c = a2a_codes;
    uint16_t* a2a_p = a2a_params;
    uint8_t* g_c = gather_codes;
    uint16_t* g_p = gather_params;
    uint8_t* own_a2a_c = NULL;
    uint16_t* own_a2a_p = NULL;
    uint8_t* own_g_c = NULL;
    uint16_t* own_g_p = NULL;
    if (a2a_c == NULL) {
        own_a2a_c = (uint8_t*)calloc((size_t)P * (size_t)(jc * cb) + 1, 1);
        a2a_c = own_a2a_c;
    }
    if (a2a_p == NULL) {
        own_a2a_p = (uint16_t*)calloc((size_t)P * (size_t)jc * 2 + 1, sizeof(uint16_t));
        a2a_p = own_a2a_p;
    }
    if (g_c == NULL) {
        own_g_c = (uint8_t*)calloc((size_t)(jc * cb) + 1, 1);
        g_c = own_g_c;
    }
    if (g_p == NULL) {
        own_g_p = (uint16_t*)calloc((size_t)jc * 2 + 1, sizeof(uint16_t));
        g_p = own_g_p;
    }
    float* sum = (float*)malloc((size_t)group * sizeof(float));
    float* vtmp = (float*)malloc((size_t)group * sizeof(float));
    float* vhat = (float*)malloc((size_t)group * sizeof(float));
    uint8_t* codes = (uint8_t*)malloc((size_t)group);
    uint16_t* y_owner = (uint16_t*)malloc((size_t)group * sizeof(uint16_t));
    if (!xp || !res || !a2a_c || !a2a_p || !g_c || !g_p || !sum || !vtmp || !vhat || !codes || !y_owner) {
        free(xp); free(res); free(own_a2a_c); free(own_a2a_p); free(own_g_c); free(own_g_p);
        free(sum); free(vtmp); free(vhat); free(codes); free(y_owner);
        return -1;
    }
    if (passes != NULL) {
        memset(passes, 0, nel);
    }
    uint32_t flag = 0;

    /* Phase 1: feedback injection on every rank's whole input (R1, R2). */
    for (int r = 0; r < P; r++) {
        for (long long k = 0; k < ld; k++) {
            size_t idx = (size_t)r * (size_t)ld + (size_t)k;
            if (j0 * group + k >= n_total) {
                xp[idx] = 0.0f;
                res[idx] = 0.0f;
                continue;
            }
            float xv = oracle_bf16_to_f32(x[idx]);
            if (feedback) {
                float c = oracle_compensation(e_long[idx], e_short[idx], eta, w);
                xp[idx] = xv + c;
            } else {
                xp[idx] = xv;
            }
            res[idx] = 0.0f;
        }
    }

    /* Phase 2: each rank quantizes the groups it does not own -> all-to-all
     * payload slot [r][j]; the sender keeps its residual x' - x_hat (R8). */
    for (long long jl = 0; jl < jc; jl++) {
        long long j = j0 + jl;
        int o = oracle_owner(j, G, P);
        long long e0 = j * group;
        int m = (int)((n_total - e0 < group) ? (n_total - e0) : group);
        for (int r = 0; r < P; r++) {
            if (r == o) {
                continue;
            }
            size_t base = (size_t)r * (size_t)ld + (size_t)(jl * group);
            uint16_t sb;
            uint16_t zb;
            flag |= oracle_quantize_group_q(&xp[base], m, bits, qmode, codes, &sb, &zb, vhat);
            for (int i = m; i < group; i++) {
                codes[i] = 0;                       /* padding of a partial group */
            }
            size_t slot = (size_t)r * (size_t)jc + (size_t)jl;
            oracle_pack_codes(codes, group, bits, &a2a_c[slot * (size_t)cb]);
            a2a_p[2 * slot] = sb;
            a2a_p[2 * slot + 1] = zb;
            for (int i = 0; i < m; i++) {
                res[base + (size_t)i] = xp[base + (size_t)i] - vhat[i];
                if (passes != NULL) {
                    passes[base + (size_t)i] = (uint8_t)(passes[base + (size_t)i] + 1);
                }
            }
        }
    }

    /* Phase 3: the owner decodes what it received, sums in binary32 in rank
     * order with its own unquantized x' (R6) and requantizes the sum into the
     * all-gather payload (R7). Its residual is sum - float(y) (R8). */
    for (long long jl = 0; jl < jc; jl++) {
        long long j = j0 + jl;
        int o = oracle_owner(j, G, P);
        long long e0 = j * group;
        int m = (int)((n_total - e0 < group) ? (n_total - e0) : group);
        for (int i = 0; i < m; i++) {
            sum[i] = 0.0f;
        }
        for (int r = 0; r < P; r++) {
            size_t base = (size_t)r * (size_t)ld + (size_t)(jl * group);
            if (r == o) {
                for (int i = 0; i < m; i++) {
                    vtmp[i] = xp[base + (size_t)i];
                }
            } else {
                size_t slot = (size_t)r * (size_t)jc + (size_t)jl;
                oracle_unpack_codes(&a2a_c[slot * (size_t)cb], group, bits, codes);
                for (int i = 0; i < m; i++) {
                    vtmp[i] = dequant(codes[i], a2a_p[2 * slot], a2a_p[2 * slot + 1], qmode);
                }
            }
            for (int i = 0; i < m; i++) {
                if (r == 0) {
                    sum[i] = vtmp[i];
                } else {
                    sum[i] = sum[i] + vtmp[i];
                }
            }
        }
        size_t obase = (size_t)o * (size_t)ld + (size_t)(jl * group);
        if (P >= 2) {
            uint16_t sb;
            uint16_t zb;
            flag |= oracle_quantize_group_q(sum, m, bits, qmode, codes, &sb, &zb, vhat);
            for (int i = m; i < group; i++) {
                codes[i] = 0;
            }
            oracle_pack_codes(codes, group, bits, &g_c[(size_t)jl * (size_t)cb]);
            g_p[2 * jl] = sb;
            g_p[2 * jl + 1] = zb;
            for (int i = 0; i < m; i++) {
                y_owner[i] = oracle_f32_to_bf16(vhat[i]);
                if (passes != NULL) {
                    for (int r = 0; r < P; r++) {
                        size_t b = (size_t)r * (size_t)ld + (size_t)(jl * group) + (size_t)i;
                        passes[b] = (uint8_t)(passes[b] + 1);
                    }
                }
            }
        } else {
            for (int i = 0; i < m; i++) {
                if (outside_domain(sum[i])) {
                    flag |= ORACLE_FLAG_RANGE;
                }
                y_owner[i] = oracle_f32_to_bf16(sum[i]);
            }
        }
        for (int i = 0; i < m; i++) {
            res[obase + (size_t)i] = sum[i] - oracle_bf16_to_f32(y_owner[i]);
        }
        if (P == 1) {
            for (int i = 0; i < m; i++) {
                y[obase + (size_t)i] = y_owner[i];
            }
        }
    }

    /* Phase 4: every rank dequantizes the gathered payload (P >= 2). */
    if (P >= 2) {
        for (long long jl = 0; jl < jc; jl++) {
            long long e0 = (j0 + jl) * group;
            int m = (int)((n_total - e0 < group) ? (n_total - e0) : group);
            oracle_unpack_codes(&g_c[(size_t)jl * (size_t)cb], group, bits, codes);
            for (int r = 0; r < P; r++) {
                size_t base = (size_t)r * (size_t)ld + (size_t)(jl * group);
                for (int i = 0; i < m; i++) {
                    float v = dequant(codes[i], g_p[2 * jl], g_p[2 * jl + 1], qmode);
                    y[base + (size_t)i] = oracle_f32_to_bf16(v);
                }
            }
        }
    }

    /* Phase 5: the residuals update both EMAs of every rank (R1). */
    if (feedback) {
        for (int r = 0; r < P; r++) {
            for (long long jl = 0; jl < jc; jl++) {
                long long e0 = (j0 + jl) * group;
                int m = (int)((n_total - e0 < group) ? (n_total - e0) : group);
                size_t base = (size_t)r * (size_t)ld + (size_t)(jl * group);
                oracle_ema_update(&e_long[base], &res[base], m, alpha_long);
                oracle_ema_update(&e_short[base], &res[base], m, alpha_short);
            }
        }
    }

    if (xprime != NULL) {
        memcpy(xprime, xp, nel * sizeof(float));
    }
    if (rho != NULL) {
        memcpy(rho, res, nel * sizeof(float));
    }
    if (flags != NULL) {
        *flags |= flag;
    }
    free(xp); free(res); free(own_a2a_c); free(own_a2a_p); free(own_g_c); free(own_g_p);
    free(sum); free(vtmp); free(vhat); free(codes); free(y_owner);
    return 0;
}

/* the default quantizer form (R4) */
int oracle_echo_allreduce(int P, long long n_total, int group, int bits,
                          long long j0, long long jc,
                          const uint16_t* x, uint16_t* y,
                          float* e_long, float* e_short,
                          float eta, float alpha_long, float alpha_short, float w,
                          uint8_t* a2a_codes, uint16_t* a2a_params,
                          uint8_t* gather_codes, uint16_t* gather_params,
                          float* xprime, float* rho, uint8_t* passes,
                          uint32_t* flags)
{
    return oracle_echo_allreduce_q(P, n_total, group, bits, ORACLE_Q_DIRECTED, j0, jc, x, y, e_long, e_short,
                                   eta, alpha_long, alpha_short, w, a2a_codes, a2a_params, gather_codes,
                                   gather_params, xprime, rho, passes, flags);
}

/* ------------------------------------------------------------------ */
/* The 16-bit baseline all-reduce (reading R15)                         */
/* ------------------------------------------------------------------ */

/* x: P rows of n bf16 bit patterns (row r at x + r * n); y: P rows of n, every
 * row receives the same bf16 result. */
void oracle_bf16_allreduce(int P, long long n, const uint16_t* x, uint16_t* y)
{
    for (long long i = 0; i < n; i++) {
        float sum = 0.0f;
        for (int r = 0; r < P; r++) {
            float v = oracle_bf16_to_f32(x[(size_t)r * (size_t)n + (size_t)i]);
            if (r == 0) {
                sum = v;
            } else {
                sum = sum + v;
            }
        }
        uint16_t out = oracle_f32_to_bf16(sum);
        for (int r = 0; r < P; r++) {
            y[(size_t)r * (size_t)n + (size_t)i] = out;
        }
    }
}
