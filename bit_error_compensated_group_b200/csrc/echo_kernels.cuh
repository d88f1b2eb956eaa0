// echo_kernels.cuh -- shared device helpers of the Echo all-reduce
// simulation, and the scalar per-group paths.
//
// The stages of the restructured all-reduce of the Echo explainer
// ("Echoの仕組み①": all-to-all of 4-bit non-owned segments, high-precision
// sum at the owner, 4-bit all-gather), with the feedback of "Echoの仕組み②"
// fused into the passes that read the inputs (kernels in echo_pipeline.cuh):
//
//   quantize  every rank's non-owned groups: x' = x + c, group min/max,
//             fp16 {s, z}, packed codes -> all-to-all payload; residual
//             x' - x_hat -> both EMAs.
//   reduce    every group at its owner: x'_owner + dequantized payloads in
//             rank order (binary32), requantize -> all-gather payload;
//             residual sum - y -> the owner's EMAs; in a whole call it also
//             writes the decoded result into all P outputs (phase 4).
//   gather    phase 4 on its own: dequantize the gathered payload once and
//             write the bf16 result into all P outputs (echo_phase_gather;
//             one rank of a multi-GPU call decodes with k_decode_rank).
//
// A call is the first two kernels.
//
// This file holds the argument block, the per-group grid (fp16 zero rounded
// toward -inf from the minimum, fp16 step rounded toward +inf from
// (max - z)/Q), and quantize_range / reduce_range: the same stages written
// one element at a time with global loads and stores guarded against the
// message end. The kernels use them for a partial last group (its byte size
// is not a multiple of 16, so bulk copies cannot move it).
//
// Thread layout: a group of GROUP elements is handled by L = GROUP/8 lanes;
// lane t holds the two 4-element chunks t and t+L, so every load and store
// instruction of a group covers one contiguous span. Group min/max use
// xor-shuffles inside the L lanes. Arithmetic is binary32 with explicit
// round-to-nearest intrinsics (__fadd_rn / __fmul_rn / __fdiv_rn never
// contract into FMA) and the directed fp16 conversions, so results are
// bit-reproducible.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "echo.h"

namespace echo_dev {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kThreads = 256;

struct Args {
    const uint16_t* in[ECHO_MAX_RANKS];   // bf16 bit patterns
    uint16_t* out[ECHO_MAX_RANKS];
    float* state;                         // [P][2][S] or nullptr (no feedback)
    uint8_t* a2a_codes;                   // [P][G][CB]
    uint32_t* a2a_params;                 // [P][G]
    uint8_t* g_codes;                     // [G][CB]
    uint32_t* g_params;                   // [G]
    uint32_t* flags;
    long long n, G, S;
    int P;
    float eta, w, one_minus_w;
    float a_long, keep_long, a_short, keep_short;
    float one;   // 1.0f, passed at run time (see add_after_mul2 in echo_pipeline.cuh)
    int write_outputs;   // reduce: also decode into all P outputs (phase 4 in the owner's pass)
    // the call's group columns: full groups [c0, c1) (c1 <= n / group; the
    // whole message: 0, n / group) and, when tail != 0, the partial last group
    long long c0, c1;
    int tail;
    // Which ranks a launch serves and how their buffers are addressed. The
    // single-GPU simulation serves ranks [0, P) with the layouts above
    // (rank_lo 0, rank_hi P, a2a_stride G, every base 0, g_seg_stride 0).
    // One rank of a multi-GPU call (rank_lo = r, rank_hi = r + 1) holds
    // only its own rows: its EMA state (state_rank_base = r), its all-to-all
    // send row or the P received rows of its segment, its gather send
    // buffer, and the P gathered segments padded to g_seg_stride groups.
    int rank_lo, rank_hi;           // quantize: these ranks' runs; reduce: these owners' runs
    int state_rank_base;            // state row of rank r: r - state_rank_base
    int a2a_rank_base;              // all-to-all slot (r, j): row r - a2a_rank_base,
    long long a2a_stride;           //   of a2a_stride groups, column j - a2a_col_base
    long long a2a_col_base;
    long long g_col_base;           // gather payload written at j - g_col_base
    long long g_seg_stride;         // > 0: gathered payload read as [owner][g_seg_stride]
    int out_lo, out_hi;             // gather decode: outputs of ranks [out_lo, out_hi)
    // limit of every bounded device-side wait (mbarrier waits of the
    // bulk-copy pipelines), in nanoseconds of the global timer
    unsigned long long wait_ns;
    // chunk_k > 0: one rank of a multi-GPU call runs chunk chunk_i of
    // chunk_k: of every owner's segment only its chunk_i-th part,
    // [sb + floor(chunk_i len / chunk_k), sb + floor((chunk_i + 1) len / chunk_k))
    // (len = the segment's groups), so that each chunk's exchanges are
    // balanced over the owners
    int chunk_i, chunk_k;
};

// Owner s's segment [sb, se) of G groups over P ranks, or, in a chunked call,
// that segment's part for chunk chunk_i of chunk_k.
__device__ __forceinline__ void segment_part(const Args& a, int s, long long* b, long long* e) {
    const long long sb = (long long)s * a.G / a.P, se = (long long)(s + 1) * a.G / a.P;
    if (a.chunk_k > 0) {
        const long long len = se - sb;
        *b = sb + (long long)a.chunk_i * len / a.chunk_k;
        *e = sb + (long long)(a.chunk_i + 1) * len / a.chunk_k;
    } else {
        *b = sb;
        *e = se;
    }
}

__device__ __forceinline__ size_t a2a_slot(const Args& a, int r, long long j) {
    return (size_t)(r - a.a2a_rank_base) * (size_t)a.a2a_stride + (size_t)(j - a.a2a_col_base);
}

// The pipelined kernels' simulation instantiations (RK = false) keep the
// plain [P][G] slot and [P][2][S] state addressing; one rank of a
// multi-GPU call (RK = true) uses the general form above. In that mode every
// buffer an Args points at -- the received rows included, which the caller's
// collectives land there -- is this GPU's own memory: the bulk copies and L2
// prefetches of the pipelines never read another GPU's memory, and Args must
// never carry a peer pointer (no load here uses cluster multicast either).
template <bool RK>
__device__ __forceinline__ size_t a2a_slot_t(const Args& a, int r, long long j) {
    return RK ? a2a_slot(a, r, j) : (size_t)r * (size_t)a.G + (size_t)j;
}

__device__ __forceinline__ float* state_row(const Args& a, int r) {
    return a.state + (size_t)(r - a.state_rank_base) * 2 * (size_t)a.S;
}

template <bool RK>
__device__ __forceinline__ float* state_row_t(const Args& a, int r) {
    return RK ? state_row(a, r) : a.state + (size_t)r * 2 * (size_t)a.S;
}

// where the gather payload of group j is read: group j itself, or, for a
// gathered buffer of P owner segments padded to g_seg_stride groups, its
// place in its owner's segment (owner(j) = (j P + P - 1) / G, the segment
// starting at floor(owner G / P))
__device__ __forceinline__ size_t g_read_slot(const Args& a, long long j) {
    if (a.g_seg_stride == 0) return (size_t)j;
    const long long o = (j * a.P + a.P - 1) / a.G;
    return (size_t)(o * a.g_seg_stride + j - o * a.G / a.P);
}

// ------------------------------------------------------------------ helpers

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

__device__ __forceinline__ uint32_t f2bf16(float v) {
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v));
}

__device__ __forceinline__ bool outside_fp16_domain(float v) {
    return !(v >= -65504.0f && v <= 65504.0f);   // NaN fails both
}

// Quantizer forms (template parameter QM): 0 = fp16 zero rounded toward -inf
// from the minimum and step rounded toward +inf from (max - z) / Q (the
// default); 1 = zero and step (max - min) / Q both rounded to nearest, codes
// clamped; 2 = integer zero point: range widened to include 0, step rounded
// up, zp = rint(-lo / s), code = rint(v / s) + zp, value (code - zp) * s.
constexpr int kQuantDirected = 0, kQuantNearest = 1, kQuantIntZero = 2;

// Quantization grid of one group. A code c decodes to c * s + zf (c * s is
// exact); encoding rounds (v - zsub) * inv to an integer and adds zq.
struct Grid {
    float s, zf, zsub, inv;
    int zq;
    uint32_t param;   // s | z << 16 (fp16 bits), or s | zp << 16 for the integer zero point
};

// Parameters of a group from its range [mn, mx] (both already +0-canonical).
template <int Q, int QM>
__device__ __forceinline__ Grid group_grid(float mn, float mx) {
    Grid g;
    if (QM == kQuantIntZero) {
        const float lo = mn < 0.0f ? mn : 0.0f, hi = mx > 0.0f ? mx : 0.0f;
        const __half sh = __float2half_ru(__fdiv_rn(__fsub_rn(hi, lo), (float)Q));
        g.s = __half2float(sh);
        g.inv = (g.s != 0.0f) ? __fdiv_rn(1.0f, g.s) : 0.0f;
        int zp = 0;
        if (g.s != 0.0f) zp = min(max(__float2int_rn(__fmul_rn(-lo, g.inv)), 0), Q);
        g.zq = zp;
        g.zsub = 0.0f;
        g.zf = __fmul_rn(__int2float_rn(-zp), g.s);   // exact: |zp| <= 255, s has 11 bits
        g.param = (uint32_t)__half_as_ushort(sh) | ((uint32_t)zp << 16);
        return g;
    }
    __half zh, sh;
    if (QM == kQuantNearest) {
        zh = __float2half_rn(mn);
        sh = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), (float)Q));
    } else {
        zh = __float2half_rd(mn);
        sh = __float2half_ru(__fdiv_rn(__fsub_rn(mx, __half2float(zh)), (float)Q));
    }
    g.s = __half2float(sh);
    g.zf = g.zsub = __half2float(zh);
    g.zq = 0;
    g.inv = (g.s != 0.0f) ? __fdiv_rn(1.0f, g.s) : 0.0f;   // s == 0 -> every code 0
    g.param = (uint32_t)__half_as_ushort(sh) | ((uint32_t)__half_as_ushort(zh) << 16);
    return g;
}

template <int L>
__device__ __forceinline__ float group_min(float v) {
#pragma unroll
    for (int o = L / 2; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(kFull, v, o));
    return v;
}

template <int L>
__device__ __forceinline__ float group_max(float v) {
#pragma unroll
    for (int o = L / 2; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
    return v;
}

// All 32 lanes must call this (it shuffles); lanes of an inactive group pass
// neutral values and ignore the result.
template <int L, int Q, int QM>
__device__ __forceinline__ Grid make_grid(float lane_min, float lane_max) {
    const float mn = __fadd_rn(group_min<L>(lane_min), 0.0f);   // -0 -> +0
    const float mx = __fadd_rn(group_max<L>(lane_max), 0.0f);
    return group_grid<Q, QM>(mn, mx);
}

template <int Q, int QM>
__device__ __forceinline__ int encode(float v, const Grid& g) {
    float u = __fmul_rn(__fsub_rn(v, g.zsub), g.inv);
    if (QM != kQuantDirected) u = fminf(fmaxf(u, -(float)(Q + 1)), (float)(Q + 1));   // rint, then clamp, agree
    const int q = __float2int_rn(u) + g.zq;   // half to even
    return min(max(q, 0), Q);
}

__device__ __forceinline__ float decode(int q, float s, float zf) {
    return __fadd_rn(__fmul_rn(__int2float_rn(q), s), zf);   // q*s is exact
}

__device__ __forceinline__ float param_s(uint32_t p) { return __half2float(__ushort_as_half((unsigned short)(p & 0xffffu))); }
__device__ __forceinline__ float param_z(uint32_t p) { return __half2float(__ushort_as_half((unsigned short)(p >> 16))); }
// the additive term of a group's decode, c * s + zf, from its parameter word
template <int QM>
__device__ __forceinline__ float param_zf(uint32_t p, float s) {
    if (QM == kQuantIntZero) return __fmul_rn(__int2float_rn(-(int)(p >> 16)), s);   // -zp * s, exact
    return param_z(p);
}

// codes of one 4-element chunk: 4 nibbles in 16 bits, or 4 bytes in 32 bits
template <int BITS>
__device__ __forceinline__ uint32_t pack4(const int q[4]) {
    if (BITS == 4) return (uint32_t)q[0] | ((uint32_t)q[1] << 4) | ((uint32_t)q[2] << 8) | ((uint32_t)q[3] << 12);
    return (uint32_t)q[0] | ((uint32_t)q[1] << 8) | ((uint32_t)q[2] << 16) | ((uint32_t)q[3] << 24);
}

template <int BITS>
__device__ __forceinline__ int unpack1(uint32_t w, int k) {
    return BITS == 4 ? (int)((w >> (4 * k)) & 0xfu) : (int)((w >> (8 * k)) & 0xffu);
}

template <int BITS>
__device__ __forceinline__ void store_chunk_codes(uint8_t* group_codes, int chunk, uint32_t w) {
    if (BITS == 4) *reinterpret_cast<uint16_t*>(group_codes + 2 * chunk) = (uint16_t)w;
    else *reinterpret_cast<uint32_t*>(group_codes + 4 * chunk) = w;
}

template <int BITS>
__device__ __forceinline__ uint32_t load_chunk_codes(const uint8_t* group_codes, int chunk) {
    if (BITS == 4) return (uint32_t)*reinterpret_cast<const uint16_t*>(group_codes + 2 * chunk);
    return *reinterpret_cast<const uint32_t*>(group_codes + 4 * chunk);
}

// 4 bf16 values starting at element e (full chunk: one 8-byte load)
__device__ __forceinline__ void load_x4(const uint16_t* x, long long e, long long n, bool full, float v[4]) {
    if (full) {
        const uint2 u = __ldcs(reinterpret_cast<const uint2*>(x + e));
        v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) v[k] = (e + k < n) ? __uint_as_float((uint32_t)x[e + k] << 16) : 0.0f;
    }
}

__device__ __forceinline__ void store_y4(uint16_t* y, long long e, long long n, bool full, const uint32_t b[4]) {
    if (full) {
        uint2 u;
        u.x = b[0] | (b[1] << 16);
        u.y = b[2] | (b[3] << 16);
        __stcs(reinterpret_cast<uint2*>(y + e), u);
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) if (e + k < n) y[e + k] = (uint16_t)b[k];
    }
}

__device__ __forceinline__ void load_f4(const float* p, long long e, long long n, bool full, float v[4]) {
    if (full) {
        const float4 u = __ldcs(reinterpret_cast<const float4*>(p + e));
        v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) v[k] = (e + k < n) ? p[e + k] : 0.0f;
    }
}

__device__ __forceinline__ void store_f4(float* p, long long e, long long n, bool full, const float v[4]) {
    if (full) {
        __stcs(reinterpret_cast<float4*>(p + e), make_float4(v[0], v[1], v[2], v[3]));
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) if (e + k < n) p[e + k] = v[k];
    }
}

// c = eta * (w * e_short + (1 - w) * e_long);  x' = x + c
__device__ __forceinline__ float inject(float x, float el, float es, const Args& a) {
    const float c = __fmul_rn(a.eta, __fadd_rn(__fmul_rn(a.w, es), __fmul_rn(a.one_minus_w, el)));
    return __fadd_rn(x, c);
}

// e <- (1 - alpha) * e + alpha * rho
__device__ __forceinline__ float ema(float e, float rho, float keep, float alpha) {
    return __fadd_rn(__fmul_rn(keep, e), __fmul_rn(alpha, rho));
}

__device__ __forceinline__ void raise_flags(const Args& a, bool bad) {
    if (__any_sync(kFull, bad) && (threadIdx.x & 31) == 0) atomicOr(a.flags, (unsigned)ECHO_FLAG_RANGE);
}

// ------------------------------------------------------------- stage kernels

// Per-lane view of one group: chunk c in {t, t + L}, elements [4c, 4c + 4).
template <int GROUP>
struct Lane {
    static constexpr int L = GROUP / 8;      // lanes per group
    static constexpr int GPW = 32 / L;       // groups per warp
    int sub, t;
    __device__ __forceinline__ Lane() {
        const int lane = threadIdx.x & 31;
        sub = lane / L;
        t = lane % L;
    }
    __device__ __forceinline__ int chunk(int h) const { return t + h * L; }
};

// Stage 1: quantize the groups [j_begin, j_end) of rank r (none owned by r).
template <int GROUP, int BITS, int QM>
__device__ __forceinline__ void quantize_range(const Args& a, int r, long long j_begin, long long j_end,
                                               long long warp, long long nwarps) {
    using LN = Lane<GROUP>;
    constexpr int L = LN::L, GPW = LN::GPW, Q = (1 << BITS) - 1, CB = GROUP * BITS / 8;
    const LN ln;
    const uint16_t* x = a.in[r];
    float* el_base = a.state ? state_row(a, r) : nullptr;
    float* es_base = a.state ? el_base + a.S : nullptr;
    for (long long j0 = j_begin + warp * GPW; j0 < j_end; j0 += nwarps * GPW) {
        const long long j = j0 + ln.sub;
        const bool act = j < j_end;
        const bool full = (j + 1) * GROUP <= a.n;
        float v[8], el[8], es[8];
        float lmin = __int_as_float(0x7f800000), lmax = -__int_as_float(0x7f800000);
        bool bad = false;
        if (act) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const long long e = j * GROUP + 4 * ln.chunk(h);
                load_x4(x, e, a.n, full, &v[4 * h]);
                if (a.state) {
                    load_f4(el_base, e, a.n, full, &el[4 * h]);
                    load_f4(es_base, e, a.n, full, &es[4 * h]);
                }
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const long long e = j * GROUP + 4 * ln.chunk(h);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int i = 4 * h + k;
                    if (a.state) v[i] = inject(v[i], el[i], es[i], a);
                    if (full || e + k < a.n) {
                        lmin = fminf(lmin, v[i]);
                        lmax = fmaxf(lmax, v[i]);
                        bad |= outside_fp16_domain(v[i]);
                    }
                }
            }
        }
        raise_flags(a, bad);
        const Grid g = make_grid<L, Q, QM>(lmin, lmax);
        if (act) {
            uint8_t* codes = a.a2a_codes + a2a_slot(a, r, j) * CB;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const long long e = j * GROUP + 4 * ln.chunk(h);
                int q[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int i = 4 * h + k;
                    const bool valid = full || e + k < a.n;
                    q[k] = valid ? encode<Q, QM>(v[i], g) : 0;
                    if (a.state) {
                        const float rho = __fsub_rn(v[i], decode(q[k], g.s, g.zf));
                        el[i] = ema(el[i], rho, a.keep_long, a.a_long);
                        es[i] = ema(es[i], rho, a.keep_short, a.a_short);
                    }
                }
                store_chunk_codes<BITS>(codes, ln.chunk(h), pack4<BITS>(q));
                if (a.state) {
                    store_f4(el_base, e, a.n, full, &el[4 * h]);
                    store_f4(es_base, e, a.n, full, &es[4 * h]);
                }
            }
            if (ln.t == 0) a.a2a_params[a2a_slot(a, r, j)] = g.param;
        }
    }
}

// Stage 2: owner o sums and requantizes its groups [j_begin, j_end).
template <int GROUP, int BITS, int QM>
__device__ __forceinline__ void reduce_range(const Args& a, int o, long long j_begin, long long j_end,
                                             long long warp, long long nwarps) {
    using LN = Lane<GROUP>;
    constexpr int L = LN::L, GPW = LN::GPW, Q = (1 << BITS) - 1, CB = GROUP * BITS / 8;
    constexpr int RB = 8;   // ranks whose payload loads are issued together
    const LN ln;
    const uint16_t* x = a.in[o];
    float* el_base = a.state ? state_row(a, o) : nullptr;
    float* es_base = a.state ? el_base + a.S : nullptr;
    for (long long j0 = j_begin + warp * GPW; j0 < j_end; j0 += nwarps * GPW) {
        const long long j = j0 + ln.sub;
        const bool act = j < j_end;
        const bool full = (j + 1) * GROUP <= a.n;
        float xo[8], el[8], es[8], acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) xo[i] = el[i] = es[i] = acc[i] = 0.0f;
        if (act) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const long long e = j * GROUP + 4 * ln.chunk(h);
                load_x4(x, e, a.n, full, &xo[4 * h]);
                if (a.state) {
                    load_f4(el_base, e, a.n, full, &el[4 * h]);
                    load_f4(es_base, e, a.n, full, &es[4 * h]);
                }
            }
            if (a.state) {
#pragma unroll
                for (int i = 0; i < 8; ++i) xo[i] = inject(xo[i], el[i], es[i], a);
            }
        }
        // binary32 sum in rank order 0..P-1: own x' unquantized, others decoded
        for (int r0 = 0; r0 < a.P; r0 += RB) {
            uint32_t cw[RB][2];
            uint32_t pw[RB];
#pragma unroll
            for (int k = 0; k < RB; ++k) {
                const int r = r0 + k;
                cw[k][0] = cw[k][1] = 0u;
                pw[k] = 0u;
                if (act && r < a.P && r != o) {
                    const size_t slot = a2a_slot(a, r, j);
                    const uint8_t* codes = a.a2a_codes + slot * CB;
                    cw[k][0] = load_chunk_codes<BITS>(codes, ln.chunk(0));
                    cw[k][1] = load_chunk_codes<BITS>(codes, ln.chunk(1));
                    pw[k] = a.a2a_params[slot];
                }
            }
#pragma unroll
            for (int k = 0; k < RB; ++k) {
                const int r = r0 + k;
                if (r < a.P) {
                    const float s = param_s(pw[k]);
                    const float z = param_zf<QM>(pw[k], s);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float term = (r == o) ? xo[i] : decode(unpack1<BITS>(cw[k][i >> 2], i & 3), s, z);
                        acc[i] = (r == 0) ? term : __fadd_rn(acc[i], term);
                    }
                }
            }
        }
        float lmin = __int_as_float(0x7f800000), lmax = -__int_as_float(0x7f800000);
        bool bad = false;
        if (act) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const long long e = j * GROUP + 4 * ln.chunk(h);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    if (full || e + k < a.n) {
                        const float v = acc[4 * h + k];
                        lmin = fminf(lmin, v);
                        lmax = fmaxf(lmax, v);
                        bad |= outside_fp16_domain(v);
                    }
                }
            }
        }
        raise_flags(a, bad);
        uint32_t yb[8];
        if (a.P >= 2) {
            const Grid g = make_grid<L, Q, QM>(lmin, lmax);
            if (act) {
                uint8_t* codes = a.g_codes + (size_t)(j - a.g_col_base) * CB;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const long long e = j * GROUP + 4 * ln.chunk(h);
                    int q[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const bool valid = full || e + k < a.n;
                        q[k] = valid ? encode<Q, QM>(acc[4 * h + k], g) : 0;
                        yb[4 * h + k] = f2bf16(decode(q[k], g.s, g.zf));
                    }
                    store_chunk_codes<BITS>(codes, ln.chunk(h), pack4<BITS>(q));
                    if (a.write_outputs) {
                        for (int r = 0; r < a.P; ++r) store_y4(a.out[r], e, a.n, full, &yb[4 * h]);
                    }
                }
                if (ln.t == 0) a.g_params[j - a.g_col_base] = g.param;
            }
        } else if (act) {
            // a single rank sends nothing: its output is its own x'
#pragma unroll
            for (int i = 0; i < 8; ++i) yb[i] = f2bf16(acc[i]);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const long long e = j * GROUP + 4 * ln.chunk(h);
                store_y4(a.out[0], e, a.n, full, &yb[4 * h]);
            }
        }
        if (act && a.state) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const long long e = j * GROUP + 4 * ln.chunk(h);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int i = 4 * h + k;
                    const float rho = __fsub_rn(acc[i], __uint_as_float(yb[i] << 16));
                    el[i] = ema(el[i], rho, a.keep_long, a.a_long);
                    es[i] = ema(es[i], rho, a.keep_short, a.a_short);
                }
                store_f4(el_base, e, a.n, full, &el[4 * h]);
                store_f4(es_base, e, a.n, full, &es[4 * h]);
            }
        }
    }
}

// Stage 3 helper: lane t of a group owns the 8 contiguous elements
// [8t, 8t + 8): their codes are one 32-bit (4-bit codes) or 64-bit (8-bit
// codes) word.
template <int BITS>
__device__ __forceinline__ uint2 load_codes8(const uint8_t* group_codes, int t) {
    if (BITS == 4) return make_uint2(*reinterpret_cast<const uint32_t*>(group_codes + 4 * t), 0u);
    return *reinterpret_cast<const uint2*>(group_codes + 8 * t);
}

}  // namespace echo_dev
