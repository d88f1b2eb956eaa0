// echo_pipeline.cuh -- bulk-copy (TMA) staged versions of the two kernels
// that stream the inputs and the EMA state.
//
// Why: each element of the quantize and reduce passes moves 18 bytes of
// input/state (bf16 x, two fp32 EMAs, read) before any math can start. With
// loads issued from registers, bytes in flight per SM are capped by the
// register file; here one producer lane per CTA streams whole tiles
// (T groups x (bf16 x, e_long, e_short)) into a ring of shared-memory stages
// with cp.async.bulk (the TMA engine, 1-D, no tensor map, no multicast), and
// the consumer warps compute from shared memory and write results straight
// back to HBM. Several 20 KB tiles per CTA are in flight at any time.
//
// Synchronization per stage: full[s] (producer arrive + transaction bytes)
// and empty[s] (one arrive per consumer warp). Every wait is bounded by a
// wall-clock limit: on expiry the kernel sets ECHO_FLAG_TIMEOUT, stops, and
// the producer lane waits (again bounded) for the copies it issued before the
// CTA exits. Partial last groups (not 16-byte sized) take the direct
// register path of echo_kernels.cuh.
#pragma once

#include "echo_kernels.cuh"

namespace echo_dev {

constexpr int kConsumerWarps = 8;
constexpr int kStages = 4;
constexpr int kPipeThreads = (kConsumerWarps + 1) * 32;
constexpr int kTileElems = kConsumerWarps * 32 * 8;           // 2048 elements per tile
constexpr int kStageBytes = kTileElems * (2 + 4 + 4);          // bf16 x + two fp32 EMAs
constexpr int kPipeSmem = kStages * kStageBytes + 2 * kStages * 8 + 16;
constexpr unsigned long long kWaitLimitNs = 1000ull * 1000ull * 1000ull;   // 1 s

// ------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for phase `parity` of `bar` to complete, at most `limit_ns`. Returns
// false on expiry (the caller reports it). `abort` lets other warps of the
// CTA cut the wait short once one of them has given up.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned long long limit_ns,
                                          const volatile int* abort) {
    if (mbar_test(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (true) {
        if (mbar_test(bar, parity)) return true;
        if (abort != nullptr && *abort) return false;
        if (global_ns() - t0 > limit_ns) return false;
    }
}

// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`.
// src, dst and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// ------------------------------------------------------------ tile walk

// A run is a contiguous range of full groups [j0, j1) of one rank. The tile
// sequence of a kernel is the concatenation of its runs cut into tiles of at
// most T groups. The cursor walks it monotonically (tile indices only grow).
struct Tile {
    int rank;
    long long j0;
    int count;
};

template <int GROUP>
struct RunWalker {
    static constexpr int T = kTileElems / GROUP;   // groups per tile
    // kind 0: non-owned runs of every rank (quantize); kind 1: owned runs (reduce)
    int kind;
    long long G, G_full;
    int P;
    int run;            // current run index
    long long base;     // first tile index of the current run
    long long run_j0, run_len;

    __device__ __forceinline__ void load_run() {
        run_j0 = 0;
        run_len = 0;
        if (kind == 0) {
            const int r = run >> 1;
            const long long lo = (long long)r * G / P, hi = (long long)(r + 1) * G / P;
            if ((run & 1) == 0) {
                run_j0 = 0;
                run_len = min(lo, G_full);
            } else {
                run_j0 = hi;
                run_len = max(0LL, G_full - hi);
            }
        } else {
            const long long lo = (long long)run * G / P, hi = (long long)(run + 1) * G / P;
            run_j0 = lo;
            run_len = max(0LL, min(hi, G_full) - lo);
        }
    }
    __device__ __forceinline__ int runs() const { return kind == 0 ? 2 * P : P; }
    __device__ __forceinline__ int rank_of_run() const { return kind == 0 ? (run >> 1) : run; }

    __device__ __forceinline__ RunWalker(int kind_, long long G_, long long G_full_, int P_)
        : kind(kind_), G(G_), G_full(G_full_), P(P_), run(0), base(0) {
        load_run();
    }

    // Tile k (k never decreases between calls); false when past the end.
    __device__ __forceinline__ bool locate(long long k, Tile* t) {
        while (run < runs()) {
            const long long nt = (run_len + T - 1) / T;
            if (k < base + nt) {
                const long long off = (k - base) * T;
                t->rank = rank_of_run();
                t->j0 = run_j0 + off;
                t->count = (int)min((long long)T, run_len - off);
                return true;
            }
            base += nt;
            ++run;
            if (run < runs()) load_run();
        }
        return false;
    }
};

struct PipeShared {
    uint64_t* full;
    uint64_t* empty;
    volatile int* abort;
    uint8_t* stages;
};

__device__ __forceinline__ PipeShared pipe_shared(uint8_t* smem) {
    PipeShared p;
    p.stages = smem;
    p.full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
    p.empty = p.full + kStages;
    p.abort = reinterpret_cast<volatile int*>(p.empty + kStages);
    return p;
}

__device__ __forceinline__ void pipe_init(const PipeShared& p) {
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&p.full[s], 1);
            mbar_init(&p.empty[s], kConsumerWarps);
        }
        *p.abort = 0;
        mbar_fence_init();
    }
    __syncthreads();
}

__device__ __forceinline__ void report_timeout(const Args& a, const PipeShared& p) {
    *p.abort = 1;
    atomicOr(a.flags, (unsigned)ECHO_FLAG_TIMEOUT);
}

// Producer lane: stream tiles of `walker` into the stage ring. `with_state`
// adds the two EMA tiles of the tile's rank.
template <int GROUP>
__device__ __forceinline__ void produce(const Args& a, const PipeShared& p, RunWalker<GROUP>& walker,
                                        bool with_state) {
    long long issued = 0;
    Tile t;
    for (long long k = blockIdx.x; walker.locate(k, &t); k += gridDim.x, ++issued) {
        const int s = (int)(issued % kStages);
        const uint32_t use = (uint32_t)(issued / kStages);
        if (issued >= kStages && !mbar_wait(&p.empty[s], (use & 1u) ^ 1u, kWaitLimitNs, p.abort)) {
            report_timeout(a, p);
            break;
        }
        uint8_t* st = p.stages + (size_t)s * kStageBytes;
        const long long e0 = t.j0 * GROUP;
        const uint32_t xbytes = (uint32_t)t.count * GROUP * 2;
        const uint32_t sbytes = (uint32_t)t.count * GROUP * 4;
        mbar_arrive_expect_tx(&p.full[s], xbytes + (with_state ? 2 * sbytes : 0));
        bulk_load(st, a.in[t.rank] + e0, xbytes, &p.full[s]);
        if (with_state) {
            const float* el = a.state + (size_t)t.rank * 2 * a.S;
            bulk_load(st + kTileElems * 2, el + e0, sbytes, &p.full[s]);
            bulk_load(st + kTileElems * 6, el + a.S + e0, sbytes, &p.full[s]);
        }
    }
    // drain: the last (up to kStages) tiles' copies must land before the CTA
    // may retire, whatever happened to the consumers
    const long long first = issued > kStages ? issued - kStages : 0;
    for (long long i = first; i < issued; ++i) {
        const int s = (int)(i % kStages);
        if (!mbar_wait(&p.full[s], (uint32_t)(i / kStages) & 1u, kWaitLimitNs, nullptr)) {
            atomicOr(a.flags, (unsigned)ECHO_FLAG_TIMEOUT);
        }
    }
}

// ------------------------------------------------------------ quantize

template <int GROUP, int BITS>
__device__ __forceinline__ void quantize_tile_group(const Args& a, const uint8_t* st, const Tile& t, int gi,
                                                    bool act) {
    using LN = Lane<GROUP>;
    constexpr int L = LN::L, Q = (1 << BITS) - 1, CB = GROUP * BITS / 8;
    const LN ln;
    const int r = t.rank;
    const long long j = t.j0 + gi;
    const uint16_t* xs = reinterpret_cast<const uint16_t*>(st) + gi * GROUP;
    const float* els = reinterpret_cast<const float*>(st + kTileElems * 2) + gi * GROUP;
    const float* ess = reinterpret_cast<const float*>(st + kTileElems * 6) + gi * GROUP;
    float v[8], el[8], es[8];
    float lmin = __int_as_float(0x7f800000), lmax = -__int_as_float(0x7f800000);
    bool bad = false;
    if (act) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int c = 4 * ln.chunk(h);
            const uint2 u = *reinterpret_cast<const uint2*>(xs + c);
            v[4 * h + 0] = bf16_lo(u.x);
            v[4 * h + 1] = bf16_hi(u.x);
            v[4 * h + 2] = bf16_lo(u.y);
            v[4 * h + 3] = bf16_hi(u.y);
            if (a.state) {
                const float4 l4 = *reinterpret_cast<const float4*>(els + c);
                const float4 s4 = *reinterpret_cast<const float4*>(ess + c);
                el[4 * h + 0] = l4.x; el[4 * h + 1] = l4.y; el[4 * h + 2] = l4.z; el[4 * h + 3] = l4.w;
                es[4 * h + 0] = s4.x; es[4 * h + 1] = s4.y; es[4 * h + 2] = s4.z; es[4 * h + 3] = s4.w;
            }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (a.state) v[i] = inject(v[i], el[i], es[i], a);
            lmin = fminf(lmin, v[i]);
            lmax = fmaxf(lmax, v[i]);
            bad |= outside_fp16_domain(v[i]);
        }
    }
    raise_flags(a, bad);
    const Grid g = make_grid<L, Q>(lmin, lmax);
    if (!act) return;
    uint8_t* codes = a.a2a_codes + ((size_t)r * a.G + j) * CB;
    float* el_g = a.state ? a.state + (size_t)r * 2 * a.S + j * GROUP : nullptr;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int c = 4 * ln.chunk(h);
        int q[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int i = 4 * h + k;
            q[k] = encode<Q>(v[i], g);
            if (a.state) {
                const float rho = __fsub_rn(v[i], decode(q[k], g.s, g.z));
                el[i] = ema(el[i], rho, a.keep_long, a.a_long);
                es[i] = ema(es[i], rho, a.keep_short, a.a_short);
            }
        }
        store_chunk_codes<BITS>(codes, ln.chunk(h), pack4<BITS>(q));
        if (a.state) {
            __stcs(reinterpret_cast<float4*>(el_g + c), make_float4(el[4 * h], el[4 * h + 1], el[4 * h + 2], el[4 * h + 3]));
            __stcs(reinterpret_cast<float4*>(el_g + a.S + c),
                   make_float4(es[4 * h], es[4 * h + 1], es[4 * h + 2], es[4 * h + 3]));
        }
    }
    if (ln.t == 0) a.a2a_params[(size_t)r * a.G + j] = g.param;
}

template <int GROUP, int BITS>
__global__ void __launch_bounds__(kPipeThreads, 2) k_quantize_tma(const Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const PipeShared p = pipe_shared(smem);
    pipe_init(p);
    const int warp = threadIdx.x >> 5;
    const long long G_full = a.n / GROUP;
    RunWalker<GROUP> walker(0, a.G, G_full, a.P);
    if (warp == kConsumerWarps) {
        if ((threadIdx.x & 31) == 0) produce<GROUP>(a, p, walker, a.state != nullptr);
        return;
    }
    constexpr int GPW = Lane<GROUP>::GPW;
    const int gi = warp * GPW + Lane<GROUP>().sub;
    long long i = 0;
    Tile t;
    for (long long k = blockIdx.x; walker.locate(k, &t); k += gridDim.x, ++i) {
        const int s = (int)(i % kStages);
        if (!mbar_wait(&p.full[s], (uint32_t)(i / kStages) & 1u, kWaitLimitNs, p.abort)) {
            if ((threadIdx.x & 31) == 0) report_timeout(a, p);
            return;
        }
        quantize_tile_group<GROUP, BITS>(a, p.stages + (size_t)s * kStageBytes, t, gi, gi < t.count);
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive(&p.empty[s]);
    }
    // the partial last group (not a multiple of 16 bytes): direct path
    if (G_full < a.G && blockIdx.x == gridDim.x - 1 && warp == 0) {
        const long long j = a.G - 1;
        for (int r = 0; r < a.P; ++r) {
            const long long lo = (long long)r * a.G / a.P, hi = (long long)(r + 1) * a.G / a.P;
            if (j < lo || j >= hi) quantize_range<GROUP, BITS>(a, r, j, j + 1, 0, 1);
        }
    }
}

// ------------------------------------------------------------ reduce

template <int GROUP, int BITS>
__device__ __forceinline__ void reduce_tile_group(const Args& a, const uint8_t* st, const Tile& t, int gi,
                                                  bool act) {
    using LN = Lane<GROUP>;
    constexpr int L = LN::L, Q = (1 << BITS) - 1, CB = GROUP * BITS / 8;
    constexpr int RB = 8;
    const LN ln;
    const int o = t.rank;
    const long long j = t.j0 + gi;
    const uint16_t* xs = reinterpret_cast<const uint16_t*>(st) + gi * GROUP;
    const float* els = reinterpret_cast<const float*>(st + kTileElems * 2) + gi * GROUP;
    const float* ess = reinterpret_cast<const float*>(st + kTileElems * 6) + gi * GROUP;
    float xo[8], acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) xo[i] = acc[i] = 0.0f;
    if (act) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int c = 4 * ln.chunk(h);
            const uint2 u = *reinterpret_cast<const uint2*>(xs + c);
            xo[4 * h + 0] = bf16_lo(u.x);
            xo[4 * h + 1] = bf16_hi(u.x);
            xo[4 * h + 2] = bf16_lo(u.y);
            xo[4 * h + 3] = bf16_hi(u.y);
            if (a.state) {
                const float4 l4 = *reinterpret_cast<const float4*>(els + c);
                const float4 s4 = *reinterpret_cast<const float4*>(ess + c);
                xo[4 * h + 0] = inject(xo[4 * h + 0], l4.x, s4.x, a);
                xo[4 * h + 1] = inject(xo[4 * h + 1], l4.y, s4.y, a);
                xo[4 * h + 2] = inject(xo[4 * h + 2], l4.z, s4.z, a);
                xo[4 * h + 3] = inject(xo[4 * h + 3], l4.w, s4.w, a);
            }
        }
    }
    for (int r0 = 0; r0 < a.P; r0 += RB) {
        uint32_t cw[RB][2];
        uint32_t pw[RB];
#pragma unroll
        for (int k = 0; k < RB; ++k) {
            const int r = r0 + k;
            cw[k][0] = cw[k][1] = 0u;
            pw[k] = 0u;
            if (act && r < a.P && r != o) {
                const size_t slot = (size_t)r * a.G + j;
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
                const float z = param_z(pw[k]);
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
        for (int i = 0; i < 8; ++i) {
            lmin = fminf(lmin, acc[i]);
            lmax = fmaxf(lmax, acc[i]);
            bad |= outside_fp16_domain(acc[i]);
        }
    }
    raise_flags(a, bad);
    uint32_t yb[8];
    if (a.P >= 2) {
        const Grid g = make_grid<L, Q>(lmin, lmax);
        if (!act) return;
        uint8_t* codes = a.g_codes + (size_t)j * CB;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            int q[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                q[k] = encode<Q>(acc[4 * h + k], g);
                yb[4 * h + k] = f2bf16(decode(q[k], g.s, g.z));
            }
            store_chunk_codes<BITS>(codes, ln.chunk(h), pack4<BITS>(q));
        }
        if (ln.t == 0) a.g_params[j] = g.param;
    } else {
        if (!act) return;
#pragma unroll
        for (int i = 0; i < 8; ++i) yb[i] = f2bf16(acc[i]);
#pragma unroll
        for (int h = 0; h < 2; ++h) store_y4(a.out[0], j * GROUP + 4 * ln.chunk(h), a.n, true, &yb[4 * h]);
    }
    if (a.state) {
        float* el_g = a.state + (size_t)o * 2 * a.S + j * GROUP;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int c = 4 * ln.chunk(h);
            const float4 l4 = *reinterpret_cast<const float4*>(els + c);
            const float4 s4 = *reinterpret_cast<const float4*>(ess + c);
            const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
            const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
            float ol[4], os[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int i = 4 * h + k;
                const float rho = __fsub_rn(acc[i], __uint_as_float(yb[i] << 16));
                ol[k] = ema(lv[k], rho, a.keep_long, a.a_long);
                os[k] = ema(sv[k], rho, a.keep_short, a.a_short);
            }
            __stcs(reinterpret_cast<float4*>(el_g + c), make_float4(ol[0], ol[1], ol[2], ol[3]));
            __stcs(reinterpret_cast<float4*>(el_g + a.S + c), make_float4(os[0], os[1], os[2], os[3]));
        }
    }
}

template <int GROUP, int BITS>
__global__ void __launch_bounds__(kPipeThreads, 2) k_reduce_tma(const Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const PipeShared p = pipe_shared(smem);
    pipe_init(p);
    const int warp = threadIdx.x >> 5;
    const long long G_full = a.n / GROUP;
    RunWalker<GROUP> walker(1, a.G, G_full, a.P);
    if (warp == kConsumerWarps) {
        if ((threadIdx.x & 31) == 0) produce<GROUP>(a, p, walker, a.state != nullptr);
        return;
    }
    constexpr int GPW = Lane<GROUP>::GPW;
    const int gi = warp * GPW + Lane<GROUP>().sub;
    long long i = 0;
    Tile t;
    for (long long k = blockIdx.x; walker.locate(k, &t); k += gridDim.x, ++i) {
        const int s = (int)(i % kStages);
        if (!mbar_wait(&p.full[s], (uint32_t)(i / kStages) & 1u, kWaitLimitNs, p.abort)) {
            if ((threadIdx.x & 31) == 0) report_timeout(a, p);
            return;
        }
        reduce_tile_group<GROUP, BITS>(a, p.stages + (size_t)s * kStageBytes, t, gi, gi < t.count);
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive(&p.empty[s]);
    }
    if (G_full < a.G && blockIdx.x == gridDim.x - 1 && warp == 0) {
        const long long j = a.G - 1;
        const int o = (int)((j * a.P + a.P - 1) / a.G);
        reduce_range<GROUP, BITS>(a, o, j, j + 1, 0, 1);
    }
}

// Watchdog self-check: one thread waits, with the same bounded wait the
// pipelines use, on an mbarrier that expects one arrival nobody makes. The
// wait expires after limit_ns, the kernel records ECHO_FLAG_TIMEOUT and
// returns normally, leaving the context usable.
__global__ void k_watchdog_check(uint32_t* flags, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        mbar_fence_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait(&bar, 0u, limit_ns, nullptr)) {
        atomicOr(flags, (unsigned)ECHO_FLAG_TIMEOUT);
    }
}

}  // namespace echo_dev
